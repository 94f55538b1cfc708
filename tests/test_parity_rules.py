"""The comparison rules of tests/parity.py on planted keep maps (CPU).

The GPU parity tests excuse a forward decision only inside the 1e-3 margin
band and, after such an excused flip, the rest of that block's chain (whose
state then differs); a backward decision only inside the band or in a block
whose forward chain diverged. On the seeded workloads the CUDA kernels have
so far never disagreed with the oracle, so these branches are exercised here
on keep maps with planted disagreements.
"""
import numpy as np

from parity import compare_bwd_decisions, compare_fwd_decisions, illegal_untouched, legal_mask


def _maps(L=256, Bt=64):
    lm = legal_mask(L, Bt, Bt)
    keep = np.where(lm, 1, 0).astype(np.uint8)[None, None]
    margin = np.where(lm, 3.0, np.nan)[None, None]
    return keep, margin


def test_identical_maps_pass():
    keep, margin = _maps()
    d = compare_fwd_decisions(keep.copy(), keep, margin, 256, 64, 64)
    assert d["bad"] == 0 and d["in_margin"] == 0 and d["compared"] == 10


def test_in_margin_flip_excuses_the_rest_of_its_chain():
    keep, margin = _maps()
    gpu = keep.copy()
    margin[0, 0, 3, 2] = 1.0 + 5e-4      # in the band
    gpu[0, 0, 3, 2] = 0                   # flipped there ...
    gpu[0, 0, 3, 0] = 0                   # ... and later in the same chain (kb descending)
    d = compare_fwd_decisions(gpu, keep, margin, 256, 64, 64)
    assert d["bad"] == 0 and d["in_margin"] == 1 and d["cascaded"] == 1
    assert d["diverged_blocks"] == {(0, 0, 3)}


def test_flip_outside_band_or_before_divergence_is_bad():
    keep, margin = _maps()
    gpu = keep.copy()
    margin[0, 0, 3, 1] = 1.0 + 5e-4
    gpu[0, 0, 3, 2] = 0        # visited before the in-band tile: not excused
    gpu[0, 0, 3, 1] = 0
    d = compare_fwd_decisions(gpu, keep, margin, 256, 64, 64)
    assert d["bad"] == 1 and d["bad_sites"][0][:4] == (0, 0, 3, 2)
    margin2 = margin.copy()
    margin2[0, 0, 2, 0] = 1.0 + 2e-3   # just outside the band
    gpu2 = keep.copy()
    gpu2[0, 0, 2, 0] = 0
    assert compare_fwd_decisions(gpu2, keep, margin2, 256, 64, 64)["bad"] == 1


def test_bwd_rules():
    keep, margin = _maps()
    gpu = keep.copy()
    gpu[0, 0, 1, 0] = 0
    margin[0, 0, 1, 0] = 1.0 - 9e-4
    gpu[0, 0, 3, 1] = 0                 # out of band but in a diverged forward block
    d = compare_bwd_decisions(gpu, keep, margin, 256, 64, 64, diverged_blocks={(0, 0, 3)})
    assert d["bad"] == 0 and d["in_margin"] == 1 and d["excused"] == 1
    d = compare_bwd_decisions(gpu, keep, margin, 256, 64, 64)
    assert d["bad"] == 1


def test_illegal_entries_untouched():
    keep, _ = _maps()
    km = np.where(legal_mask(256, 64, 64)[None, None], keep, 255).astype(np.uint8)
    assert illegal_untouched(km, 256, 64, 64)
    km[0, 0, 0, 3] = 0
    assert not illegal_untouched(km, 256, 64, 64)
