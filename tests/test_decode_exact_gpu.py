"""Split-independent decode on the GPU (C ABI mala_decode_exact) against the
fp64 oracle's single sequential pass.

The forward gate of the last query row visits the key tiles from the newest
to the oldest against the state over the kept tiles, the first tile kept
(agihunt.info, "MassAlloc Attention: Let Attention Allocate Its Own Compute",
method paragraphs). mala_decode_exact must reach that single pass's decisions
whatever split of the tiles it uses for the PV work: the decisions are
compared with oracle.decode_single_pass (one chain per row, the chain rule of
tests/parity.py) and must be the same for every split count; O and LSE are
held to the usual tolerances.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import LSE_ABS, O_REL_L2, rel_l2
from test_decode_gpu import compare_decode_decisions
from workloads import C4, SUBSET_SEED_OFFSET, DecodeWorkload, bf16_bits_to_f64, default_workers, make_decode_inputs

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def run_case(mala, w, tau, split_counts, rows=None, workers=1):
    inp = make_decode_inputs(w, workers=workers)
    q, kc, vc = (_dev(inp[x]) for x in ("q", "kcache", "vcache"))
    B, Hq, d = inp["q"].shape
    nk = -(-w.Lk // w.Bk)
    res = [mala.decode_exact(q, kc, vc, w.scale, tau, w.Bk, n_splits=s, keep_map=True) for s in split_counts]
    assert mala.mala_check_status() == 0
    km0 = res[0][3].cpu().numpy()
    for r in res[1:]:  # the decisions do not depend on the split
        assert np.array_equal(r[3].cpu().numpy(), km0)
        assert torch.equal(r[2], res[0][2])
    if rows is None:
        rows = [(b, h) for b in range(B) for h in range(Hq)]
    ref = oracle.decode_single_pass(bf16_bits_to_f64(inp["q"]), bf16_bits_to_f64(inp["kcache"]),
                                    bf16_bits_to_f64(inp["vcache"]), w.scale, tau, w.Bk, sel=rows)
    dec = compare_decode_decisions(km0, ref["keep"], ref["margin"], nk, 1, rows)
    assert dec["bad"] == 0, dec["bad_sites"][:10]
    assert dec["in_margin"] + dec["cascaded"] <= max(2, dec["compared"] // 1000), dec
    kept = res[0][2].cpu().numpy()
    for (b, h) in rows:
        assert kept[b * Hq + h] == int((km0[b, h] == 1).sum())
    errs = []
    for (o, lse, _, _, ns) in res:
        o_h = o.float().cpu().numpy().astype(np.float64)
        lse_h = lse.cpu().numpy().astype(np.float64)
        e_o = rel_l2(np.stack([o_h[b, h] for (b, h) in rows]), np.stack([ref["o"][b, h] for (b, h) in rows]))
        e_lse = max(abs(lse_h[b, h] - ref["lse"][b, h]) for (b, h) in rows)
        assert e_o <= O_REL_L2, (ns, e_o)
        assert e_lse <= LSE_ABS, (ns, e_lse)
        errs.append((ns, e_o, e_lse))
    print(f"[decode exact parity] B={B} H={Hq}/{w.Hkv} Lk={w.Lk} d={w.d} Bk={w.Bk} tau={tau}: "
          + " ".join(f"S={ns}: o={eo:.2e} lse={el:.2e}" for ns, eo, el in errs)
          + f" tiles={dec['compared']} in_margin={dec['in_margin']} kept={int(kept.sum())}")


@pytest.mark.parametrize("B,Hq,Hkv,Lk,d,Bk,tau", [
    (2, 8, 2, 5000, 128, 128, 1.0),     # ragged last tile, GQA
    (2, 8, 2, 5000, 128, 128, 0.0),
    (3, 4, 4, 3333, 64, 64, 0.5),
    (1, 16, 2, 8192, 128, 128, 4.0),    # group of 8
    (4, 2, 1, 1, 128, 128, 1.0),        # a single key
    (2, 6, 2, 700, 128, 64, 16.0),
])
def test_decode_exact(cuda_lib, B, Hq, Hkv, Lk, d, Bk, tau):
    w = DecodeWorkload("exact", B, Hq, Hkv, Lk, d, Bk, seed=8000 + Lk + Hq)
    run_case(cuda_lib, w, tau, split_counts=(1, 3, 7, 40))


def test_decode_exact_fullsize_sampled(cuda_lib):
    """The 128K decode workload; 12 seeded (b, head) rows checked against the oracle."""
    rng = np.random.default_rng(C4.seed + SUBSET_SEED_OFFSET + 3)
    rows = sorted({(0, 0), (C4.B - 1, C4.Hq - 1)} | {(int(rng.integers(C4.B)), int(rng.integers(C4.Hq)))
                                                       for _ in range(10)})
    run_case(cuda_lib, C4, 1.0, split_counts=(0, 1), rows=rows, workers=default_workers())


def test_decode_exact_long_split_segments(cuda_lib):
    """A split of more than 1024 tiles (one split over 70000 keys in 64-key
    tiles) is listed and streamed in segments; two splits take one each."""
    w = DecodeWorkload("exact_long", 1, 4, 2, 70000, 64, 64, seed=8101)
    run_case(cuda_lib, w, 1.0, split_counts=(1, 2))
