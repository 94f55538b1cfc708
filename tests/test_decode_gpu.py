"""MALA decode on the GPU (C ABI mala_decode) against the fp64 oracle.

The keep decisions of one split form a chain (newest tile to oldest); the
comparison follows the same rule as the forward (tests/parity.py): identical
except in margin, with the rest of a chain excused after an in-margin flip.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import LSE_ABS, MARGIN, O_REL_L2, rel_l2
from workloads import C4, DecodeWorkload, bf16_bits_to_f64, make_decode_inputs

pytestmark = pytest.mark.gpu


def _to_dev(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def compare_decode_decisions(gpu_keep, ref_keep, ref_margin, nk, n_splits, rows):
    T = -(-nk // n_splits)
    out = {"bad": 0, "in_margin": 0, "cascaded": 0, "compared": 0, "bad_sites": []}
    for (b, h) in rows:
        for s in range(n_splits):
            t0, t1 = min(s * T, nk), min((s + 1) * T, nk)
            diverged = False
            for kb in range(t1 - 1, t0 - 1, -1):
                out["compared"] += 1
                a, o = int(gpu_keep[b, h, kb]), int(ref_keep[b, h, kb])
                if a == o:
                    continue
                g = ref_margin[b, h, kb]
                if diverged:
                    out["cascaded"] += 1
                elif np.isfinite(g) and abs(g - 1.0) < MARGIN:
                    out["in_margin"] += 1
                    diverged = True
                else:
                    out["bad"] += 1
                    out["bad_sites"].append((b, h, kb, a, o, float(g)))
    return out


def run_decode_case(mala, w, tau, n_splits=0, Lk=None, sample_rows=None, workers=1):
    Lk = w.Lk if Lk is None else Lk
    inp = make_decode_inputs(w, Lk=Lk, workers=workers)
    q, kc, vc = (_to_dev(inp[x]) for x in ("q", "kcache", "vcache"))
    o, lse, kept, km, ns = mala.decode(q, kc, vc, w.scale, tau, w.Bk, n_splits=n_splits, keep_map=True)
    assert mala.mala_check_status() == 0
    B, Hq, d = inp["q"].shape
    Hkv = inp["kcache"].shape[2]
    G = Hq // Hkv
    nk = -(-Lk // w.Bk)
    o_h = o.float().cpu().numpy().astype(np.float64)
    lse_h = lse.cpu().numpy().astype(np.float64)
    km_h = km.cpu().numpy()
    kept_h = kept.cpu().numpy()
    assert np.isin(km_h, (0, 1)).all()
    assert (kept_h == km_h.reshape(B * Hq, -1).sum(1)).all()
    rows = sample_rows if sample_rows is not None else [(b, h) for b in range(B) for h in range(Hq)]
    ref_keep = np.zeros((B, Hq, nk), dtype=np.uint8)
    ref_margin = np.full((B, Hq, nk), np.nan)
    ref_o = np.zeros((B, Hq, d))
    ref_lse = np.zeros((B, Hq))
    for (b, h) in rows:  # one (b, query head) at a time, on its KV slice
        hk = h // G
        r = oracle.decode(bf16_bits_to_f64(inp["q"][b:b + 1, h:h + 1]),
                          bf16_bits_to_f64(inp["kcache"][b:b + 1, :, hk:hk + 1]),
                          bf16_bits_to_f64(inp["vcache"][b:b + 1, :, hk:hk + 1]), w.scale, tau, w.Bk, ns)
        ref_keep[b, h], ref_margin[b, h] = r["keep"][0, 0], r["margin"][0, 0]
        ref_o[b, h], ref_lse[b, h] = r["o"][0, 0], r["lse"][0, 0]
    dec = compare_decode_decisions(km_h, ref_keep, ref_margin, nk, ns, rows)
    assert dec["bad"] == 0, dec["bad_sites"][:10]
    assert dec["in_margin"] + dec["cascaded"] <= max(2, dec["compared"] // 1000), dec
    sel_o = np.stack([o_h[b, h] for (b, h) in rows])
    sel_ref = np.stack([ref_o[b, h] for (b, h) in rows])
    e_o = rel_l2(sel_o, sel_ref)
    e_lse = max(abs(lse_h[b, h] - ref_lse[b, h]) for (b, h) in rows)
    print(f"[decode parity] B={B} H={Hq}/{Hkv} Lk={Lk} d={d} Bk={w.Bk} tau={tau} splits={ns}: "
          f"o_rel_l2={e_o:.3e} lse_abs={e_lse:.3e} tiles={dec['compared']} in_margin={dec['in_margin']} "
          f"kept={int(sum(kept_h[b * Hq + h] for (b, h) in rows))}/{len(rows) * nk}")
    assert e_o <= O_REL_L2, e_o
    assert e_lse <= LSE_ABS, e_lse


@pytest.mark.parametrize("Lk,d,Bk,tau,n_splits", [
    (2000, 128, 128, 1.0, 3),
    (2000, 128, 128, 0.0, 3),
    (4096, 128, 128, 1.0, 1),
    (4096, 128, 128, 1.0, 0),      # default split count
    (1000, 64, 64, 1.0, 4),        # ragged last tile
    (777, 128, 64, 0.5, 5),
    (1, 128, 128, 1.0, 1),         # one key
    (300, 64, 128, 4.0, 7),        # more splits than tiles
])
def test_decode_small(cuda_lib, Lk, d, Bk, tau, n_splits):
    w = DecodeWorkload("dec_small", 2, 8, 2, Lk, d, Bk, seed=5000 + Lk + d)
    run_decode_case(cuda_lib, w, tau, n_splits=n_splits)


def test_decode_gqa8(cuda_lib):
    w = DecodeWorkload("dec_gqa8", 1, 16, 2, 3000, 128, 128, seed=5101)
    run_decode_case(cuda_lib, w, 1.0, n_splits=4)


@pytest.mark.parametrize("Hq,Hkv,Lk,d,Bk,tau,n_splits", [
    (4, 2, 2500, 128, 128, 1.0, 3),    # two heads per group: one (key, head) value per lane
    (6, 2, 2500, 128, 128, 1.0, 2),    # three heads padded to four
    (4, 2, 1500, 64, 128, 0.5, 3),     # d = 64
    (6, 2, 900, 64, 64, 2.0, 2),       # d = 64, 64-key tiles, padded heads
])
def test_decode_group_sizes(cuda_lib, Hq, Hkv, Lk, d, Bk, tau, n_splits):
    """Group sizes and tile shapes of the batched scoring: the (step, head) dot
    products of a tile are reduced together and each lane keeps one or two of
    them; padded heads take part in the reduction and are never gated."""
    w = DecodeWorkload("dec_groups", 2, Hq, Hkv, Lk, d, Bk, seed=5200 + Hq + Lk + d)
    run_decode_case(cuda_lib, w, tau, n_splits=n_splits)
