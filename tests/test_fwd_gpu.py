"""MALA forward on the GPU (C ABI mala_fwd) against the fp64 oracle.

Element-wise comparisons on seeded inputs at sizes the oracle finishes in
seconds: several tiles, a ragged last tile, GQA, both tile sizes, tau = 0
(full attention) and tau > 0. Rules and tolerances are in tests/parity.py.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from parity import (LSE_ABS, O_REL_L2, compare_fwd_decisions, illegal_untouched, rel_l2)
from workloads import C0, C1, C1_IID, TrainWorkload, bf16_bits_to_f64, make_train_inputs

pytestmark = pytest.mark.gpu


def _to_dev(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def _to_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def run_fwd_case(mala, w, tau, L=None, prefetch_v=False):
    L = w.L if L is None else L
    inp = make_train_inputs(w, L=L)
    q, k, v = (_to_dev(inp[x]) for x in ("q", "k", "v"))
    o, lse, kept, km = mala.forward(q, k, v, w.scale, tau, w.Bq, w.Bk, keep_map=True, prefetch_v=prefetch_v)
    assert mala.mala_check_status() == 0
    torch.cuda.synchronize()
    qf, kf, vf = (bf16_bits_to_f64(inp[x]) for x in ("q", "k", "v"))
    ref = oracle.fwd(qf, kf, vf, w.scale, tau, w.Bq, w.Bk)
    km_h = km.cpu().numpy()
    assert illegal_untouched(km_h, L, w.Bq, w.Bk)
    dec = compare_fwd_decisions(km_h, ref["keep"], ref["margin"], L, w.Bq, w.Bk)
    assert dec["bad"] == 0, dec["bad_sites"][:10]
    assert dec["in_margin"] + dec["cascaded"] <= max(2, dec["compared"] // 1000), dec
    kept_h = kept.cpu().numpy()
    assert (kept_h == (km_h == 1).reshape(kept_h.shape[0], -1).sum(1)).all()
    e_o = rel_l2(_to_f64(o), ref["o"])
    e_lse = float(np.abs(lse.cpu().numpy().astype(np.float64) - ref["lse"]).max())
    assert e_o <= O_REL_L2, e_o
    assert e_lse <= LSE_ABS, e_lse
    if tau == 0:
        assert (km_h == 1).sum() == (ref["keep"] == 1).sum()
    print(f"[fwd parity{' prefetch_v' if prefetch_v else ''}] L={L} d={w.d} H={w.Hq}/{w.Hkv} Bq={w.Bq} "
          f"Bk={w.Bk} tau={tau}: o_rel_l2={e_o:.3e} "
          f"lse_abs={e_lse:.3e} tiles={dec['compared']} in_margin={dec['in_margin']} cascaded={dec['cascaded']} "
          f"kept={int(kept_h.sum())}")
    return {"o_rel_l2": e_o, "lse_abs": e_lse, "o": o, "lse": lse, "kept": kept, "km": km,
            **{k_: v_ for k_, v_ in dec.items() if k_ != "diverged_blocks"}}


@pytest.mark.parametrize("tau", [0.0, 1.0])
def test_fwd_c0(cuda_lib, tau):
    run_fwd_case(cuda_lib, C0, tau)


@pytest.mark.parametrize("L,d,Hq,Hkv,Bt,tau", [
    (1000, 128, 4, 2, 128, 1.0),   # ragged last tile, GQA
    (1000, 128, 4, 2, 128, 0.0),
    (777, 64, 2, 1, 64, 1.0),      # two query blocks per CTA, ragged, GQA
    (300, 128, 2, 2, 64, 0.5),
    (129, 64, 3, 3, 128, 4.0),     # one row past a tile boundary
    (1, 128, 2, 1, 128, 1.0),      # a single row
    (64, 128, 1, 1, 64, 1.0),
])
def test_fwd_small_shapes(cuda_lib, L, d, Hq, Hkv, Bt, tau):
    w = TrainWorkload("small", 1, Hq, Hkv, L, d, Bt, Bt, seed=3000 + L + d)
    run_fwd_case(cuda_lib, w, tau)


@pytest.mark.parametrize("L,d,Hq,Hkv,Bq,Bk,tau", [
    (1000, 128, 4, 2, 64, 128, 1.0),   # two query blocks per key tile, ragged, GQA
    (1000, 128, 4, 2, 128, 64, 1.0),   # two key blocks per 128 keys
    (777, 64, 2, 1, 128, 64, 0.5),
    (513, 64, 2, 2, 64, 128, 4.0),
    (700, 128, 2, 1, 128, 64, 0.0),
])
def test_fwd_mixed_tiles(cuda_lib, L, d, Hq, Hkv, Bq, Bk, tau):
    w = TrainWorkload("mixed", 1, Hq, Hkv, L, d, Bq, Bk, seed=3200 + L + Bq)
    run_fwd_case(cuda_lib, w, tau)


def test_fwd_batch2(cuda_lib):
    w = TrainWorkload("batch2", 2, 4, 4, 640, 128, 128, 128, seed=3101)
    run_fwd_case(cuda_lib, w, 1.0)


@pytest.mark.parametrize("w,tau", [(C1, 0.0), (C1, 1.0), (C1_IID, 0.0), (C1_IID, 1.0)])
def test_fwd_c1(cuda_lib, w, tau):
    run_fwd_case(cuda_lib, w, tau)


def pair_v_tiles(km, L, Bq):
    """V tiles a gated forward loads: each CTA owns a pair of 128-row query tiles
    of one (b, hq), and a key tile's V is loaded once if some query block of the
    pair keeps it (agihunt.info MALA digest, method paragraphs: a skipped tile
    does no V load)."""
    B, H, nq, nk = km.shape
    per = 256 // Bq
    total = 0
    for pr in range(-(-L // 256)):
        blocks = list(range(pr * per, min((pr + 1) * per, nq)))
        total += int((km[:, :, blocks, :] == 1).any(axis=2).sum())
    return total


@pytest.mark.parametrize("tau,Bq", [(1.0, 128), (16.0, 128), (16.0, 64)])
def test_fwd_loads_v_only_for_kept_tiles(cuda_lib, tau, Bq):
    mala = cuda_lib
    L = 2048
    w = TrainWorkload("vtiles", 1, 4, 2, L, 128, Bq, 128, seed=3300)
    inp = make_train_inputs(w)
    q, k, v = (_to_dev(inp[x]) for x in ("q", "k", "v"))
    counter = torch.zeros(1, dtype=torch.int64, device="cuda")
    assert mala.mala_test_hooks(0, -1, counter) == 0
    try:
        o, lse, kept, km = mala.forward(q, k, v, w.scale, tau, w.Bq, w.Bk, keep_map=True)
        assert mala.mala_check_status() == 0
    finally:
        mala.mala_test_hooks(0, -1, None)
    km_h = km.cpu().numpy()
    ref = oracle.fwd(*(bf16_bits_to_f64(inp[x]) for x in ("q", "k", "v")), w.scale, tau, w.Bq, w.Bk)
    dec = compare_fwd_decisions(km_h, ref["keep"], ref["margin"], L, w.Bq, w.Bk)
    assert dec["bad"] == 0, dec["bad_sites"][:10]
    loaded = int(counter.item())
    assert loaded == pair_v_tiles(km_h, L, w.Bq)
    # key tiles the CTAs walk: kb = 0 .. the tile of the pair's last row
    visits = w.B * w.Hq * sum((min(pr * 256 + 256, L) - 1) // w.Bk + 1 for pr in range(-(-L // 256)))
    print(f"[fwd V tiles] tau={tau} Bq={Bq}: loaded {loaded} of {visits} walked")
    if tau >= 16:
        assert loaded < 0.9 * visits


@pytest.mark.parametrize("L,d,Hq,Hkv,Bq,Bk,tau", [
    (1000, 128, 4, 2, 128, 128, 1.0),  # ragged, GQA
    (777, 64, 2, 1, 64, 64, 1.0),
    (1000, 128, 4, 2, 64, 128, 4.0),   # many skips, two query blocks per tile
    (513, 64, 2, 2, 128, 64, 16.0),
])
def test_fwd_prefetch_v_same_results(cuda_lib, L, d, Hq, Hkv, Bq, Bk, tau):
    """mala_fwd_ex with MALA_FWD_PREFETCH_V: V of every tile fetched ahead of the
    vote. Decisions and arithmetic are those of the default path, so the outputs
    match the oracle and equal the default path's bit for bit."""
    w = TrainWorkload("prefetch", 1, Hq, Hkv, L, d, Bq, Bk, seed=3400 + L + Bq)
    a = run_fwd_case(cuda_lib, w, tau, prefetch_v=True)
    b = run_fwd_case(cuda_lib, w, tau, prefetch_v=False)
    for name in ("o", "lse", "kept", "km"):
        assert torch.equal(a[name], b[name]), name


def test_fwd_prefetch_v_loads_every_tile(cuda_lib):
    mala = cuda_lib
    L = 2048
    w = TrainWorkload("vtiles", 1, 4, 2, L, 128, 128, 128, seed=3300)
    inp = make_train_inputs(w)
    q, k, v = (_to_dev(inp[x]) for x in ("q", "k", "v"))
    counter = torch.zeros(1, dtype=torch.int64, device="cuda")
    assert mala.mala_test_hooks(0, -1, counter) == 0
    try:
        _, _, _, km = mala.forward(q, k, v, w.scale, 16.0, w.Bq, w.Bk, keep_map=True, prefetch_v=True)
        assert mala.mala_check_status() == 0
    finally:
        mala.mala_test_hooks(0, -1, None)
    visits = w.B * w.Hq * sum((min(pr * 256 + 256, L) - 1) // w.Bk + 1 for pr in range(-(-L // 256)))
    assert int(counter.item()) == visits
    assert pair_v_tiles(km.cpu().numpy(), L, w.Bq) < 0.9 * visits  # tau = 16 skips, the V loads do not


def test_fwd_ex_rejects_unknown_flags(cuda_lib):
    mala = cuda_lib
    L, d = 128, 128  # properly sized buffers, although the flags are checked before anything is read
    q = torch.zeros((1, L, 1, d), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((1, 1, L), dtype=torch.float32, device="cuda")
    kept = torch.empty((1,), dtype=torch.int32, device="cuda")
    wsb = mala.mala_fwd_workspace_size(1, 1, L, d)
    ws = torch.empty((wsb,), dtype=torch.uint8, device="cuda")
    rc = mala.mala_fwd_ex(q, q, q, o, lse, 1, 1, 1, L, d, 0.1, 1.0, 128, 128, ws, wsb, kept, None, None, flags=2)
    assert rc == mala.MALA_ERR_INVALID_ARG
    rc = mala.mala_fwd_ex(q, q, q, o, lse, 1, 1, 1, L, d, 0.1, 1.0, 128, 128, ws, wsb, kept, None, None,
                          flags=mala.MALA_FWD_PREFETCH_V)
    assert rc == mala.MALA_OK and mala.mala_check_status() == 0
