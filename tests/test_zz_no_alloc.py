"""mala_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (a plugin inside an engine that owns all device memory, a serving
loop that cannot take the synchronisation a cudaMalloc may bring) call this
entry point instead of mala_decode; its scratch is a fixed device array inside
the library. The checks below call it through the C ABI twice in a row, on two
different inputs, and compare each result with mala_decode's (which takes a
caller-allocated workspace) under the decode tolerances used elsewhere:
O within relative L2 2e-3, LSE within 1e-3, identical per-head counts and
keep maps. The second call also shows that contents left in the shared array
by the first call do not leak into the next result. A third pair of calls
first fills the array (eight splits, every one with tiles) and then asks for
more splits than the cache has tiles, so that the empty splits must be
overwritten with empty partials; that result is also checked against the
fp64 oracle under the same split count.

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import LSE_ABS, O_REL_L2, rel_l2
from workloads import DecodeWorkload, bf16_bits_to_f64, make_decode_inputs

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def _inputs(seed, Lk, with_host=False):
    w = DecodeWorkload("noalloc", 2, 8, 2, Lk, 128, 128, seed=seed)
    inp = make_decode_inputs(w)
    dev = (w, _dev(inp["q"]), _dev(inp["kcache"]), _dev(inp["vcache"]))
    return dev + (inp,) if with_host else dev


def _noalloc(mala, w, q, kc, vc, tau, n_splits):
    B, Hq, d = q.shape
    Lk, Hkv = kc.shape[1], kc.shape[2]
    nk = -(-Lk // w.Bk)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    kept = torch.empty((B * Hq,), dtype=torch.int32, device=q.device)
    km = torch.full((B, Hq, nk), 255, dtype=torch.uint8, device=q.device)
    rc = mala.mala_decode_noalloc(q, kc, vc, o, lse, B, Hq, Hkv, Lk, d, w.scale, tau, w.Bk, n_splits, kept, km)
    assert rc == 0, mala.mala_status_string(rc)
    return o, lse, kept, km


def test_noalloc_decode_matches_decode_twice(cuda_lib):
    mala = cuda_lib
    cases = [(7001, 3000, 1.0, 5), (7002, 2048, 1.0, 0)]
    for seed, Lk, tau, n_splits in cases:
        w, q, kc, vc = _inputs(seed, Lk)
        o2, lse2, kept2, km2 = _noalloc(mala, w, q, kc, vc, tau, n_splits)
        assert mala.mala_check_status() == 0
        o1, lse1, kept1, km1, _ = mala.decode(q, kc, vc, w.scale, tau, w.Bk, n_splits=n_splits, keep_map=True)
        assert mala.mala_check_status() == 0
        e_o = rel_l2(o2.float().cpu().numpy(), o1.float().cpu().numpy())
        e_lse = float((lse2 - lse1).abs().max())
        assert e_o <= O_REL_L2, e_o
        assert e_lse <= LSE_ABS, e_lse
        assert torch.equal(kept1, kept2)
        assert torch.equal(km1, km2)


def test_noalloc_empty_splits_after_a_full_call(cuda_lib):
    mala = cuda_lib
    # fill every split slot of the array's first eight with finite partials
    w, q, kc, vc = _inputs(7003, 3000)
    _noalloc(mala, w, q, kc, vc, 1.0, 8)
    assert mala.mala_check_status() == 0
    # 300 keys are three 128-key tiles: splits 3..7 are empty
    w, q, kc, vc, inp = _inputs(7004, 300, with_host=True)
    o2, lse2, kept2, km2 = _noalloc(mala, w, q, kc, vc, 1.0, 8)
    assert mala.mala_check_status() == 0
    o1, lse1, kept1, km1, _ = mala.decode(q, kc, vc, w.scale, 1.0, w.Bk, n_splits=8, keep_map=True)
    assert mala.mala_check_status() == 0
    assert rel_l2(o2.float().cpu().numpy(), o1.float().cpu().numpy()) <= O_REL_L2
    assert float((lse2 - lse1).abs().max()) <= LSE_ABS
    assert torch.equal(kept1, kept2) and torch.equal(km1, km2)
    ref = oracle.decode(bf16_bits_to_f64(inp["q"]), bf16_bits_to_f64(inp["kcache"]),
                        bf16_bits_to_f64(inp["vcache"]), w.scale, 1.0, w.Bk, 8)
    e_o = rel_l2(o2.float().cpu().numpy().astype(np.float64), ref["o"])
    e_lse = float(np.abs(lse2.cpu().numpy().astype(np.float64) - ref["lse"]).max())
    assert e_o <= O_REL_L2, e_o
    assert e_lse <= LSE_ABS, e_lse
    assert (km2.cpu().numpy() == ref["keep"]).all()


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_lib):
    mala = cuda_lib
    cap = mala.mala_decode_noalloc_max_bytes()
    assert cap == 8 << 20
    # properly sized inputs whose split partials exceed the array: one 128-key
    # tile per sequence cut into 2100 splits needs 2100 * 8 * (128 + 1) * 4
    # bytes of partials (more splits than tiles is allowed)
    B, Hq, Hkv, Lk, d, Bk, n_splits = 1, 8, 8, 128, 128, 128, 2100
    assert mala.mala_decode_workspace_size(B, Hq, d, n_splits) > cap
    w = DecodeWorkload("noalloc_cap", B, Hq, Hkv, Lk, d, Bk, seed=7005)
    inp = make_decode_inputs(w)
    q, kc, vc = _dev(inp["q"]), _dev(inp["kcache"]), _dev(inp["vcache"])
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    kept = torch.empty((B * Hq,), dtype=torch.int32, device="cuda")
    rc = mala.mala_decode_noalloc(q, kc, vc, o, lse, B, Hq, Hkv, Lk, d, w.scale, 1.0, Bk, n_splits, kept, None)
    assert rc == mala.MALA_ERR_WORKSPACE
    assert mala.mala_check_status() == 0
