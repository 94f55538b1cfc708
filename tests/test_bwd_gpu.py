"""MALA backward on the GPU (C ABI mala_bwd) against the fp64 oracle.

The oracle's backward consumes the oracle's own forward O / LSE; the CUDA
backward consumes the CUDA forward's O / LSE (as a caller would). Tolerances
and decision rules are in tests/parity.py. Large cases compare sampled query
blocks (dQ rows) and key blocks (dK / dV rows).
"""
import numpy as np
import pytest
import torch

import oracle
from parity import (GRAD_REL_L2, compare_bwd_decisions, compare_fwd_decisions, illegal_untouched, legal_mask,
                    rel_l2)
from workloads import C0, C1, C1_IID, SUBSET_SEED_OFFSET, TrainWorkload, bf16_bits_to_f64, make_train_inputs

pytestmark = pytest.mark.gpu


def _to_dev(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def run_bwd_case(mala, w, tau, L=None, sample=None):
    """sample = (n_query_blocks, n_key_blocks) to compare sampled rows only."""
    L = w.L if L is None else L
    inp = make_train_inputs(w, L=L)
    q, k, v, do = (_to_dev(inp[x]) for x in ("q", "k", "v", "do"))
    o, lse, kept_f, km_f = mala.forward(q, k, v, w.scale, tau, w.Bq, w.Bk, keep_map=True)
    dq, dk, dv, kept_b, km_b = mala.backward(q, k, v, o, do, lse, w.scale, tau, w.Bq, w.Bk, keep_map=True)
    assert mala.mala_check_status() == 0
    qf, kf, vf, dof = (bf16_bits_to_f64(inp[x]) for x in ("q", "k", "v", "do"))
    ref = oracle.fwd(qf, kf, vf, w.scale, tau, w.Bq, w.Bk)
    B, _, Hq, d = qf.shape
    Hkv = kf.shape[2]
    nq, nk = -(-L // w.Bq), -(-L // w.Bk)
    selq = selk = None
    if sample is not None:
        rng = np.random.default_rng(w.seed + SUBSET_SEED_OFFSET)
        selq = [(B - 1, Hq - 1, nq - 1), (0, 0, 0)] + [
            (int(rng.integers(B)), int(rng.integers(Hq)), int(rng.integers(nq))) for _ in range(sample[0] - 2)]
        selk = [(0, 0, 0), (B - 1, Hkv - 1, nk - 1)] + [
            (int(rng.integers(B)), int(rng.integers(Hkv)), int(rng.integers(nk))) for _ in range(sample[1] - 2)]
    refb = oracle.bwd(qf, kf, vf, ref["o"], dof, ref["lse"], w.scale, tau, w.Bq, w.Bk, selq=selq, selk=selk)

    kmf, kmb = km_f.cpu().numpy(), km_b.cpu().numpy()
    assert illegal_untouched(kmb, L, w.Bq, w.Bk)
    fd = compare_fwd_decisions(kmf, ref["keep"], ref["margin"], L, w.Bq, w.Bk)
    assert fd["bad"] == 0, fd["bad_sites"][:10]
    rows = None if selq is None else sorted(set(selq))
    bd = compare_bwd_decisions(kmb, refb["keep"], refb["margin"], L, w.Bq, w.Bk, fd["diverged_blocks"], rows=rows)
    assert bd["bad"] == 0, bd["bad_sites"][:10]
    # nesting on the CUDA outputs: backward keeps only tiles the forward kept
    lm = legal_mask(L, w.Bq, w.Bk)
    viol = (kmb == 1) & (kmf == 0) & lm
    assert viol.sum() <= bd["in_margin"] + bd["excused"], int(viol.sum())
    kb_h = kept_b.cpu().numpy()
    assert (kb_h == (kmb == 1).reshape(kb_h.shape[0], -1).sum(1)).all()

    g = {"dq": _f64(dq), "dk": _f64(dk), "dv": _f64(dv)}
    errs = {}
    if selq is None:
        for name in ("dq", "dk", "dv"):
            if np.abs(refb[name]).max() < 1e-12:
                # exact gradient is zero (e.g. L = 1: dS = P (dP - D) = 0); hold the
                # CUDA result to an absolute bound instead of a relative one
                errs[name] = float(np.abs(g[name]).max())
            else:
                errs[name] = rel_l2(g[name], refb[name])
    else:
        def rows_of(sel, Bt, Lx):
            return [(b, slice(x * Bt, min((x + 1) * Bt, Lx)), h) for (b, h, x) in sorted(set(sel))]
        a = np.concatenate([g["dq"][b, r, h].ravel() for (b, r, h) in rows_of(selq, w.Bq, L)])
        e = np.concatenate([refb["dq"][b, r, h].ravel() for (b, r, h) in rows_of(selq, w.Bq, L)])
        errs["dq"] = rel_l2(a, e)
        for name in ("dk", "dv"):
            a = np.concatenate([g[name][b, r, h].ravel() for (b, r, h) in rows_of(selk, w.Bk, L)])
            e = np.concatenate([refb[name][b, r, h].ravel() for (b, r, h) in rows_of(selk, w.Bk, L)])
            errs[name] = rel_l2(a, e)
    print(f"[bwd parity] L={L} d={d} H={Hq}/{Hkv} Bq={w.Bq} Bk={w.Bk} tau={tau}: "
          + " ".join(f"{n}={v:.3e}" for n, v in errs.items())
          + f" tiles={bd['compared']} in_margin={bd['in_margin']} excused={bd['excused']} kept={int(kb_h.sum())}")
    for name, e in errs.items():
        assert e <= GRAD_REL_L2, (name, e)
    return errs


@pytest.mark.parametrize("tau", [0.0, 1.0])
def test_bwd_c0(cuda_lib, tau):
    run_bwd_case(cuda_lib, C0, tau)


@pytest.mark.parametrize("L,d,Hq,Hkv,Bt,tau", [
    (1000, 128, 4, 2, 128, 1.0),   # ragged, GQA
    (1000, 128, 4, 2, 128, 0.0),
    (777, 64, 2, 1, 64, 1.0),      # two key / query blocks per CTA, ragged, GQA
    (300, 128, 2, 2, 64, 0.5),
    (129, 64, 3, 3, 128, 4.0),
    (1, 128, 2, 1, 128, 1.0),
    (64, 128, 1, 1, 64, 1.0),
])
def test_bwd_small_shapes(cuda_lib, L, d, Hq, Hkv, Bt, tau):
    w = TrainWorkload("small", 1, Hq, Hkv, L, d, Bt, Bt, seed=4000 + L + d)
    run_bwd_case(cuda_lib, w, tau)


@pytest.mark.parametrize("L,d,Hq,Hkv,Bq,Bk,tau", [
    (1000, 128, 4, 2, 64, 128, 1.0),
    (1000, 128, 4, 2, 128, 64, 1.0),
    (777, 64, 2, 1, 128, 64, 0.5),
    (513, 64, 2, 2, 64, 128, 4.0),
    (700, 128, 2, 1, 64, 128, 0.0),
])
def test_bwd_mixed_tiles(cuda_lib, L, d, Hq, Hkv, Bq, Bk, tau):
    w = TrainWorkload("mixed", 1, Hq, Hkv, L, d, Bq, Bk, seed=4200 + L + Bq)
    run_bwd_case(cuda_lib, w, tau)


def test_bwd_batch2(cuda_lib):
    w = TrainWorkload("batch2", 2, 4, 2, 640, 128, 128, 128, seed=4101)
    run_bwd_case(cuda_lib, w, 1.0)


@pytest.mark.parametrize("w,tau", [(C1, 1.0), (C1, 0.0), (C1_IID, 1.0)])
def test_bwd_c1_sampled(cuda_lib, w, tau):
    run_bwd_case(cuda_lib, w, tau, sample=(8, 6))
