"""The gate at a near tie, on the GPU.

Parity on the seeded workloads alone never put a tile close to its threshold.
Here tau is tuned, with the fp64 oracle only, so that one chosen tile's gate
margin g = max ratio / (tau / Lq) lands at a set distance from 1 (g scales as
1 / tau while the decisions before the tile stay the same, so one rescaling
of tau and a check suffice). Outside the 1e-3 band the bar allows no
disagreement, so at |g - 1| = 5e-3 and 2e-3 the CUDA decision on that tile,
and on every other tile, must equal the oracle's, both in the forward
(ratio against the evolving state; agihunt.info, "MassAlloc Attention: Let
Attention Allocate Its Own Compute", method paragraphs) and in the backward
(against the final LSE). A case inside the band (|g - 1| = 1e-4) runs the
in-band excuse of tests/parity.py when the two sides happen to differ.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from parity import LSE_ABS, MARGIN, O_REL_L2, compare_bwd_decisions, compare_fwd_decisions, rel_l2
from workloads import TrainWorkload, bf16_bits_to_f64, make_train_inputs

pytestmark = pytest.mark.gpu

CASES = [(512, 64, 64, 5100), (1024, 128, 128, 5101)]


def _dev(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def _case(L, d, Bt, seed):
    w = TrainWorkload("margin", 1, 2, 2, L, d, Bt, Bt, seed=seed)
    inp = make_train_inputs(w)
    return w, inp, tuple(bf16_bits_to_f64(inp[x]) for x in ("q", "k", "v", "do"))


def _closest_site(margin):
    idx = np.argwhere(np.isfinite(margin))
    return tuple(min(idx, key=lambda ix: abs(math.log(margin[tuple(ix)]))))


def tune_fwd(w, qf, kf, vf, target):
    """tau putting the forward margin of one tile at `target` (oracle only)."""
    tau = 1.0
    ref = oracle.fwd(qf, kf, vf, w.scale, tau, w.Bq, w.Bk)
    site = _closest_site(ref["margin"])
    for _ in range(6):
        tau *= ref["margin"][site] / target
        ref = oracle.fwd(qf, kf, vf, w.scale, tau, w.Bq, w.Bk)
        if abs(ref["margin"][site] - target) < 1e-9:
            return tau, site, ref
    raise AssertionError("tau tuning did not settle")


def tune_bwd(w, qf, kf, vf, dof, target):
    """tau putting the backward margin of one tile at `target` (oracle only)."""
    tau = 1.0
    f = oracle.fwd(qf, kf, vf, w.scale, tau, w.Bq, w.Bk)
    b = oracle.bwd(qf, kf, vf, f["o"], dof, f["lse"], w.scale, tau, w.Bq, w.Bk)
    site = _closest_site(b["margin"])
    for _ in range(6):
        tau *= b["margin"][site] / target
        f = oracle.fwd(qf, kf, vf, w.scale, tau, w.Bq, w.Bk)
        b = oracle.bwd(qf, kf, vf, f["o"], dof, f["lse"], w.scale, tau, w.Bq, w.Bk)
        if abs(b["margin"][site] - target) < 1e-9:
            return tau, site, f, b
    raise AssertionError("tau tuning did not settle")


@pytest.mark.parametrize("L,d,Bt,seed", CASES)
@pytest.mark.parametrize("target", [1 - 5e-3, 1 + 5e-3, 1 - 2e-3, 1 + 2e-3, 1 + 1e-4])
def test_fwd_decision_near_threshold(cuda_lib, L, d, Bt, seed, target):
    mala = cuda_lib
    w, inp, (qf, kf, vf, _) = _case(L, d, Bt, seed)
    tau, site, ref = tune_fwd(w, qf, kf, vf, target)
    q, k, v = (_dev(inp[x]) for x in ("q", "k", "v"))
    o, lse, kept, km = mala.forward(q, k, v, w.scale, tau, w.Bq, w.Bk, keep_map=True)
    assert mala.mala_check_status() == 0
    km_h = km.cpu().numpy()
    dec = compare_fwd_decisions(km_h, ref["keep"], ref["margin"], L, w.Bq, w.Bk)
    assert dec["bad"] == 0, dec["bad_sites"]
    if abs(target - 1) >= MARGIN:
        assert km_h[site] == ref["keep"][site]
        assert dec["in_margin"] == 0 and dec["cascaded"] == 0
    assert rel_l2(o.float().cpu().numpy(), ref["o"]) <= O_REL_L2
    assert np.abs(lse.cpu().numpy() - ref["lse"]).max() <= LSE_ABS
    print(f"[gate margin fwd] L={L} target g={target} tau={tau:.6f} site={site} keep={int(km_h[site])} "
          f"in_margin={dec['in_margin']} cascaded={dec['cascaded']}")


@pytest.mark.parametrize("L,d,Bt,seed", CASES)
@pytest.mark.parametrize("target", [1 - 5e-3, 1 + 5e-3, 1 - 2e-3, 1 + 2e-3, 1 + 1e-4])
def test_bwd_decision_near_threshold(cuda_lib, L, d, Bt, seed, target):
    mala = cuda_lib
    w, inp, (qf, kf, vf, dof) = _case(L, d, Bt, seed)
    tau, site, f, b = tune_bwd(w, qf, kf, vf, dof, target)
    q, k, v, do = (_dev(inp[x]) for x in ("q", "k", "v", "do"))
    o, lse, _, kmf = mala.forward(q, k, v, w.scale, tau, w.Bq, w.Bk, keep_map=True)
    assert mala.mala_check_status() == 0
    decf = compare_fwd_decisions(kmf.cpu().numpy(), f["keep"], f["margin"], L, w.Bq, w.Bk)
    assert decf["bad"] == 0, decf["bad_sites"]
    _, _, _, _, kmb = mala.backward(q, k, v, o, do, lse, w.scale, tau, w.Bq, w.Bk, keep_map=True)
    assert mala.mala_check_status() == 0
    kmb_h = kmb.cpu().numpy()
    dec = compare_bwd_decisions(kmb_h, b["keep"], b["margin"], L, w.Bq, w.Bk, decf["diverged_blocks"])
    assert dec["bad"] == 0, dec["bad_sites"]
    if abs(target - 1) >= MARGIN and not decf["diverged_blocks"]:
        assert kmb_h[site] == b["keep"][site]
    print(f"[gate margin bwd] L={L} target g={target} tau={tau:.6f} site={site} keep={int(kmb_h[site])} "
          f"in_margin={dec['in_margin']} excused={dec['excused']}")
