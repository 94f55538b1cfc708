"""Failure paths on the GPU: an expired bounded wait and a V value outside
the fp16 range, each reported by mala_check_status, with the context left
usable and the next call correct.

A bounded wait is made to expire without any fault: the test hooks
(mala_test_hooks) shorten every wait to a few milliseconds and make one
role of the kernel wait, before a chosen key tile, on a barrier that nothing
completes. The kernel then raises its abort flag and the device status word,
every role leaves its loop, the copies and MMAs in flight are drained, the
tensor memory is freed, and mala_check_status returns
MALA_ERR_DEVICE_TIMEOUT. The same inputs then go through a normal call, which
must match the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import GRAD_REL_L2, LSE_ABS, O_REL_L2, rel_l2
from workloads import DecodeWorkload, TrainWorkload, bf16_bits_to_f64, make_decode_inputs, make_train_inputs

pytestmark = pytest.mark.gpu

WAIT_NS = 5_000_000  # 5 ms per wait while a stall is planted


def _dev(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


class stalled:
    """Plant a stall before key tile `tile` (and short waits) for the calls inside."""

    def __init__(self, mala, tile):
        self.mala, self.tile = mala, tile

    def __enter__(self):
        assert self.mala.mala_test_hooks(WAIT_NS, self.tile, None) == 0

    def __exit__(self, *exc):
        self.mala.mala_test_hooks(0, -1, None)
        return False


def _train(L=1024, Hq=4, Hkv=2, seed=4100):
    w = TrainWorkload("failure", 1, Hq, Hkv, L, 128, 128, 128, seed=seed)
    inp = make_train_inputs(w)
    return w, inp, tuple(_dev(inp[x]) for x in ("q", "k", "v", "do"))


@pytest.mark.parametrize("tau,tile", [(1.0, 2), (0.0, 1), (1.0, 0)])
def test_fwd_wait_expires_then_recovers(cuda_lib, tau, tile):
    mala = cuda_lib
    w, inp, (q, k, v, _) = _train()
    with stalled(mala, tile):
        mala.forward(q, k, v, w.scale, tau, w.Bq, w.Bk)
        rc = mala.mala_check_status()
    assert rc == mala.MALA_ERR_DEVICE_TIMEOUT, mala.mala_status_string(rc)
    assert mala.mala_check_status() == 0  # the status word was cleared
    o, lse, kept, _ = mala.forward(q, k, v, w.scale, tau, w.Bq, w.Bk)
    assert mala.mala_check_status() == 0
    ref = oracle.fwd(*(bf16_bits_to_f64(inp[x]) for x in ("q", "k", "v")), w.scale, tau, w.Bq, w.Bk)
    assert rel_l2(_f64(o), ref["o"]) <= O_REL_L2
    assert np.abs(lse.cpu().numpy() - ref["lse"]).max() <= LSE_ABS


@pytest.mark.parametrize("tau,tile", [(1.0, 3), (0.0, 0)])
def test_bwd_wait_expires_then_recovers(cuda_lib, tau, tile):
    mala = cuda_lib
    w, inp, (q, k, v, do) = _train(seed=4101)
    o, lse, _, _ = mala.forward(q, k, v, w.scale, tau, w.Bq, w.Bk)
    assert mala.mala_check_status() == 0
    with stalled(mala, tile):
        mala.backward(q, k, v, o, do, lse, w.scale, tau, w.Bq, w.Bk)
        rc = mala.mala_check_status()
    assert rc == mala.MALA_ERR_DEVICE_TIMEOUT, mala.mala_status_string(rc)
    dq, dk, dv, _, _ = mala.backward(q, k, v, o, do, lse, w.scale, tau, w.Bq, w.Bk)
    assert mala.mala_check_status() == 0
    qf, kf, vf, dof = (bf16_bits_to_f64(inp[x]) for x in ("q", "k", "v", "do"))
    # the backward consumes the CUDA forward's O and LSE (checked in the forward tests)
    ref = oracle.bwd(qf, kf, vf, _f64(o), dof, lse.cpu().numpy().astype(np.float64), w.scale, tau, w.Bq, w.Bk)
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        assert rel_l2(_f64(t), ref[name]) <= GRAD_REL_L2, name


@pytest.mark.parametrize("tile", [0, 4])
def test_decode_wait_expires_then_recovers(cuda_lib, tile):
    mala = cuda_lib
    wd = DecodeWorkload("failure_decode", 2, 8, 2, 3000, 128, 128, seed=4102)
    inp = make_decode_inputs(wd)
    q, kc, vc = (_dev(inp[x]) for x in ("q", "kcache", "vcache"))
    with stalled(mala, tile):
        mala.decode(q, kc, vc, wd.scale, 1.0, wd.Bk, n_splits=2)
        rc = mala.mala_check_status()
    assert rc == mala.MALA_ERR_DEVICE_TIMEOUT, mala.mala_status_string(rc)
    o, lse, _, _, ns = mala.decode(q, kc, vc, wd.scale, 1.0, wd.Bk, n_splits=2)
    assert mala.mala_check_status() == 0
    ref = oracle.decode(*(bf16_bits_to_f64(inp[x]) for x in ("q", "kcache", "vcache")), wd.scale, 1.0, wd.Bk, ns)
    assert rel_l2(_f64(o), ref["o"]) <= O_REL_L2
    assert np.abs(lse.cpu().numpy() - ref["lse"]).max() <= LSE_ABS


def test_fwd_v_outside_fp16_range_is_reported(cuda_lib):
    mala = cuda_lib
    w, inp, (q, k, v, _) = _train(L=300, seed=4103)
    vbad = v.clone()
    vbad[0, 17, 1, 5] = 1.0e5  # representable in bf16, beyond the fp16 range the PV product reads
    mala.forward(q, k, vbad, w.scale, 1.0, w.Bq, w.Bk)
    rc = mala.mala_check_status()
    assert rc == mala.MALA_ERR_RANGE, mala.mala_status_string(rc)
    o, lse, _, _ = mala.forward(q, k, v, w.scale, 1.0, w.Bq, w.Bk)
    assert mala.mala_check_status() == 0
    ref = oracle.fwd(*(bf16_bits_to_f64(inp[x]) for x in ("q", "k", "v")), w.scale, 1.0, w.Bq, w.Bk)
    assert rel_l2(_f64(o), ref["o"]) <= O_REL_L2


def test_hooks_reject_bad_stall(cuda_lib):
    assert cuda_lib.mala_test_hooks(0, -2, None) == cuda_lib.MALA_ERR_INVALID_ARG
    assert cuda_lib.mala_test_hooks(0, -1, None) == 0
