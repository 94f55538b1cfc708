"""Matched-work diagnostics on the CUDA forward's decisions.

The fidelity comparison of the pages (agihunt.info, "MassAlloc Attention: Let
Attention Allocate Its Own Compute", fidelity paragraphs: MALA against a
reference-mass oracle with the same key-slot budget, omitted probability mass
and output error) is computed by oracle/matched_work.py. Here it is fed the
keep map that mala_fwd produced on the 8K workload and compared with the same
analysis of the fp64 oracle's own decisions: the key slots per query, the
omitted masses and the output errors must agree exactly wherever the two keep
maps agree, and the maps may differ only in the gate's 1e-3 margin band.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.matched_work import matched_work, summary
from parity import compare_fwd_decisions
from workloads import C1, bf16_bits_to_f64, make_train_inputs

pytestmark = pytest.mark.gpu

HEADS = [(0, 3), (0, 11)]


def test_matched_work_of_cuda_keep_map_c1(cuda_lib):
    mala = cuda_lib
    w = C1
    inp = make_train_inputs(w)
    q, k, v = (torch.from_numpy(inp[x].view(np.int16)).view(torch.bfloat16).cuda() for x in ("q", "k", "v"))
    _, _, _, km = mala.forward(q, k, v, w.scale, 1.0, w.Bq, w.Bk, keep_map=True)
    assert mala.mala_check_status() == 0
    km_cuda = km.cpu().numpy()
    kept_cuda = (km_cuda == 1).astype(np.uint8)  # illegal entries hold the fill value 255
    qf, kf, vf = (bf16_bits_to_f64(inp[x]) for x in ("q", "k", "v"))
    nq = -(-w.L // w.Bq)
    sel = [(b, h, qb) for (b, h) in HEADS for qb in range(nq)]
    ref = oracle.fwd(qf, kf, vf, w.scale, 1.0, w.Bq, w.Bk, sel=sel)
    dec = compare_fwd_decisions(km_cuda, ref["keep"], ref["margin"], w.L, w.Bq, w.Bk, rows=sel)
    assert dec["bad"] == 0, dec["bad_sites"][:10]
    kept_ora = (ref["keep"] == 1).astype(np.uint8)
    r_cuda = matched_work(qf, kf, vf, w.scale, 1.0, w.Bq, w.Bk, heads=HEADS, keep=kept_cuda)
    r_ora = matched_work(qf, kf, vf, w.scale, 1.0, w.Bq, w.Bk, heads=HEADS, keep=kept_ora)
    # rows of blocks whose decisions agree must give identical figures
    same = np.concatenate([[bool((kept_cuda[b, h, qb] == kept_ora[b, h, qb]).all())] * min(w.Bq, w.L - qb * w.Bq)
                           for (b, h) in HEADS for qb in range(nq)])
    assert same.mean() > 0.99
    for name in r_cuda:
        assert np.abs(r_cuda[name][same] - r_ora[name][same]).max() < 1e-12, name
    s_c, s_o = summary(r_cuda), summary(r_ora)
    assert abs(s_c["slot_frac"] - s_o["slot_frac"]) < 1e-3
    assert (r_cuda["omit_mala"] < 1.0 / 2.0).all()  # the omitted-mass bound tau / (1 + tau) at tau = 1
    print(f"[matched work, CUDA keep map, 8K, heads {HEADS}] slots {s_c['slot_frac']:.4f} of live keys; omitted "
          f"mass MALA {s_c['omit_mala_mean']:.3e} vs reference {s_c['omit_ref_mean']:.3e}; output error MALA "
          f"{s_c['err_mala_mean']:.3e} vs reference {s_c['err_ref_mean']:.3e}")
