"""Full-size workloads in the launch configuration bench.py times, checked on
sampled outputs the oracle can compute one by one.

  32K GQA (B=1, Hq=32, Hkv=8, L=32768) and 128K (B=1, Hq=Hkv=8, L=131072),
  tau=1: the whole forward and backward run on the GPU; the oracle computes
  seeded query blocks (O, LSE, forward and backward decisions, dQ) and the
  last key blocks of two KV heads (dK, dV; these need only the final query
  blocks' normalisers). The property checks (nesting, counts == keep maps,
  finite outputs) cover every tile.
  Decode (B=8, Hq=32, Hkv=8, Lk=131072, default split count), tau=1: seeded
  (b, query head) rows, each against the oracle on its own KV slice.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import (GRAD_REL_L2, LSE_ABS, O_REL_L2, compare_bwd_decisions, compare_fwd_decisions, legal_mask,
                    rel_l2)
from workloads import C2, C3, C4, SUBSET_SEED_OFFSET, bf16_bits_to_f64, default_workers, make_train_inputs
from test_decode_gpu import run_decode_case

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def run_full(mala, w, n_qblocks):
    tau = 1.0
    inp = make_train_inputs(w, workers=default_workers())
    q, k, v, do = (_dev(inp[x]) for x in ("q", "k", "v", "do"))
    o, lse, kept_f, km_f = mala.forward(q, k, v, w.scale, tau, w.Bq, w.Bk, keep_map=True)
    dq, dk, dv, kept_b, km_b = mala.backward(q, k, v, o, do, lse, w.scale, tau, w.Bq, w.Bk, keep_map=True)
    assert mala.mala_check_status() == 0
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    nq, nk = -(-L // w.Bq), -(-L // w.Bk)
    kmf, kmb = km_f.cpu().numpy(), km_b.cpu().numpy()
    lm = legal_mask(L, w.Bq, w.Bk)
    # properties over every tile
    assert np.isin(kmf[..., lm], (0, 1)).all() and np.isin(kmb[..., lm], (0, 1)).all()
    assert (kept_f.cpu().numpy() == (kmf == 1).reshape(B * Hq, -1).sum(1)).all()
    assert (kept_b.cpu().numpy() == (kmb == 1).reshape(B * Hq, -1).sum(1)).all()
    for t in (o, lse, dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    # sampled rows against the oracle
    rng = np.random.default_rng(w.seed + SUBSET_SEED_OFFSET)
    selq = [(0, Hq - 1, nq - 1), (0, 0, nq // 2)] + [
        (0, int(rng.integers(Hq)), int(rng.integers(nq))) for _ in range(n_qblocks - 2)]
    selq = sorted(set(selq))
    G = Hq // Hkv
    kv_heads = (0, Hkv - 1)
    selk = [(0, h, kb) for h in kv_heads for kb in (nk - 1, nk - 2)]
    # the dK / dV sample needs the normaliser of every query row at or after its key block
    need = set(selq) | {(0, hq, qb) for h in kv_heads for hq in range(h * G, (h + 1) * G)
                        for qb in range(nk - 2, nq)}
    qf, kf, vf, dof = (bf16_bits_to_f64(inp[x]) for x in ("q", "k", "v", "do"))
    ref = oracle.fwd(qf, kf, vf, w.scale, tau, w.Bq, w.Bk, sel=sorted(need))
    o_ref, lse_ref = np.nan_to_num(ref["o"]), np.nan_to_num(ref["lse"])
    refb = oracle.bwd(qf, kf, vf, o_ref, dof, lse_ref, w.scale, tau, w.Bq, w.Bk, selq=selq, selk=selk)
    fd = compare_fwd_decisions(kmf, ref["keep"], ref["margin"], L, w.Bq, w.Bk, rows=selq)
    assert fd["bad"] == 0, fd["bad_sites"][:10]
    bd = compare_bwd_decisions(kmb, refb["keep"], refb["margin"], L, w.Bq, w.Bk, fd["diverged_blocks"], rows=selq)
    assert bd["bad"] == 0, bd["bad_sites"][:10]
    viol = ((kmb == 1) & (kmf == 0) & lm).sum()
    assert viol <= 2, viol  # nesting everywhere, up to margin tiles

    def gather(arr, sel, Bt, hax):
        return np.concatenate([arr[b, x * Bt:min((x + 1) * Bt, L), h].ravel() for (b, h, x) in sel])

    og, lg = _f64(o), lse.cpu().numpy().astype(np.float64)
    e_o = rel_l2(gather(og, selq, w.Bq, 2), gather(ref["o"], selq, w.Bq, 2))
    e_lse = max(float(np.abs(lg[b, h, x * w.Bq:(x + 1) * w.Bq] - ref["lse"][b, h, x * w.Bq:(x + 1) * w.Bq]).max())
                for (b, h, x) in selq)
    e_dq = rel_l2(gather(_f64(dq), selq, w.Bq, 2), gather(refb["dq"], selq, w.Bq, 2))
    e_dk = rel_l2(gather(_f64(dk), selk, w.Bk, 2), gather(refb["dk"], selk, w.Bk, 2))
    e_dv = rel_l2(gather(_f64(dv), selk, w.Bk, 2), gather(refb["dv"], selk, w.Bk, 2))
    print(f"[full {w.name}] o={e_o:.3e} lse={e_lse:.3e} dq={e_dq:.3e} dk={e_dk:.3e} dv={e_dv:.3e} "
          f"fwd_tiles={fd['compared']} bwd_tiles={bd['compared']} in_margin={fd['in_margin']}+{bd['in_margin']}")
    assert e_o <= O_REL_L2 and e_lse <= LSE_ABS
    assert e_dq <= GRAD_REL_L2 and e_dk <= GRAD_REL_L2 and e_dv <= GRAD_REL_L2


def test_full_32k_gqa(cuda_lib):
    run_full(cuda_lib, C2, n_qblocks=6)


def test_full_128k(cuda_lib):
    run_full(cuda_lib, C3, n_qblocks=3)


def test_full_decode_128k(cuda_lib):
    rng = np.random.default_rng(C4.seed + SUBSET_SEED_OFFSET)
    rows = sorted({(0, 0), (C4.B - 1, C4.Hq - 1)} | {(int(rng.integers(C4.B)), int(rng.integers(C4.Hq)))
                                                    for _ in range(6)})
    run_decode_case(cuda_lib, C4, 1.0, n_splits=0, sample_rows=rows, workers=default_workers())
