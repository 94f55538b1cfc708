"""MALA prefill on the GPU (C ABI mala_prefill) against the fp64 oracle.

Lq new queries at positions P0 .. P0 + Lq - 1 (P0 = Lk - Lq) attend to a
cache of Lk keys that already holds them at its end; query row i uses the
threshold tau / (P0 + i + 1) (agihunt.info, "MassAlloc Attention: Let
Attention Allocate Its Own Compute", method paragraphs). Inputs are the
training recipe's sequence of Lk positions, whose last Lq query rows are the
new queries. Cases cover offsets that are and are not multiples of the tile
sizes, Bq != Bk, GQA, a single new query, tau = 0, and Lq == Lk (which must
give exactly what mala_fwd gives). Rules and tolerances are in tests/parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import LSE_ABS, O_REL_L2, compare_fwd_decisions, illegal_untouched, rel_l2
from workloads import TrainWorkload, bf16_bits_to_f64, default_workers, make_train_inputs

pytestmark = pytest.mark.gpu

SAMPLE_SEED_OFFSET = 77


def _to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def run_prefill_case(mala, w, Lq, tau, n_sample=None, workers=1):
    """w.L is Lk. n_sample: compare that many sampled query blocks only."""
    Lk = w.L
    inp = make_train_inputs(w, L=Lk, workers=workers)
    qn_bits = inp["q"][:, Lk - Lq:]
    q, k, v = _to_dev(qn_bits), _to_dev(inp["k"]), _to_dev(inp["v"])
    o, lse, kept, km = mala.prefill(q, k, v, w.scale, tau, w.Bq, w.Bk, keep_map=True)
    assert mala.mala_check_status() == 0
    torch.cuda.synchronize()
    assert o.shape == q.shape and lse.shape == (w.B, w.Hq, Lq)
    nq = -(-Lq // w.Bq)
    sel = None
    if n_sample is not None:
        rng = np.random.default_rng(w.seed + SAMPLE_SEED_OFFSET)
        sel = sorted({(w.B - 1, w.Hq - 1, nq - 1), (0, 0, 0)} | {
            (int(rng.integers(w.B)), int(rng.integers(w.Hq)), int(rng.integers(nq))) for _ in range(n_sample - 2)})
    ref = oracle.prefill(bf16_bits_to_f64(qn_bits), bf16_bits_to_f64(inp["k"]), bf16_bits_to_f64(inp["v"]),
                         w.scale, tau, w.Bq, w.Bk, sel=sel)
    km_h = km.cpu().numpy()
    assert illegal_untouched(km_h, Lq, w.Bq, w.Bk, Lk)
    dec = compare_fwd_decisions(km_h, ref["keep"], ref["margin"], Lq, w.Bq, w.Bk, rows=sel, Lk=Lk)
    assert dec["bad"] == 0, dec["bad_sites"][:10]
    assert dec["in_margin"] + dec["cascaded"] <= max(2, dec["compared"] // 1000), dec
    kept_h = kept.cpu().numpy()
    assert (kept_h == (km_h == 1).reshape(kept_h.shape[0], -1).sum(1)).all()
    o_h, lse_h = _f64(o), lse.cpu().numpy().astype(np.float64)
    if sel is None:
        e_o = rel_l2(o_h, ref["o"])
        e_lse = float(np.abs(lse_h - ref["lse"]).max())
    else:
        rows = [(b, slice(x * w.Bq, min((x + 1) * w.Bq, Lq)), h) for (b, h, x) in sel]
        e_o = rel_l2(np.concatenate([o_h[b, r, h].ravel() for (b, r, h) in rows]),
                     np.concatenate([ref["o"][b, r, h].ravel() for (b, r, h) in rows]))
        e_lse = max(float(np.abs(lse_h[b, h, r] - ref["lse"][b, h, r]).max()) for (b, r, h) in rows)
    assert e_o <= O_REL_L2, e_o
    assert e_lse <= LSE_ABS, e_lse
    if tau == 0 and sel is None:
        assert (km_h == 1).sum() == (ref["keep"] == 1).sum()
    print(f"[prefill parity] Lk={Lk} Lq={Lq} d={w.d} H={w.Hq}/{w.Hkv} Bq={w.Bq} Bk={w.Bk} tau={tau}: "
          f"o_rel_l2={e_o:.3e} lse_abs={e_lse:.3e} tiles={dec['compared']} in_margin={dec['in_margin']} "
          f"cascaded={dec['cascaded']} kept={int(kept_h.sum())}")
    return o, lse, km


@pytest.mark.parametrize("Lk,Lq,d,Hq,Hkv,Bq,Bk,tau", [
    (2000, 300, 128, 4, 2, 128, 128, 1.0),   # offset 1700: not a tile multiple; ragged last block
    (2048, 512, 128, 4, 2, 128, 128, 1.0),   # offset a tile multiple
    (1500, 1, 128, 2, 1, 128, 128, 1.0),     # a single new query
    (1537, 129, 64, 2, 1, 64, 64, 1.0),      # one row past a tile boundary
    (3000, 777, 64, 2, 2, 64, 128, 0.5),     # Bq != Bk
    (2500, 257, 128, 4, 4, 128, 64, 0.0),    # full attention, Bq != Bk
    (4096, 333, 128, 8, 2, 64, 64, 4.0),
    (640, 600, 128, 2, 1, 128, 128, 1.0),    # short cache: most rows in the first pair
])
def test_prefill_shapes(cuda_lib, Lk, Lq, d, Hq, Hkv, Bq, Bk, tau):
    w = TrainWorkload("prefill", 1, Hq, Hkv, Lk, d, Bq, Bk, seed=5000 + Lk + Lq)
    run_prefill_case(cuda_lib, w, Lq, tau)


def test_prefill_batch2(cuda_lib):
    w = TrainWorkload("prefill_b2", 2, 4, 2, 1800, 128, 128, 128, seed=5101)
    run_prefill_case(cuda_lib, w, 700, 1.0)


@pytest.mark.parametrize("Bq,Bk", [(128, 128), (64, 128)])
def test_prefill_whole_sequence_is_forward(cuda_lib, Bq, Bk):
    """Lq == Lk is the training forward: identical bits, decisions and counts."""
    w = TrainWorkload("prefill_eq", 1, 4, 2, 1000, 128, Bq, Bk, seed=5202)
    inp = make_train_inputs(w)
    q, k, v = (_to_dev(inp[x]) for x in ("q", "k", "v"))
    o1, lse1, kept1, km1 = cuda_lib.forward(q, k, v, w.scale, 1.0, Bq, Bk, keep_map=True)
    o2, lse2, kept2, km2 = cuda_lib.prefill(q, k, v, w.scale, 1.0, Bq, Bk, keep_map=True)
    assert cuda_lib.mala_check_status() == 0
    assert torch.equal(o1, o2) and torch.equal(lse1, lse2)
    assert torch.equal(kept1, kept2) and torch.equal(km1, km2)


def test_prefill_long_cache_sampled(cuda_lib):
    """A 4K-query chunk after 28K cached keys, GQA 32/8, sampled query blocks."""
    w = TrainWorkload("prefill_32k", 1, 32, 8, 32768, 128, 128, 128, seed=5303)
    run_prefill_case(cuda_lib, w, 4096, 1.0, n_sample=6, workers=default_workers())
