"""MALA on packed variable-length batches on the GPU (C ABI mala_fwd_varlen /
mala_bwd_varlen) against the fp64 oracle.

A packed batch is independent sequences end to end (agihunt.info, "MassAlloc
Attention: Let Attention Allocate Its Own Compute", method paragraphs: the
gate of a query looks only at the keys it sees). Every sequence is drawn with
the training recipe on its own seed; prefill-style sequences keep the last Lq
query rows of their Lk positions. Cases mix lengths that end inside and on
tile boundaries, single-row and empty query sets, GQA, Bq != Bk and several
tau. Rules and tolerances are in tests/parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import (GRAD_REL_L2, LSE_ABS, O_REL_L2, compare_bwd_decisions, compare_fwd_decisions,
                    illegal_untouched, rel_l2)
from workloads import TrainWorkload, bf16_bits_to_f64, make_train_inputs

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def packed_inputs(lens_q, lens_k, d, Hq, Hkv, seed):
    """bf16 bit tensors of a packed batch: q/dO [total_q,Hq,d], k/v [total_k,Hkv,d]."""
    parts = {"q": [], "k": [], "v": [], "do": []}
    for s, (lq, lk) in enumerate(zip(lens_q, lens_k)):
        if lk == 0:
            continue
        t = make_train_inputs(TrainWorkload("varlen", 1, Hq, Hkv, lk, d, 128, 128, seed=seed + s))
        parts["q"].append(t["q"][0, lk - lq:])
        parts["do"].append(t["do"][0, lk - lq:])
        parts["k"].append(t["k"][0])
        parts["v"].append(t["v"][0])
    out = {x: np.concatenate(v, 0) for x, v in parts.items()}
    out["cu_q"] = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    out["cu_k"] = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    return out


def check_fwd(inp, ref, o, lse, km, kept, lens_q, lens_k, Bq, Bk):
    km_h, kept_h = km.cpu().numpy(), kept.cpu().numpy()
    Hq = o.shape[1]
    stats = {"compared": 0, "in_margin": 0, "cascaded": 0}
    diverged = {}
    for s, (lq, lk) in enumerate(zip(lens_q, lens_k)):
        if lq == 0:
            assert (km_h[s] == 255).all()
            assert (kept_h[s * Hq:(s + 1) * Hq] == 0).all()
            continue
        nq, nk = -(-lq // Bq), -(-lk // Bk)
        assert illegal_untouched(km_h[s:s + 1, :, :nq, :nk], lq, Bq, Bk, lk)
        assert (km_h[s, :, nq:] == 255).all() and (km_h[s, :, :, nk:] == 255).all()
        dec = compare_fwd_decisions(km_h[s:s + 1, :, :nq, :nk], ref["keep"][s:s + 1, :, :nq, :nk],
                                    ref["margin"][s:s + 1, :, :nq, :nk], lq, Bq, Bk, Lk=lk)
        assert dec["bad"] == 0, (s, dec["bad_sites"][:10])
        diverged[s] = {(h, qb) for (_, h, qb) in dec["diverged_blocks"]}
        for k_ in stats:
            stats[k_] += dec[k_]
        assert (kept_h[s * Hq:(s + 1) * Hq] == (km_h[s] == 1).reshape(Hq, -1).sum(1)).all()
    assert stats["in_margin"] + stats["cascaded"] <= max(2, stats["compared"] // 1000), stats
    e_o = rel_l2(_f64(o), ref["o"])
    e_lse = float(np.abs(lse.cpu().numpy().astype(np.float64) - ref["lse"]).max())
    assert e_o <= O_REL_L2, e_o
    assert e_lse <= LSE_ABS, e_lse
    return e_o, e_lse, stats, diverged


FWD_CASES = [
    # lens_q, lens_k, d, Hq, Hkv, Bq, Bk, tau
    ([1000, 1, 300, 129, 640], None, 128, 4, 2, 128, 128, 1.0),     # training batch: ragged and tile-exact
    ([1000, 1, 300, 129, 640], None, 128, 4, 2, 128, 128, 0.0),
    ([77, 0, 512, 300], [2000, 40, 512, 1300], 128, 4, 2, 128, 128, 1.0),  # prompts after cached prefixes
    ([333, 1, 700], [1333, 1, 900], 64, 2, 1, 64, 128, 4.0),        # Bq != Bk
    ([256, 257, 255], [700, 257, 1000], 128, 2, 2, 128, 64, 0.5),
    ([1500, 64], None, 64, 6, 2, 64, 64, 1.0),
]


@pytest.mark.parametrize("lens_q,lens_k,d,Hq,Hkv,Bq,Bk,tau", FWD_CASES)
def test_fwd_varlen(cuda_lib, lens_q, lens_k, d, Hq, Hkv, Bq, Bk, tau):
    lens_k = lens_q if lens_k is None else lens_k
    inp = packed_inputs(lens_q, lens_k, d, Hq, Hkv, seed=6000 + sum(lens_q))
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    cq, ck = torch.from_numpy(inp["cu_q"]).cuda(), torch.from_numpy(inp["cu_k"]).cuda()
    scale = d ** -0.5
    o, lse, kept, km = cuda_lib.forward_varlen(q, k, v, cq, ck, max(lens_q), max(lens_k), scale, tau, Bq, Bk,
                                               keep_map=True)
    assert cuda_lib.mala_check_status() == 0
    ref = oracle.varlen_fwd(bf16_bits_to_f64(inp["q"]), bf16_bits_to_f64(inp["k"]), bf16_bits_to_f64(inp["v"]),
                            inp["cu_q"], inp["cu_k"], scale, tau, Bq, Bk)
    e_o, e_lse, st, _ = check_fwd(inp, ref, o, lse, km, kept, lens_q, lens_k, Bq, Bk)
    print(f"[fwd varlen parity] lens_q={lens_q} lens_k={lens_k} d={d} H={Hq}/{Hkv} Bq={Bq} Bk={Bk} tau={tau}: "
          f"o_rel_l2={e_o:.3e} lse_abs={e_lse:.3e} tiles={st['compared']} in_margin={st['in_margin']}")


def test_fwd_varlen_equal_lengths_is_the_batched_call(cuda_lib):
    """Equal-length sequences packed end to end give exactly the batched forward."""
    B, L, Hq, Hkv, d = 3, 700, 4, 2, 128
    t = make_train_inputs(TrainWorkload("eq", B, Hq, Hkv, L, d, 128, 128, seed=6101))
    q, k, v = (_dev(t[x]) for x in ("q", "k", "v"))
    o1, lse1, kept1, km1 = cuda_lib.forward(q, k, v, d ** -0.5, 1.0, keep_map=True)
    cu = torch.arange(B + 1, dtype=torch.int32, device="cuda") * L
    pk = lambda x: x.reshape(B * L, x.shape[2], d)
    o2, lse2, kept2, km2 = cuda_lib.forward_varlen(pk(q), pk(k), pk(v), cu, cu, L, L, d ** -0.5, 1.0, keep_map=True)
    assert cuda_lib.mala_check_status() == 0
    assert torch.equal(pk(o1), o2)
    assert torch.equal(lse1.permute(1, 0, 2).reshape(Hq, B * L), lse2)
    assert torch.equal(kept1, kept2) and torch.equal(km1, km2)


BWD_CASES = [
    # lens, d, Hq, Hkv, Bq, Bk, tau
    ([1000, 1, 300, 129, 640], 128, 4, 2, 128, 128, 1.0),
    ([1000, 1, 300, 129, 640], 128, 4, 2, 128, 128, 0.0),
    ([333, 900, 2], 64, 2, 1, 64, 128, 4.0),
    ([256, 513], 128, 2, 2, 128, 64, 0.5),
]


@pytest.mark.parametrize("lens,d,Hq,Hkv,Bq,Bk,tau", BWD_CASES)
def test_bwd_varlen(cuda_lib, lens, d, Hq, Hkv, Bq, Bk, tau):
    inp = packed_inputs(lens, lens, d, Hq, Hkv, seed=6200 + sum(lens))
    q, k, v, do = (_dev(inp[x]) for x in ("q", "k", "v", "do"))
    cu = torch.from_numpy(inp["cu_q"]).cuda()
    scale = d ** -0.5
    L = max(lens)
    o, lse, kept_f, km_f = cuda_lib.forward_varlen(q, k, v, cu, cu, L, L, scale, tau, Bq, Bk, keep_map=True)
    dq, dk, dv, kept_b, km_b = cuda_lib.backward_varlen(q, k, v, o, do, lse, cu, L, scale, tau, Bq, Bk,
                                                        keep_map=True)
    assert cuda_lib.mala_check_status() == 0
    qf, kf, vf, dof = (bf16_bits_to_f64(inp[x]) for x in ("q", "k", "v", "do"))
    ref = oracle.varlen_fwd(qf, kf, vf, inp["cu_q"], inp["cu_q"], scale, tau, Bq, Bk)
    _, _, _, diverged = check_fwd(inp, ref, o, lse, km_f, kept_f, lens, lens, Bq, Bk)
    refb = oracle.varlen_bwd(qf, kf, vf, ref["o"], dof, ref["lse"], inp["cu_q"], scale, tau, Bq, Bk)
    kmb = km_b.cpu().numpy()
    kb_h = kept_b.cpu().numpy()
    for s, ls in enumerate(lens):
        nq, nk = -(-ls // Bq), -(-ls // Bk)
        assert illegal_untouched(kmb[s:s + 1, :, :nq, :nk], ls, Bq, Bk)
        bd = compare_bwd_decisions(kmb[s:s + 1, :, :nq, :nk], refb["keep"][s:s + 1, :, :nq, :nk],
                                   refb["margin"][s:s + 1, :, :nq, :nk], ls, Bq, Bk,
                                   {(0, h, qb) for (h, qb) in diverged[s]})
        assert bd["bad"] == 0, (s, bd["bad_sites"][:10])
        assert (kb_h[s * Hq:(s + 1) * Hq] == (kmb[s] == 1).reshape(Hq, -1).sum(1)).all()
    errs = {n: rel_l2(_f64(t), refb[n]) for n, t in (("dq", dq), ("dk", dk), ("dv", dv))}
    print(f"[bwd varlen parity] lens={lens} d={d} H={Hq}/{Hkv} Bq={Bq} Bk={Bk} tau={tau}: "
          + " ".join(f"{n}={e:.3e}" for n, e in errs.items()))
    for n, e in errs.items():
        assert e <= GRAD_REL_L2, (n, e)


def test_varlen_bad_sequence_table_is_reported(cuda_lib):
    """A sequence whose table entry lies outside the tensors is left untouched and
    reported by mala_check_status (the kernel checks the entry before any access);
    the other sequences are computed as usual."""
    lens = [300, 200]
    inp = packed_inputs(lens, lens, 64, 2, 1, seed=6300)
    q, k, v = (_dev(inp[x]) for x in ("q", "k", "v"))
    good = torch.from_numpy(inp["cu_q"]).cuda()
    bad = good.clone()
    bad[2] = 100000  # the second sequence would end far past the tensors
    o, lse, kept, _ = cuda_lib.forward_varlen(q, k, v, bad, bad, 300, 300, 0.125, 1.0, 64, 64)
    assert cuda_lib.mala_check_status() == cuda_lib.MALA_ERR_INVALID_ARG
    assert cuda_lib.mala_check_status() == 0  # the status word is cleared once read
    o2, lse2, kept2, _ = cuda_lib.forward_varlen(q, k, v, good, good, 300, 300, 0.125, 1.0, 64, 64)
    assert cuda_lib.mala_check_status() == 0
    assert torch.equal(o[:300], o2[:300]) and torch.equal(lse[:, :300], lse2[:, :300])
    assert int(kept[2:].sum()) == 0
