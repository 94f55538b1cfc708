"""Pins of the oracle's packed (variable-length) batches and paged decode.

A packed batch is independent sequences laid end to end (agihunt.info,
"MassAlloc Attention: Let Attention Allocate Its Own Compute", method
paragraphs: the gate is per query over the keys it sees; limitations
paragraph: the KV cache is kept whole and decode reads it). The oracle
composes its single-sequence routines; these tests pin the composition
against things other than those routines' own packing:

- an independent 50-digit brute force (tests/mala_bruteforce.py) run on each
  sequence's rows, for forward, prefill-style sequences (Lk > Lq), backward
  and paged decode;
- tau = 0 equals dense causal softmax attention of each sequence (torch fp64),
  and its gradient equals torch autograd of that attention;
- equal-length packed sequences equal the batched (B > 1) oracle call, whose
  loop over the batch is separate C code;
- paged decode with shuffled pages (and a pool holding unrelated pages) equals
  decode of the contiguous cache; entries of the block table past a
  sequence's pages are never read.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import mala_bruteforce as bf
from test_oracle import case


def packed_case(lens_q, lens_k, d, Hq, Hkv, seed, sharpen=1.0):
    """Sequences drawn with the training recipe; sequence s keeps the last
    lens_q[s] query rows of its lens_k[s] positions."""
    qs, ks, vs, dos = [], [], [], []
    for s, (lq, lk) in enumerate(zip(lens_q, lens_k)):
        if lk == 0:
            continue
        q, k, v, do = case(lk, d, Hq, Hkv, seed=seed + s, sharpen=sharpen)
        qs.append(q[0, lk - lq:])
        dos.append(do[0, lk - lq:])
        ks.append(k[0])
        vs.append(v[0])
    cu_q = np.concatenate([[0], np.cumsum(lens_q)])
    cu_k = np.concatenate([[0], np.cumsum(lens_k)])
    cat = lambda xs, h: np.concatenate(xs, 0) if xs else np.zeros((0, h, d))
    return cat(qs, Hq), cat(ks, Hkv), cat(vs, Hkv), cat(dos, Hq), cu_q, cu_k


VARLEN_CASES = [
    # lens_q, lens_k, d, Hq, Hkv, Bq, Bk, tau, sharpen, seed
    ([17, 1, 30, 8], [17, 1, 30, 8], 8, 2, 1, 8, 8, 1.0, 2.0, 81),      # training batch, ragged
    ([5, 12, 0, 9], [21, 12, 6, 30], 8, 2, 2, 4, 8, 1.0, 1.5, 82),      # cached prefixes, an empty query set
    ([16, 7], [40, 7], 4, 2, 1, 8, 4, 4.0, 2.0, 83),                    # Bq != Bk
    ([9, 24], [9, 40], 8, 2, 1, 8, 8, 0.5, 3.0, 84),
]


@pytest.mark.parametrize("lens_q,lens_k,d,Hq,Hkv,Bq,Bk,tau,sharpen,seed", VARLEN_CASES)
def test_varlen_fwd_matches_bruteforce_per_sequence(lens_q, lens_k, d, Hq, Hkv, Bq, Bk, tau, sharpen, seed):
    q, k, v, _, cu_q, cu_k = packed_case(lens_q, lens_k, d, Hq, Hkv, seed, sharpen)
    sc = 1 / math.sqrt(d)
    r = oracle.varlen_fwd(q, k, v, cu_q, cu_k, sc, tau, Bq, Bk)
    for s in range(len(lens_q)):
        if lens_q[s] == 0:
            assert (r["keep"][s] == 255).all()
            continue
        a, b = cu_q[s], cu_q[s + 1]
        ref = bf.bf_prefill(q[None, a:b], k[None, cu_k[s]:cu_k[s + 1]], v[None, cu_k[s]:cu_k[s + 1]], sc, tau, Bq,
                            Bk)
        nq, nk = ref["keep"].shape[2:]
        lm = oracle._legal(lens_q[s], lens_k[s], Bq, Bk)
        assert (r["keep"][s, :, :nq, :nk][:, lm] == ref["keep"][0][:, lm]).all()
        assert (r["keep"][s, :, :nq, :nk][:, ~lm] == 255).all()
        assert np.abs(r["o"][a:b] - ref["o"][0]).max() < 1e-10
        assert np.abs(r["lse"][:, a:b] - ref["lse"][0]).max() < 1e-10
        assert (r["kept"][s * Hq:(s + 1) * Hq] == (ref["keep"][0] == 1).reshape(Hq, -1).sum(1)).all()


def test_varlen_fwd_tau0_is_dense_per_sequence():
    lens_q, lens_k = [20, 3, 33], [45, 3, 33]
    q, k, v, _, cu_q, cu_k = packed_case(lens_q, lens_k, 16, 4, 2, 90)
    sc = 0.25
    r = oracle.varlen_fwd(q, k, v, cu_q, cu_k, sc, 0.0, 8, 16)
    G = 2
    for s in range(3):
        a, b = cu_q[s], cu_q[s + 1]
        ka, kb = cu_k[s], cu_k[s + 1]
        qt = torch.from_numpy(q[a:b]).permute(1, 0, 2)                      # [Hq, Lq, d]
        kt = torch.from_numpy(np.repeat(k[ka:kb], G, axis=1)).permute(1, 0, 2)
        vt = torch.from_numpy(np.repeat(v[ka:kb], G, axis=1)).permute(1, 0, 2)
        sco = (qt @ kt.transpose(-1, -2)) * sc
        P0 = lens_k[s] - lens_q[s]
        mask = torch.arange(lens_k[s])[None, :] > (P0 + torch.arange(lens_q[s]))[:, None]
        sco = sco.masked_fill(mask, float("-inf"))
        o = torch.softmax(sco, -1) @ vt
        assert np.abs(r["o"][a:b] - o.permute(1, 0, 2).numpy()).max() < 1e-12
        assert np.abs(r["lse"][:, a:b] - torch.logsumexp(sco, -1).numpy()).max() < 1e-12


def test_varlen_equal_lengths_is_the_batched_call():
    L, B = 40, 3
    q, k, v, do = case(L, 8, 4, 2, seed=91, B=B, sharpen=2.0)
    sc = 1 / math.sqrt(8)
    cu = np.arange(B + 1) * L
    pk = lambda x: x.reshape(B * L, x.shape[2], x.shape[3])
    rv = oracle.varlen_fwd(pk(q), pk(k), pk(v), cu, cu, sc, 1.0, 8, 8)
    rb = oracle.fwd(q, k, v, sc, 1.0, 8, 8)
    assert np.array_equal(rv["o"], pk(rb["o"]))
    assert np.array_equal(rv["lse"], rb["lse"].transpose(1, 0, 2).reshape(4, B * L))
    lm = oracle._legal(L, L, 8, 8)
    assert (rv["keep"][:, :, lm] == rb["keep"][:, :, lm]).all()
    gv = oracle.varlen_bwd(pk(q), pk(k), pk(v), rv["o"], pk(do), rv["lse"], cu, sc, 1.0, 8, 8)
    gb = oracle.bwd(q, k, v, rb["o"], do, rb["lse"], sc, 1.0, 8, 8)
    for name in ("dq", "dk", "dv"):
        assert np.array_equal(gv[name], pk(gb[name])), name
    assert (gv["keep"][:, :, lm] == gb["keep"][:, :, lm]).all()


@pytest.mark.parametrize("lens,Bt,tau,seed", [([19, 1, 26], 8, 1.0, 95), ([12, 30], 4, 4.0, 96)])
def test_varlen_bwd_matches_bruteforce_per_sequence(lens, Bt, tau, seed):
    d, Hq, Hkv = 8, 2, 1
    q, k, v, do, cu, _ = packed_case(lens, lens, d, Hq, Hkv, seed, sharpen=2.0)
    sc = 1 / math.sqrt(d)
    f = oracle.varlen_fwd(q, k, v, cu, cu, sc, tau, Bt, Bt)
    g = oracle.varlen_bwd(q, k, v, f["o"], do, f["lse"], cu, sc, tau, Bt, Bt)
    for s in range(len(lens)):
        a, b = cu[s], cu[s + 1]
        rf = bf.bf_forward(q[None, a:b], k[None, a:b], v[None, a:b], sc, tau, Bt, Bt)
        rb = bf.bf_backward(q[None, a:b], k[None, a:b], v[None, a:b], do[None, a:b], sc, tau, Bt, Bt, rf)
        lm = oracle._legal(lens[s], lens[s], Bt, Bt)
        nq, nk = lm.shape
        assert (g["keep"][s, :, :nq, :nk][:, lm] == rb["keep"][0][:, lm]).all()
        for name in ("dq", "dk", "dv"):
            assert np.abs(g[name][a:b] - rb[name][0]).max() < 1e-9, name


def test_varlen_bwd_tau0_is_autograd_per_sequence():
    lens = [13, 29, 2]
    q, k, v, do, cu, _ = packed_case(lens, lens, 8, 4, 2, 97)
    sc = 0.3
    f = oracle.varlen_fwd(q, k, v, cu, cu, sc, 0.0, 8, 8)
    g = oracle.varlen_bwd(q, k, v, f["o"], do, f["lse"], cu, sc, 0.0, 8, 8)
    for s in range(3):
        a, b = cu[s], cu[s + 1]
        qt = torch.from_numpy(q[None, a:b]).requires_grad_()
        kt = torch.from_numpy(k[None, a:b]).requires_grad_()
        vt = torch.from_numpy(v[None, a:b]).requires_grad_()
        o = torch.nn.functional.scaled_dot_product_attention(
            qt.permute(0, 2, 1, 3), kt.repeat_interleave(2, 2).permute(0, 2, 1, 3),
            vt.repeat_interleave(2, 2).permute(0, 2, 1, 3), is_causal=True, scale=sc).permute(0, 2, 1, 3)
        (o * torch.from_numpy(do[None, a:b])).sum().backward()
        for name, ref in (("dq", qt.grad), ("dk", kt.grad), ("dv", vt.grad)):
            assert np.abs(g[name][a:b] - ref.numpy()[0]).max() < 1e-11, (s, name)


def _paged(kc, vc, lens, page, rng, extra_pages=3):
    """Scatter per-sequence caches (lists of [Lk, Hkv, d]) into a shuffled page
    pool with unrelated pages; table entries past a sequence's pages hold ids
    of unrelated pages."""
    npg = [-(-L // page) for L in lens]
    total = sum(npg) + extra_pages
    Hkv, d = kc[0].shape[1], kc[0].shape[2]
    kp = rng.standard_normal((total, page, Hkv, d))
    vp = rng.standard_normal((total, page, Hkv, d))
    ids = rng.permutation(total)
    maxp = max(npg) + 1
    table = np.full((len(lens), maxp), ids[-1], dtype=np.int32)  # an unrelated page
    n = 0
    for b, L in enumerate(lens):
        for j in range(npg[b]):
            pid = ids[n]
            n += 1
            table[b, j] = pid
            rows = kc[b][j * page:(j + 1) * page]
            kp[pid, :len(rows)] = rows
            vp[pid, :len(rows)] = vc[b][j * page:(j + 1) * page]
    return kp, vp, table


@pytest.mark.parametrize("lens,page,n_splits,tau", [([50, 9, 33], 8, 3, 1.0), ([64, 17], 4, 5, 0.5),
                                                   ([31, 31], 8, 1, 4.0)])
def test_paged_decode_matches_bruteforce(lens, page, n_splits, tau):
    d, Hq, Hkv = 8, 4, 2
    rng = np.random.default_rng(7 + page)
    qs, kc, vc = [], [], []
    for b, L in enumerate(lens):
        q, k, v, _ = case(L, d, Hq, Hkv, seed=120 + b, sharpen=2.0)
        qs.append(q[0, -1])
        kc.append(k[0])
        vc.append(v[0])
    kp, vp, table = _paged(kc, vc, lens, page, rng)
    qd = np.stack(qs)
    sc = 1 / math.sqrt(d)
    r = oracle.paged_decode(qd, kp, vp, table, lens, sc, tau, n_splits)
    for b, L in enumerate(lens):
        ref = bf.bf_decode(qd[b:b + 1], kc[b][None], vc[b][None], sc, tau, page, n_splits)
        nk = -(-L // page)
        assert (r["keep"][b, :, :nk] == ref["keep"][0]).all()
        assert (r["keep"][b, :, nk:] == 255).all()
        assert np.abs(r["o"][b] - ref["o"][0]).max() < 1e-10
        assert np.abs(r["lse"][b] - ref["lse"][0]).max() < 1e-10


def test_paged_decode_identity_table_is_contiguous_decode():
    L, B, page = 48, 2, 8
    q, k, v, _ = case(L, 8, 4, 2, seed=130, B=B, sharpen=2.0)
    qd = q[:, -1]
    npg = L // page
    kp = k.reshape(B * npg, page, 2, 8)
    vp = v.reshape(B * npg, page, 2, 8)
    table = np.arange(B * npg, dtype=np.int32).reshape(B, npg)
    r = oracle.paged_decode(qd, kp, vp, table, [L] * B, 0.35, 1.0, 2)
    rc = oracle.decode(qd, k, v, 0.35, 1.0, page, 2)
    assert np.array_equal(r["o"], rc["o"]) and np.array_equal(r["lse"], rc["lse"])
    assert np.array_equal(r["keep"], rc["keep"])


def test_paged_decode_tau0_is_dense_row():
    lens, page = [37, 5, 60], 8
    rng = np.random.default_rng(3)
    qs, kc, vc = [], [], []
    for b, L in enumerate(lens):
        q, k, v, _ = case(L, 8, 2, 1, seed=140 + b)
        qs.append(q[0, -1])
        kc.append(k[0])
        vc.append(v[0])
    kp, vp, table = _paged(kc, vc, lens, page, rng)
    r = oracle.paged_decode(np.stack(qs), kp, vp, table, lens, 0.4, 0.0, 4)
    for b in range(3):
        s = 0.4 * np.einsum("hd,jhd->hj", np.repeat(qs[b][None], 1, 0).reshape(2, 8), np.repeat(kc[b], 2, axis=1))
        lse = np.log(np.exp(s - s.max(1, keepdims=True)).sum(1)) + s.max(1)
        o = np.einsum("hj,jhd->hd", np.exp(s - lse[:, None]), np.repeat(vc[b], 2, axis=1))
        assert np.abs(r["lse"][b] - lse).max() < 1e-12
        assert np.abs(r["o"][b] - o).max() < 1e-12
