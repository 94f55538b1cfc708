"""Pins for the fp64 CPU oracle: it is checked against things other than itself.

Method source: agihunt.info, "MassAlloc Attention: Let Attention Allocate Its
Own Compute", method paragraphs and the limitations paragraph (omitted-mass
bound tau/(1+tau), nested backward support, tau -> 0 recovers full
attention).

Pins used here:
  * tau = 0 forward  == dense causal softmax attention (torch fp64 SDPA) and
    LSE == logsumexp over all causal keys;
  * tau = 0 backward == torch fp64 autograd of dense attention, and central
    finite differences of the oracle's own tau = 0 forward;
  * tau > 0: an independent 50-digit brute force with explicit retained-key
    sets and unstabilised ratios gives identical keep maps and equal
    O / LSE / dQ / dK / dV / decode outputs;
  * tau > 0 backward == torch fp64 autograd of attention restricted to the
    forward's retained keys, whenever the backward keeps the same tiles;
  * invariants: nesting (backward keep set within forward keep set), no
    empty row, omitted mass < tau/(1+tau), counts == popcount, tau = 0 counts
    == number of legal tiles;
  * structure: GQA == the same computation with K/V repeated per query head;
    selected-block mode == full mode; decode with one split == forward row
    L-1 with Bq = 1; decode at tau = 0 == dense row for any split count.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from workloads import TrainWorkload, bf16_bits_to_f64, make_train_inputs, C0
import mala_bruteforce as bf


def case(L, d, Hq, Hkv, seed, sharpen=1.0, B=1, kind="structured"):
    w = TrainWorkload("tiny", B, Hq, Hkv, L, d, 16, 16, seed=seed, kind=kind)
    t = make_train_inputs(w)
    q, k, v, do = (bf16_bits_to_f64(t[x]) for x in ("q", "k", "v", "do"))
    return q * sharpen, k, v, do


def dense_ref(q, k, v, scale):
    """torch fp64 causal SDPA with K/V repeated over the GQA group."""
    G = q.shape[2] // k.shape[2]
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(np.repeat(k, G, axis=2)).permute(0, 2, 1, 3)
    vt = torch.from_numpy(np.repeat(v, G, axis=2)).permute(0, 2, 1, 3)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    s = (qt @ kt.transpose(-1, -2)) * scale
    L = q.shape[1]
    s = s.masked_fill(torch.triu(torch.ones(L, L, dtype=torch.bool), 1), float("-inf"))
    return o.permute(0, 2, 1, 3).numpy(), torch.logsumexp(s, -1).numpy()


def legal_count(L, Bq, Bk):
    """Tile (qb, kb) is legal iff kb*Bk <= last row of block qb."""
    nq = -(-L // Bq)
    return sum((min((qb + 1) * Bq, L) - 1) // Bk + 1 for qb in range(nq))


# ---------------------------------------------------------------- tau = 0 pins
@pytest.mark.parametrize("L,d,Hq,Hkv,Bt", [(1024, 64, 2, 2, 64), (200, 32, 4, 2, 16), (77, 16, 2, 1, 8)])
def test_fwd_tau0_is_dense_attention(L, d, Hq, Hkv, Bt):
    q, k, v, _ = case(L, d, Hq, Hkv, seed=11)
    scale = 1 / math.sqrt(d)
    r = oracle.fwd(q, k, v, scale, 0.0, Bt, Bt)
    o_ref, lse_ref = dense_ref(q, k, v, scale)
    assert np.abs(r["o"] - o_ref).max() < 1e-12
    assert np.abs(r["lse"] - lse_ref).max() < 1e-12
    assert r["keep"].sum() == legal_count(L, Bt, Bt) * Hq
    assert (r["kept"] == legal_count(L, Bt, Bt)).all()


@pytest.mark.parametrize("L,d,Hq,Hkv,Bt", [(96, 16, 2, 2, 16), (53, 8, 4, 2, 8)])
def test_bwd_tau0_is_autograd_of_dense(L, d, Hq, Hkv, Bt):
    q, k, v, do = case(L, d, Hq, Hkv, seed=12)
    scale = 1 / math.sqrt(d)
    f = oracle.fwd(q, k, v, scale, 0.0, Bt, Bt)
    g = oracle.bwd(q, k, v, f["o"], do, f["lse"], scale, 0.0, Bt, Bt)
    G = Hq // Hkv
    qt = torch.from_numpy(q).requires_grad_()
    kt = torch.from_numpy(k).requires_grad_()
    vt = torch.from_numpy(v).requires_grad_()
    o = torch.nn.functional.scaled_dot_product_attention(
        qt.permute(0, 2, 1, 3), kt.repeat_interleave(G, 2).permute(0, 2, 1, 3),
        vt.repeat_interleave(G, 2).permute(0, 2, 1, 3), is_causal=True, scale=scale).permute(0, 2, 1, 3)
    (o * torch.from_numpy(do)).sum().backward()
    for name, ref in (("dq", qt.grad), ("dk", kt.grad), ("dv", vt.grad)):
        assert np.abs(g[name] - ref.numpy()).max() < 1e-11, name


def test_bwd_tau0_finite_differences():
    L, d, Hq, Hkv, Bt = 13, 4, 2, 1, 4
    q, k, v, do = case(L, d, Hq, Hkv, seed=13)
    scale = 0.5
    f = oracle.fwd(q, k, v, scale, 0.0, Bt, Bt)
    g = oracle.bwd(q, k, v, f["o"], do, f["lse"], scale, 0.0, Bt, Bt)
    loss = lambda qq, kk, vv: float((oracle.fwd(qq, kk, vv, scale, 0.0, Bt, Bt)["o"] * do).sum())
    h = 1e-6
    rng = np.random.default_rng(0)
    for name, arr, grad in (("q", q, g["dq"]), ("k", k, g["dk"]), ("v", v, g["dv"])):
        for _ in range(12):
            idx = tuple(rng.integers(0, s) for s in arr.shape)
            ap, am = arr.copy(), arr.copy()
            ap[idx] += h
            am[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = ap, am
            fd = (loss(args_p["q"], args_p["k"], args_p["v"]) - loss(args_m["q"], args_m["k"], args_m["v"])) / (2 * h)
            assert abs(fd - grad[idx]) < 1e-7 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


# ---------------------------------------------------------- brute-force pins
BF_CASES = [
    # L, d, Hq, Hkv, Bt, tau, sharpen, seed
    (32, 8, 2, 1, 4, 1.0, 1.0, 21),
    (37, 8, 2, 2, 8, 0.5, 2.0, 22),
    (64, 8, 1, 1, 16, 1.0, 2.0, 23),
    (48, 8, 2, 1, 8, 4.0, 1.5, 24),
    (29, 4, 2, 2, 4, 1.0, 3.0, 25),
    (40, 8, 2, 1, 8, 0.0, 1.0, 26),
    (64, 8, 2, 1, 8, 4.0, 1.0, 71),
]


@pytest.mark.parametrize("L,d,Hq,Hkv,Bt,tau,sharpen,seed", BF_CASES)
def test_bruteforce_forward_backward(L, d, Hq, Hkv, Bt, tau, sharpen, seed):
    q, k, v, do = case(L, d, Hq, Hkv, seed=seed, sharpen=sharpen)
    scale = 1 / math.sqrt(d)
    f = oracle.fwd(q, k, v, scale, tau, Bt, Bt)
    ref = bf.bf_forward(q, k, v, scale, tau, Bt, Bt)
    assert (f["keep"] == ref["keep"]).all()
    assert np.abs(f["o"] - ref["o"]).max() < 1e-10
    assert np.abs(f["lse"] - ref["lse"]).max() < 1e-10
    g = oracle.bwd(q, k, v, f["o"], do, f["lse"], scale, tau, Bt, Bt)
    rb = bf.bf_backward(q, k, v, do, scale, tau, Bt, Bt, ref)
    assert (g["keep"] == rb["keep"]).all()
    for name in ("dq", "dk", "dv"):
        assert np.abs(g[name] - rb[name]).max() < 1e-9, name


def test_bruteforce_cases_exercise_both_decisions():
    """The brute-force sweep above must see kept AND skipped non-forced tiles."""
    skipped_fwd = skipped_bwd_only = 0
    for (L, d, Hq, Hkv, Bt, tau, sharpen, seed) in BF_CASES:
        if tau == 0:
            continue
        q, k, v, do = case(L, d, Hq, Hkv, seed=seed, sharpen=sharpen)
        f = oracle.fwd(q, k, v, 1 / math.sqrt(d), tau, Bt, Bt)
        g = oracle.bwd(q, k, v, f["o"], do, f["lse"], 1 / math.sqrt(d), tau, Bt, Bt)
        nq = -(-L // Bt)
        legal = np.zeros_like(f["keep"], dtype=bool)
        for qb in range(nq):
            legal[:, :, qb, : (min((qb + 1) * Bt, L) - 1) // Bt + 1] = True
        skipped_fwd += int((legal & (f["keep"] == 0)).sum())
        skipped_bwd_only += int(((f["keep"] == 1) & (g["keep"] == 0)).sum())
    assert skipped_fwd > 10
    assert skipped_bwd_only > 0


@pytest.mark.parametrize("Lk,d,Hq,Hkv,Bk,tau,n_splits", [(50, 8, 2, 1, 8, 1.0, 1), (50, 8, 2, 1, 8, 1.0, 3),
                                                          (64, 4, 4, 2, 4, 0.5, 5), (33, 8, 2, 2, 4, 4.0, 2)])
def test_bruteforce_decode(Lk, d, Hq, Hkv, Bk, tau, n_splits):
    q, k, v, _ = case(Lk, d, Hq, Hkv, seed=31, sharpen=2.0)
    qd = q[:, -1]  # the last row's query: every key visible
    r = oracle.decode(qd, k, v, 1 / math.sqrt(d), tau, Bk, n_splits)
    ref = bf.bf_decode(qd, k, v, 1 / math.sqrt(d), tau, Bk, n_splits)
    assert (r["keep"] == ref["keep"]).all()
    assert np.abs(r["o"] - ref["o"]).max() < 1e-10
    assert np.abs(r["lse"] - ref["lse"]).max() < 1e-10


# ------------------------------------------------------- invariants (C0 size)
@pytest.fixture(scope="module")
def c0():
    t = make_train_inputs(C0)
    q, k, v, do = (bf16_bits_to_f64(t[x]) for x in ("q", "k", "v", "do"))
    return q, k, v, do


@pytest.mark.parametrize("tau", [0.25, 1.0, 4.0])
def test_invariants_c0(c0, tau):
    q, k, v, do = c0
    sc = C0.scale
    f = oracle.fwd(q, k, v, sc, tau, C0.Bq, C0.Bk)
    g = oracle.bwd(q, k, v, f["o"], do, f["lse"], sc, tau, C0.Bq, C0.Bk)
    # nesting: every tile the backward keeps, the forward kept
    assert not ((g["keep"] == 1) & (f["keep"] == 0)).any()
    # counts
    assert (f["kept"] == f["keep"].reshape(f["kept"].shape[0], -1).sum(1)).all()
    assert (g["kept"] == g["keep"].reshape(g["kept"].shape[0], -1).sum(1)).all()
    # no empty row: the forced diagonal tile holds a live key for every row;
    # omitted mass below tau/(1+tau)
    lse_dense = oracle.dense_lse(q, k, sc)
    omega = 1.0 - np.exp(f["lse"] - lse_dense)
    assert np.isfinite(f["lse"]).all()
    assert (omega < tau / (1 + tau)).all()
    assert (omega > -1e-12).all()
    # backward-omitted mass per row: sum over bwd-skipped live keys of exp(s - LSE) < tau
    B, L, Hq, d = q.shape
    G = Hq // k.shape[2]
    for hq in range(Hq):
        s = (q[0, :, hq] @ k[0, :, hq // G].T) * sc
        P = np.exp(s - f["lse"][0, hq][:, None])
        P[np.triu_indices(L, 1)] = 0.0
        tile_keep = np.kron(g["keep"][0, hq], np.ones((C0.Bq, C0.Bk)))[:L, :L]
        omitted = (P * (1 - tile_keep)).sum(1)
        assert (omitted < tau).all()
        # no empty backward row for tau <= 1
        if tau <= 1.0:
            assert ((P * tile_keep) > 0).any(1).all()


def test_gqa_equals_repeated_heads():
    q, k, v, do = case(90, 16, 4, 2, seed=41, sharpen=2.0)
    sc, tau, Bt = 0.25, 1.0, 16
    f = oracle.fwd(q, k, v, sc, tau, Bt, Bt)
    kr, vr = np.repeat(k, 2, axis=2), np.repeat(v, 2, axis=2)
    fr = oracle.fwd(q, kr, vr, sc, tau, Bt, Bt)
    assert (f["keep"] == fr["keep"]).all()
    assert np.abs(f["o"] - fr["o"]).max() == 0
    g = oracle.bwd(q, k, v, f["o"], do, f["lse"], sc, tau, Bt, Bt)
    gr = oracle.bwd(q, kr, vr, f["o"], do, f["lse"], sc, tau, Bt, Bt)
    assert np.abs(g["dq"] - gr["dq"]).max() == 0
    assert np.abs(g["dk"] - gr["dk"].reshape(1, 90, 2, 2, 16).sum(3)).max() < 1e-12
    assert np.abs(g["dv"] - gr["dv"].reshape(1, 90, 2, 2, 16).sum(3)).max() < 1e-12


def test_selection_mode_matches_full():
    q, k, v, do = case(150, 16, 4, 2, seed=42, sharpen=2.0)
    sc, tau, Bt = 0.25, 1.0, 16
    f = oracle.fwd(q, k, v, sc, tau, Bt, Bt)
    sel = [(0, 1, 3), (0, 3, 9), (0, 0, 0)]
    fs = oracle.fwd(q, k, v, sc, tau, Bt, Bt, sel=sel)
    for (b, hq, qb) in sel:
        rows = slice(qb * Bt, min((qb + 1) * Bt, 150))
        assert np.array_equal(fs["o"][b, rows, hq], f["o"][b, rows, hq])
        assert np.array_equal(fs["keep"][b, hq, qb], f["keep"][b, hq, qb])
    g = oracle.bwd(q, k, v, f["o"], do, f["lse"], sc, tau, Bt, Bt)
    selk = [(0, 1, 0), (0, 0, 9), (0, 1, 5)]
    gs = oracle.bwd(q, k, v, f["o"], do, f["lse"], sc, tau, Bt, Bt, selq=sel, selk=selk)
    for (b, hq, qb) in sel:
        rows = slice(qb * Bt, min((qb + 1) * Bt, 150))
        assert np.array_equal(gs["dq"][b, rows, hq], g["dq"][b, rows, hq])
    for (b, h, kb) in selk:
        rows = slice(kb * Bt, min((kb + 1) * Bt, 150))
        assert np.allclose(gs["dk"][b, rows, h], g["dk"][b, rows, h], rtol=0, atol=1e-13)
        assert np.allclose(gs["dv"][b, rows, h], g["dv"][b, rows, h], rtol=0, atol=1e-13)


def test_bwd_is_autograd_of_retained_attention_when_sets_agree():
    """If the backward keeps exactly the forward's tiles, its result is the exact
    gradient of softmax attention restricted to the forward's retained keys."""
    hits = 0
    for seed in range(60, 70):
        q, k, v, do = case(64, 8, 2, 2, seed=seed, sharpen=2.5)
        sc, tau, Bt = 1 / math.sqrt(8), 1.0, 8
        f = oracle.fwd(q, k, v, sc, tau, Bt, Bt)
        g = oracle.bwd(q, k, v, f["o"], do, f["lse"], sc, tau, Bt, Bt)
        if not np.array_equal(f["keep"], g["keep"]) or f["keep"].sum() == g["keep"].size:
            continue
        L = 64
        qt = torch.from_numpy(q).requires_grad_()
        kt = torch.from_numpy(k).requires_grad_()
        vt = torch.from_numpy(v).requires_grad_()
        s = torch.einsum("blhd,bjhd->bhlj", qt, kt) * sc
        mask = torch.from_numpy(np.kron(f["keep"][0], np.ones((1, Bt, Bt)))[:, :L, :L] > 0)[None]
        mask &= ~torch.triu(torch.ones(L, L, dtype=torch.bool), 1)
        p = torch.softmax(s.masked_fill(~mask, float("-inf")), -1)
        o = torch.einsum("bhlj,bjhd->blhd", p, vt)
        assert np.abs(o.detach().numpy() - f["o"]).max() < 1e-12
        (o * torch.from_numpy(do)).sum().backward()
        for name, ref in (("dq", qt.grad), ("dk", kt.grad), ("dv", vt.grad)):
            assert np.abs(g[name] - ref.numpy()).max() < 1e-11, name
        hits += 1
    assert hits >= 2


# ------------------------------------------------------------------ decode pins
@pytest.mark.parametrize("Lk,Bk", [(200, 16), (129, 8)])
def test_decode_one_split_is_forward_last_row(Lk, Bk):
    q, k, v, _ = case(Lk, 16, 4, 2, seed=51, sharpen=2.0)
    sc, tau = 0.25, 1.0
    r = oracle.decode(q[:, -1], k, v, sc, tau, Bk, 1)
    f = oracle.fwd(q, k, v, sc, tau, 1, Bk, sel=[(0, h, Lk - 1) for h in range(4)])
    assert np.abs(r["o"] - f["o"][:, -1]).max() < 1e-13
    assert np.abs(r["lse"] - f["lse"][:, :, -1]).max() < 1e-13
    assert np.array_equal(r["keep"], f["keep"][:, :, Lk - 1, :])


@pytest.mark.parametrize("n_splits", [1, 2, 3, 7, 40])
def test_decode_tau0_is_dense_row(n_splits):
    Lk, Bk = 300, 16
    q, k, v, _ = case(Lk, 16, 4, 2, seed=52)
    sc = 0.25
    r = oracle.decode(q[:, -1], k, v, sc, 0.0, Bk, n_splits, with_parts=True)
    o_ref, lse_ref = dense_ref(q, k, v, sc)
    assert np.abs(r["o"] - o_ref[:, -1]).max() < 1e-12
    assert np.abs(r["lse"] - lse_ref[:, :, -1]).max() < 1e-12
    assert (r["kept"] == -(-Lk // Bk)).all()
