"""Pins of the oracle's prefill against an existing cache (and of Bq != Bk).

Prefill: Lq new queries at positions P0 .. P0 + Lq - 1 (P0 = Lk - Lq) of a
sequence of Lk keys; query row i sees keys 0 .. P0 + i and its threshold uses
Lq_i = P0 + i + 1 (agihunt.info, "MassAlloc Attention: Let Attention Allocate
Its Own Compute", method paragraphs: the same tile gate, with Lq the number
of causally visible keys of the query). Query blocks are cut from the first
new query.

Pins: an independent 50-digit brute force with explicit kept-key sets
(tests/mala_bruteforce.py) on tiny cases, including offsets that are not a
multiple of Bq and Bq != Bk; tau = 0 equals the dense causal softmax rows of
the whole sequence (torch fp64); an offset that is a multiple of Bq gives the
same blocks, hence the same decisions and outputs, as the training forward of
the whole sequence; the omitted-mass bound; counts == kept tiles.
"""
import math

import numpy as np
import pytest

import oracle
import mala_bruteforce as bf
from test_oracle import case, dense_ref

PREFILL_CASES = [
    # Lk, Lq, d, Hq, Hkv, Bq, Bk, tau, sharpen, seed
    (44, 21, 8, 2, 1, 8, 8, 1.0, 1.5, 61),
    (40, 40, 8, 2, 2, 8, 4, 0.5, 2.0, 62),
    (37, 13, 8, 2, 1, 4, 8, 4.0, 1.0, 63),
    (48, 16, 4, 1, 1, 8, 16, 1.0, 3.0, 64),
    (33, 9, 8, 2, 2, 16, 8, 1.0, 2.0, 65),
    (30, 30, 8, 2, 1, 4, 8, 0.0, 1.0, 66),
]


@pytest.mark.parametrize("Lk,Lq,d,Hq,Hkv,Bq,Bk,tau,sharpen,seed", PREFILL_CASES)
def test_prefill_matches_bruteforce(Lk, Lq, d, Hq, Hkv, Bq, Bk, tau, sharpen, seed):
    q, k, v, _ = case(Lk, d, Hq, Hkv, seed=seed, sharpen=sharpen)
    qn = q[:, Lk - Lq:]
    sc = 1 / math.sqrt(d)
    r = oracle.prefill(qn, k, v, sc, tau, Bq, Bk)
    ref = bf.bf_prefill(qn, k, v, sc, tau, Bq, Bk)
    assert (r["keep"] == ref["keep"]).all()
    assert np.abs(r["o"] - ref["o"]).max() < 1e-10
    assert np.abs(r["lse"] - ref["lse"]).max() < 1e-10
    assert (r["kept"] == (r["keep"] == 1).reshape(r["kept"].shape[0], -1).sum(1)).all()


@pytest.mark.parametrize("P0,Lq,Bq,Bk", [(100, 60, 16, 16), (37, 91, 8, 16), (64, 64, 16, 8)])
def test_prefill_tau0_is_dense_rows(P0, Lq, Bq, Bk):
    Lk = P0 + Lq
    q, k, v, _ = case(Lk, 16, 4, 2, seed=70 + P0)
    sc = 1 / math.sqrt(16)
    r = oracle.prefill(q[:, P0:], k, v, sc, 0.0, Bq, Bk)
    o_d, lse_d = dense_ref(q, k, v, sc)
    assert np.abs(r["o"] - o_d[:, P0:]).max() < 1e-12
    assert np.abs(r["lse"] - lse_d[:, :, P0:]).max() < 1e-12


@pytest.mark.parametrize("tau", [0.5, 1.0, 4.0])
def test_prefill_aligned_offset_equals_training_forward(tau):
    L, Bq, Bk, P0 = 160, 16, 16, 96
    q, k, v, _ = case(L, 16, 4, 2, seed=81, sharpen=2.0)
    sc = 1 / math.sqrt(16)
    full = oracle.fwd(q, k, v, sc, tau, Bq, Bk)
    r = oracle.prefill(q[:, P0:], k, v, sc, tau, Bq, Bk)
    assert (r["keep"] == full["keep"][:, :, P0 // Bq:]).all()
    assert np.abs(r["o"] - full["o"][:, P0:]).max() < 1e-12
    assert np.abs(r["lse"] - full["lse"][:, :, P0:]).max() < 1e-12


@pytest.mark.parametrize("tau", [0.5, 1.0, 4.0])
def test_prefill_omitted_mass_bound(tau):
    P0, Lq = 70, 90
    Lk = P0 + Lq
    q, k, v, _ = case(Lk, 16, 2, 1, seed=91, sharpen=2.0)
    sc = 1 / math.sqrt(16)
    r = oracle.prefill(q[:, P0:], k, v, sc, tau, 16, 8)
    _, lse_d = dense_ref(q, k, v, sc)
    omega = 1.0 - np.exp(r["lse"] - lse_d[:, :, P0:])
    assert (omega >= -1e-12).all()
    assert (omega < tau / (1 + tau)).all()


BQBK_CASES = [
    # L, d, Hq, Hkv, Bq, Bk, tau, sharpen, seed
    (40, 8, 2, 1, 8, 4, 1.0, 2.0, 101),
    (37, 8, 2, 2, 4, 8, 4.0, 1.5, 102),
    (48, 8, 1, 1, 16, 8, 0.5, 2.0, 103),
]


@pytest.mark.parametrize("L,d,Hq,Hkv,Bq,Bk,tau,sharpen,seed", BQBK_CASES)
def test_bq_ne_bk_matches_bruteforce(L, d, Hq, Hkv, Bq, Bk, tau, sharpen, seed):
    q, k, v, do = case(L, d, Hq, Hkv, seed=seed, sharpen=sharpen)
    sc = 1 / math.sqrt(d)
    f = oracle.fwd(q, k, v, sc, tau, Bq, Bk)
    ref = bf.bf_forward(q, k, v, sc, tau, Bq, Bk)
    assert (f["keep"] == ref["keep"]).all()
    assert np.abs(f["o"] - ref["o"]).max() < 1e-10
    g = oracle.bwd(q, k, v, f["o"], do, f["lse"], sc, tau, Bq, Bk)
    rb = bf.bf_backward(q, k, v, do, sc, tau, Bq, Bk, ref)
    assert (g["keep"] == rb["keep"]).all()
    for name in ("dq", "dk", "dv"):
        assert np.abs(g[name] - rb[name]).max() < 1e-9
