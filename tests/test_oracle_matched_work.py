"""Pins of the matched-work diagnostics (oracle/matched_work.py).

For every row the report compares MALA's retained keys (the live keys of its
kept tiles) with the reference-mass policy given the same number of key slots
(the row's largest probabilities) -- the fidelity comparison of agihunt.info,
"MassAlloc Attention: Let Attention Allocate Its Own Compute", fidelity
paragraphs. Pinned by an independent per-row computation on tiny cases (the
50-digit brute force's keep map, math.exp probabilities, explicit sorting),
by the optimality of the reference (it never omits more than MALA at the same
budget), by tau = 0 (every live key retained, nothing omitted, dense output)
and by MALA's omitted-mass bound tau / (1 + tau).
"""
import math

import numpy as np
import pytest

import mala_bruteforce as bf
from oracle.matched_work import matched_work, summary
from test_oracle import case


def by_hand(q, k, v, scale, keep, Bq, Bk, b, h, G):
    """Per row: slots, omitted masses and output errors, from scratch."""
    L, d = q.shape[1], q.shape[3]
    out = []
    for i in range(L):
        qb = i // Bq
        s = [scale * float(np.dot(q[b, i, h], k[b, j, h // G])) for j in range(i + 1)]
        mx = max(s)
        e = [math.exp(x - mx) for x in s]
        z = sum(e)
        p = [x / z for x in e]
        dense = [sum(p[j] * v[b, j, h // G, c] for j in range(i + 1)) for c in range(d)]
        kept = [j for j in range(i + 1) if keep[b, h, qb, j // Bk] == 1]
        slots = len(kept)
        # MALA's output: softmax over the kept keys
        zk = sum(e[j] for j in kept)
        o_m = [sum(e[j] * v[b, j, h // G, c] for j in kept) / zk for c in range(d)]
        top = sorted(range(i + 1), key=lambda j: (-p[j], j))[:slots]
        zt = sum(e[j] for j in top)
        o_r = [sum(e[j] * v[b, j, h // G, c] for j in top) / zt for c in range(d)]
        nrm = math.sqrt(sum(x * x for x in dense))
        err = lambda o: math.sqrt(sum((a - c_) ** 2 for a, c_ in zip(o, dense))) / nrm
        out.append((slots, i + 1, 1 - sum(p[j] for j in kept), 1 - sum(p[j] for j in top), err(o_m), err(o_r)))
    return np.array(out)


@pytest.mark.parametrize("L,d,Hq,Hkv,Bt,tau,sharpen,seed", [(64, 8, 2, 1, 8, 1.0, 2.0, 71),
                                                             (33, 8, 2, 2, 4, 4.0, 1.5, 151)])
def test_matched_work_by_hand(L, d, Hq, Hkv, Bt, tau, sharpen, seed):
    q, k, v, _ = case(L, d, Hq, Hkv, seed=seed, sharpen=sharpen)
    sc = 1 / math.sqrt(d)
    keep = bf.bf_forward(q, k, v, sc, tau, Bt, Bt)["keep"]
    r = matched_work(q, k, v, sc, tau, Bt, Bt)
    G = Hq // Hkv
    ref = np.concatenate([by_hand(q, k, v, sc, keep, Bt, Bt, 0, h, G) for h in range(Hq)])
    for col, name in enumerate(("slots", "live", "omit_mala", "omit_ref", "err_mala", "err_ref")):
        assert np.abs(r[name] - ref[:, col]).max() < 1e-10, name
    assert (r["slots"] < r["live"]).any()  # the case skips something


@pytest.mark.parametrize("tau", [0.5, 1.0, 4.0])
def test_reference_never_omits_more_and_mala_obeys_its_bound(tau):
    q, k, v, _ = case(256, 16, 2, 1, seed=160, sharpen=2.0)
    r = matched_work(q, k, v, 0.25, tau, 16, 16)
    assert (r["omit_ref"] <= r["omit_mala"] + 1e-12).all()
    assert (r["omit_mala"] < tau / (1 + tau)).all()
    s = summary(r)
    assert 0 < s["slot_frac"] <= 1 and 0 <= s["rows_within_10pct"] <= 1


def test_tau0_retains_everything():
    q, k, v, _ = case(100, 8, 2, 2, seed=161)
    r = matched_work(q, k, v, 0.3, 0.0, 16, 16)
    assert (r["slots"] == r["live"]).all()
    assert np.abs(r["omit_mala"]).max() < 1e-12 and np.abs(r["omit_ref"]).max() < 1e-12
    assert r["err_mala"].max() < 1e-12 and r["err_ref"].max() < 1e-12


def test_given_keep_map_equals_the_oracle_decisions():
    # the analysis of a keep map passed in (as the CUDA forward's is) equals the
    # analysis of the oracle's own decisions when the maps are the same
    q, k, v, _ = case(200, 16, 2, 1, seed=162, sharpen=2.0)
    from oracle import fwd
    keep = fwd(q, k, v, 0.25, 1.0, 16, 16)["keep"]
    a = matched_work(q, k, v, 0.25, 1.0, 16, 16)
    b = matched_work(q, k, v, 0.25, 1.0, 16, 16, keep=keep)
    for name in a:
        assert np.abs(a[name] - b[name]).max() < 1e-12, name
    # a different map changes the slots and the masses accordingly
    keep2 = keep.copy()
    keep2[0, 0, 5, 2] = 1 - keep2[0, 0, 5, 2]
    c = matched_work(q, k, v, 0.25, 1.0, 16, 16, keep=keep2)
    rows = slice(5 * 16, 6 * 16)
    assert (np.abs(c["slots"][rows] - a["slots"][rows]) == 16).all()
