"""Independent brute-force MALA in 50-digit arithmetic (mpmath), for tiny cases.

Written a second way on purpose, to pin the fp64 oracle: no online softmax,
no running max, no rescaling. Each row keeps an explicit SET of retained keys
and every ratio is the unstabilised exp(s_ij) / sum_{k in set} exp(s_ik).
Method source: agihunt.info, "MassAlloc Attention: Let Attention Allocate Its
Own Compute", method paragraphs (tile gate vs tau/Lq with Lq = i+1; forward
against the evolving normaliser from the diagonal toward earlier keys, first
legal tile retained, one row keeps the block; backward against the finalised
normaliser, no forced tile).
"""
from __future__ import annotations

import mpmath as mp
import numpy as np

mp.mp.dps = 50


def _scores(q, k, scale, b, hq, hkv, L, d):
    """Exact s_ij (mpf) for the live causal pairs of one (b, hq)."""
    sc = mp.mpf(scale)
    out = {}
    for i in range(L):
        qi = [mp.mpf(float(x)) for x in q[b, i, hq]]
        for j in range(i + 1):
            kj = k[b, j, hkv]
            out[(i, j)] = sc * mp.fsum(qi[c] * mp.mpf(float(kj[c])) for c in range(d))
    return out


def bf_forward(q, k, v, scale, tau, Bq, Bk):
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    nq, nk = -(-L // Bq), -(-L // Bk)
    tau_m = mp.mpf(tau)
    keep = np.zeros((B, Hq, nq, nk), dtype=np.uint8)
    o = np.zeros(q.shape)
    lse = np.zeros((B, Hq, L))
    kept_sets = {}
    E_all = {}
    for b in range(B):
        for hq in range(Hq):
            hkv = hq // G
            S = _scores(q, k, scale, b, hq, hkv, L, d)
            E = {key: mp.exp(val) for key, val in S.items()}
            E_all[(b, hq)] = E
            for qb in range(nq):
                rows = range(qb * Bq, min((qb + 1) * Bq, L))
                sets = {i: set() for i in rows}
                last = max(rows)
                kb_first = last // Bk
                for kb in range(kb_first, -1, -1):
                    keys = range(kb * Bk, min((kb + 1) * Bk, L))
                    if kb == kb_first or tau == 0:
                        kp = True
                    else:
                        kp = False
                        for i in rows:
                            live = [j for j in keys if j <= i]
                            if not live:
                                continue
                            if not sets[i]:
                                kp = True
                                continue
                            Z = mp.fsum(E[(i, j)] for j in sets[i])
                            for j in live:
                                if E[(i, j)] / Z >= tau_m / (i + 1):
                                    kp = True
                    keep[b, hq, qb, kb] = 1 if kp else 0
                    if kp:
                        for i in rows:
                            sets[i].update(j for j in keys if j <= i)
                for i in rows:
                    Z = mp.fsum(E[(i, j)] for j in sets[i])
                    lse[b, hq, i] = float(mp.log(Z))
                    for c in range(d):
                        o[b, i, hq, c] = float(mp.fsum(E[(i, j)] * mp.mpf(float(v[b, j, hkv, c]))
                                                       for j in sets[i]) / Z)
                    kept_sets[(b, hq, i)] = sets[i]
    return {"o": o, "lse": lse, "keep": keep, "sets": kept_sets, "E": E_all}


def bf_backward(q, k, v, do, scale, tau, Bq, Bk, fwd):
    """Backward against the brute-force forward's own O and normaliser."""
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    nq, nk = -(-L // Bq), -(-L // Bk)
    tau_m = mp.mpf(tau)
    sc = mp.mpf(scale)
    dq = [[[[mp.mpf(0)] * d for _ in range(Hq)] for _ in range(L)] for _ in range(B)]
    dk = [[[[mp.mpf(0)] * d for _ in range(Hkv)] for _ in range(L)] for _ in range(B)]
    dv = [[[[mp.mpf(0)] * d for _ in range(Hkv)] for _ in range(L)] for _ in range(B)]
    keep = np.zeros((B, Hq, nq, nk), dtype=np.uint8)
    for b in range(B):
        for hq in range(Hq):
            hkv = hq // G
            E = fwd["E"][(b, hq)]
            Z = {i: mp.fsum(E[(i, j)] for j in fwd["sets"][(b, hq, i)]) for i in range(L)}
            # D_i = <dO_i, O_i> with O_i = sum_{kept} E v / Z (exact, not the rounded fwd output)
            Oex = {}
            D = {}
            for i in range(L):
                Oex[i] = [mp.fsum(E[(i, j)] * mp.mpf(float(v[b, j, hkv, c])) for j in fwd["sets"][(b, hq, i)]) / Z[i]
                          for c in range(d)]
                D[i] = mp.fsum(mp.mpf(float(do[b, i, hq, c])) * Oex[i][c] for c in range(d))
            for qb in range(nq):
                rows = range(qb * Bq, min((qb + 1) * Bq, L))
                for kb in range(nk):
                    keys = range(kb * Bk, min((kb + 1) * Bk, L))
                    live = [(i, j) for i in rows for j in keys if j <= i]
                    if not live:
                        continue
                    kp = tau == 0 or any(E[(i, j)] / Z[i] >= tau_m / (i + 1) for (i, j) in live)
                    keep[b, hq, qb, kb] = 1 if kp else 0
                    if not kp:
                        continue
                    for (i, j) in live:
                        P = E[(i, j)] / Z[i]
                        dP = mp.fsum(mp.mpf(float(do[b, i, hq, c])) * mp.mpf(float(v[b, j, hkv, c])) for c in range(d))
                        dS = P * (dP - D[i])
                        for c in range(d):
                            dv[b][j][hkv][c] += P * mp.mpf(float(do[b, i, hq, c]))
                            dk[b][j][hkv][c] += sc * dS * mp.mpf(float(q[b, i, hq, c]))
                            dq[b][i][hq][c] += sc * dS * mp.mpf(float(k[b, j, hkv, c]))
    to = lambda t: np.array([[[[float(x) for x in row] for row in hh] for hh in ll] for ll in t])
    return {"dq": to(dq), "dk": to(dk), "dv": to(dv), "keep": keep}


def bf_decode(q, kc, vc, scale, tau, Bk, n_splits):
    """Decode of row Lk-1 with contiguous splits of T = ceil(nk/n_splits) tiles."""
    B, Hq, d = q.shape
    Lk, Hkv = kc.shape[1], kc.shape[2]
    G = Hq // Hkv
    nk = -(-Lk // Bk)
    T = -(-nk // n_splits)
    tau_m = mp.mpf(tau)
    sc = mp.mpf(scale)
    o = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    keep = np.zeros((B, Hq, nk), dtype=np.uint8)
    for b in range(B):
        for hq in range(Hq):
            hkv = hq // G
            qi = [mp.mpf(float(x)) for x in q[b, hq]]
            E = [mp.exp(sc * mp.fsum(qi[c] * mp.mpf(float(kc[b, j, hkv, c])) for c in range(d))) for j in range(Lk)]
            parts = []
            for s in range(n_splits):
                t0, t1 = min(s * T, nk), min((s + 1) * T, nk)
                kept = set()
                for kb in range(t1 - 1, t0 - 1, -1):
                    keys = range(kb * Bk, min((kb + 1) * Bk, Lk))
                    if kb == t1 - 1 or tau == 0:
                        kp = True
                    else:
                        Z = mp.fsum(E[j] for j in kept)
                        kp = any(E[j] / Z >= tau_m / Lk for j in keys)
                    keep[b, hq, kb] = 1 if kp else 0
                    if kp:
                        kept.update(keys)
                if kept:
                    parts.append(kept)
            allkept = set().union(*parts)
            Z = mp.fsum(E[j] for j in allkept)
            lse[b, hq] = float(mp.log(Z))
            for c in range(d):
                o[b, hq, c] = float(mp.fsum(E[j] * mp.mpf(float(vc[b, j, hkv, c])) for j in allkept) / Z)
    return {"o": o, "lse": lse, "keep": keep}


def bf_prefill(q, k, v, scale, tau, Bq, Bk):
    """Forward of Lq new queries at positions P0 + i (P0 = Lk - Lq) against Lk
    keys, with query blocks cut from the first new query and thresholds
    tau / (P0 + i + 1). Explicit kept-key sets, unstabilised ratios."""
    B, Lq, Hq, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    P0 = Lk - Lq
    G = Hq // Hkv
    nq, nk = -(-Lq // Bq), -(-Lk // Bk)
    tau_m = mp.mpf(tau)
    sc = mp.mpf(scale)
    keep = np.zeros((B, Hq, nq, nk), dtype=np.uint8)
    o = np.zeros(q.shape)
    lse = np.zeros((B, Hq, Lq))
    for b in range(B):
        for hq in range(Hq):
            hkv = hq // G
            E = {}
            for i in range(Lq):
                qi = [mp.mpf(float(x)) for x in q[b, i, hq]]
                for j in range(P0 + i + 1):
                    E[(i, j)] = mp.exp(sc * mp.fsum(qi[c] * mp.mpf(float(k[b, j, hkv, c])) for c in range(d)))
            for qb in range(nq):
                rows = range(qb * Bq, min((qb + 1) * Bq, Lq))
                sets = {i: set() for i in rows}
                kb_first = (P0 + max(rows)) // Bk
                for kb in range(kb_first, -1, -1):
                    keys = range(kb * Bk, min((kb + 1) * Bk, Lk))
                    if kb == kb_first or tau == 0:
                        kp = True
                    else:
                        kp = False
                        for i in rows:
                            live = [j for j in keys if j <= P0 + i]
                            if not live:
                                continue
                            if not sets[i]:
                                kp = True
                                continue
                            Z = mp.fsum(E[(i, j)] for j in sets[i])
                            if any(E[(i, j)] / Z >= tau_m / (P0 + i + 1) for j in live):
                                kp = True
                    keep[b, hq, qb, kb] = 1 if kp else 0
                    if kp:
                        for i in rows:
                            sets[i].update(j for j in keys if j <= P0 + i)
                for i in rows:
                    Z = mp.fsum(E[(i, j)] for j in sets[i])
                    lse[b, hq, i] = float(mp.log(Z))
                    for c in range(d):
                        o[b, i, hq, c] = float(mp.fsum(E[(i, j)] * mp.mpf(float(v[b, j, hkv, c]))
                                                       for j in sets[i]) / Z)
    return {"o": o, "lse": lse, "keep": keep}
