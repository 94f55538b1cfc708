"""Comparison rules between the CUDA path and the fp64 oracle.

Tolerances (from the operator's stated parity bar):
  * tile keep/skip decisions identical, except tiles whose gate margin
    |g - 1| < 1e-3, g = max over rows of ratio / (tau/Lq);
  * O within relative L2 error 2e-3, LSE within absolute error 1e-3;
  * dQ / dK / dV within relative L2 error 1e-2.

Forward decisions of one query block form a chain (each depends on the state
left by the earlier ones), so after a legitimate in-margin disagreement the
two sides continue from different states. Decisions later in that chain are
then reported as "cascaded" and not held to equality; every other decision
must match exactly. Backward decisions are independent of each other given
the LSE, so a disagreement there is allowed only in margin, or in a query
block whose forward chain already diverged (its LSE differs).
"""
from __future__ import annotations

import numpy as np

MARGIN = 1e-3
O_REL_L2 = 2e-3
LSE_ABS = 1e-3
GRAD_REL_L2 = 1e-2


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def legal_mask(L, Bq, Bk, Lk=None):
    """Legal tiles of L query rows at positions Lk - L .. Lk - 1 against Lk
    keys (Lk = L: the training case). Query blocks start at the first row."""
    Lk = L if Lk is None else Lk
    P0 = Lk - L
    nq, nk = -(-L // Bq), -(-Lk // Bk)
    m = np.zeros((nq, nk), dtype=bool)
    for qb in range(nq):
        m[qb, : (P0 + min((qb + 1) * Bq, L) - 1) // Bk + 1] = True
    return m


def compare_fwd_decisions(gpu_keep, ora_keep, ora_margin, L, Bq, Bk, rows=None, Lk=None):
    """Walk every selected (b, hq, qb) chain in visit order (kb descending).

    Returns dict(bad, in_margin, cascaded, diverged_blocks, compared).
    ``rows`` restricts to a list of (b, hq, qb); default all. ``Lk`` > L: a
    prefill of L new queries against Lk keys.
    """
    lm = legal_mask(L, Bq, Bk, Lk)
    B, H, nq, nk = ora_keep.shape
    if rows is None:
        rows = [(b, h, qb) for b in range(B) for h in range(H) for qb in range(nq)]
    out = {"bad": 0, "in_margin": 0, "cascaded": 0, "compared": 0, "diverged_blocks": set(), "bad_sites": []}
    for (b, h, qb) in rows:
        diverged = False
        for kb in range(nk - 1, -1, -1):
            if not lm[qb, kb]:
                continue
            out["compared"] += 1
            a, o = int(gpu_keep[b, h, qb, kb]), int(ora_keep[b, h, qb, kb])
            if a == o:
                continue
            g = ora_margin[b, h, qb, kb]
            if diverged:
                out["cascaded"] += 1
            elif np.isfinite(g) and abs(g - 1.0) < MARGIN:
                out["in_margin"] += 1
                diverged = True
                out["diverged_blocks"].add((b, h, qb))
            else:
                out["bad"] += 1
                out["bad_sites"].append((b, h, qb, kb, a, o, float(g)))
    return out


def compare_bwd_decisions(gpu_keep, ora_keep, ora_margin, L, Bq, Bk, diverged_blocks=(), rows=None):
    lm = legal_mask(L, Bq, Bk)
    B, H, nq, nk = ora_keep.shape
    if rows is None:
        rows = [(b, h, qb) for b in range(B) for h in range(H) for qb in range(nq)]
    out = {"bad": 0, "in_margin": 0, "excused": 0, "compared": 0, "bad_sites": []}
    dv = set(diverged_blocks)
    for (b, h, qb) in rows:
        for kb in range(nk):
            if not lm[qb, kb]:
                continue
            out["compared"] += 1
            a, o = int(gpu_keep[b, h, qb, kb]), int(ora_keep[b, h, qb, kb])
            if a == o:
                continue
            g = ora_margin[b, h, qb, kb]
            if (b, h, qb) in dv:
                out["excused"] += 1
            elif np.isfinite(g) and abs(g - 1.0) < MARGIN:
                out["in_margin"] += 1
            else:
                out["bad"] += 1
                out["bad_sites"].append((b, h, qb, kb, a, o, float(g)))
    return out


def illegal_untouched(keep_map, L, Bq, Bk, Lk=None) -> bool:
    """Entries of illegal tiles keep the caller's fill value 255."""
    lm = legal_mask(L, Bq, Bk, Lk)
    km = np.asarray(keep_map)
    return bool((km[..., ~lm] == 255).all()) and bool(np.isin(km[..., lm], (0, 1)).all())
