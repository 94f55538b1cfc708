"""Matched-work fidelity diagnostics (fp64, CPU) -- TEST / ANALYSIS INFRASTRUCTURE.

The fidelity study of the pages (agihunt.info, "MassAlloc Attention: Let
Attention Allocate Its Own Compute", fidelity paragraphs) compares MALA with a
reference that is given the same work: the same number of key slots per query.
This module does that on synthetic inputs. For every query row i:

- dense probabilities p_ij = softmax over the live keys j <= i (fp64);
- MALA's retained keys: the live keys of the tiles its forward kept for the
  row's block (``oracle.fwd``'s keep map); k_i = their count (the row's key
  slots) and MALA's output O_i is the oracle forward's;
- the reference-mass policy with the same budget: the k_i keys of largest p_ij
  (the most mass any k_i keys can hold), its output the softmax restricted to
  them;
- omitted mass 1 - sum of the retained p_ij, and the relative L2 error of each
  output against the dense output.

``matched_work`` returns per-row arrays and ``summary`` aggregates them;
``tests/report_matched_work.py`` prints the report on the 1K and 8K workloads.
Only tests import this module.
"""
from __future__ import annotations

import numpy as np

from . import fwd as _mala_fwd


def _rows_of_block(L, Bq, qb):
    return np.arange(qb * Bq, min((qb + 1) * Bq, L))


def matched_work(q, k, v, scale: float, tau: float, Bq: int, Bk: int, heads=None, keep=None):
    """q [B,L,Hq,d], k/v [B,L,Hkv,d] fp64. Returns a dict of per-row arrays over
    the selected (b, hq) (default all): slots, live, omit_mala, omit_ref,
    err_mala, err_ref (relative L2 error of the row's output).

    With ``keep`` (a keep map [B,Hq,nq,nk] from elsewhere, e.g. the CUDA
    forward's) the retained keys come from that map and MALA's output is the
    softmax over them -- what the forward computes with those decisions, up to
    rounding; without it, the oracle forward decides and supplies its output."""
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    if keep is None:
        f = _mala_fwd(q, k, v, scale, tau, Bq, Bk)
        keep, o_mala = f["keep"], f["o"]
    else:
        o_mala = None
    nq = -(-L // Bq)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(Hq)]
    out = {x: [] for x in ("slots", "live", "omit_mala", "omit_ref", "err_mala", "err_ref")}
    for (b, h) in heads:
        kk, vv = k[b, :, h // G], v[b, :, h // G]
        for qb in range(nq):
            rows = _rows_of_block(L, Bq, qb)
            s = scale * (q[b, rows, h] @ kk.T)                         # [R, L]
            live = np.arange(L)[None, :] <= rows[:, None]
            s = np.where(live, s, -np.inf)
            s -= s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)                          # dense probabilities
            o_dense = p @ vv
            kept_keys = np.zeros(L, dtype=bool)
            for kb in np.nonzero(keep[b, h, qb] == 1)[0]:
                kept_keys[kb * Bk:(kb + 1) * Bk] = True
            ret = live & kept_keys[None, :]                            # MALA's retained live keys
            slots = ret.sum(axis=1)
            assert (slots >= 1).all()  # the block's first tile holds every row's own key
            omit_mala = 1.0 - (p * ret).sum(axis=1)
            # reference-mass policy: the `slots` largest probabilities of each row
            ps = -np.sort(-p, axis=1)
            cums = np.cumsum(ps, axis=1)
            omit_ref = 1.0 - cums[np.arange(len(rows)), slots - 1]
            # its output: softmax restricted to those keys (ties broken by key index)
            order = np.argsort(-p, axis=1, kind="stable")
            rank = np.empty_like(order)
            np.put_along_axis(rank, order, np.arange(L)[None, :].repeat(len(rows), 0), axis=1)
            pr = np.where(rank < slots[:, None], p, 0.0)
            o_ref = (pr @ vv) / pr.sum(axis=1, keepdims=True)
            nrm = np.linalg.norm(o_dense, axis=1)
            out["slots"].append(slots)
            out["live"].append(live.sum(axis=1))
            out["omit_mala"].append(omit_mala)
            out["omit_ref"].append(omit_ref)
            if o_mala is None:  # the softmax over MALA's retained keys
                pm = p * ret
                om = (pm @ vv) / pm.sum(axis=1, keepdims=True)
            else:
                om = o_mala[b, rows, h]
            out["err_mala"].append(np.linalg.norm(om - o_dense, axis=1) / nrm)
            out["err_ref"].append(np.linalg.norm(o_ref - o_dense, axis=1) / nrm)
    return {x: np.concatenate(v_) for x, v_ in out.items()}


def summary(r) -> dict:
    """Means over rows, and the fraction of rows where MALA's omitted mass is
    within 10% (relative) of the reference's at the same budget."""
    return {
        "rows": int(r["slots"].size),
        "slot_frac": float(r["slots"].sum() / r["live"].sum()),
        "omit_mala_mean": float(r["omit_mala"].mean()),
        "omit_ref_mean": float(r["omit_ref"].mean()),
        "omit_mala_max": float(r["omit_mala"].max()),
        "err_mala_mean": float(r["err_mala"].mean()),
        "err_ref_mean": float(r["err_ref"].mean()),
        "rows_within_10pct": float(np.mean(r["omit_mala"] <= 1.1 * r["omit_ref"] + 1e-15)),
    }
