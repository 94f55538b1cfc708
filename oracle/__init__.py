"""MALA CPU oracle (fp64) -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA product path never calls it,
and it shares no code with ``mass_gated_causal_b200``.

The arithmetic lives in ``mala_oracle.c`` (plain C, fp64, OpenMP over
independent query blocks / key blocks); this module compiles it with gcc,
loads it with ctypes and marshals numpy arrays. Method source: agihunt.info,
"MassAlloc Attention: Let Attention Allocate Its Own Compute", method
paragraphs (tile gate against tau/Lq, evolving forward state, final-LSE
backward test, decode).

Every function takes fp64 inputs. Callers that start from bf16 bit tensors
use ``workloads.bf16_bits_to_f64`` first (exact).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mala_oracle.c")
_LIB = os.path.join(_HERE, "libmala_oracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_u8p = ctypes.POINTER(ctypes.c_uint8)


def build(force: bool = False) -> str:
    """Compile the oracle shared library with gcc (fp64, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i, d_ = ctypes.c_int, ctypes.c_double
        lib.oracle_fwd.argtypes = [_dp, _dp, _dp, i, i, i, i, i, d_, d_, i, i, _i32p, i,
                                   _dp, _dp, _u8p, _dp, _i64p]
        lib.oracle_fwd.restype = None
        lib.oracle_prefill.argtypes = [_dp, _dp, _dp, i, i, i, i, i, i, d_, d_, i, i, _i32p, i,
                                       _dp, _dp, _u8p, _dp, _i64p]
        lib.oracle_prefill.restype = None
        lib.oracle_dense_lse.argtypes = [_dp, _dp, i, i, i, i, i, d_, _dp]
        lib.oracle_dense_lse.restype = None
        lib.oracle_bwd.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, i, i, i, i, i, d_, d_, i, i,
                                   _i32p, i, _i32p, i, _dp, _dp, _dp, _u8p, _dp, _i64p]
        lib.oracle_bwd.restype = None
        lib.oracle_decode.argtypes = [_dp, _dp, _dp, i, i, i, i, i, d_, d_, i, i, _i32p, i,
                                      _dp, _dp, _u8p, _dp, _i64p, _dp, _dp]
        lib.oracle_decode.restype = None
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a, t):
    return None if a is None else a.ctypes.data_as(t)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def _sel(sel, width):
    if sel is None:
        return None, 0
    a = np.ascontiguousarray(np.asarray(sel, dtype=np.int32).reshape(-1, width))
    return a, a.shape[0]


def fwd(q, k, v, scale: float, tau: float, Bq: int, Bk: int,
        sel: Optional[Sequence] = None, with_margin: bool = True):
    """MALA forward. q [B,L,Hq,d], k/v [B,L,Hkv,d] (fp64).

    Returns dict with o [B,L,Hq,d], lse [B,Hq,L], keep [B,Hq,nq,nk] (uint8),
    margin [B,Hq,nq,nk] (fp64, NaN on illegal/forced tiles), kept [B*Hq].
    With ``sel`` (array of (b, hq, qb)), only those blocks are computed; other
    rows of o/lse are NaN and other keep-map rows are 255.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    nq, nk = -(-L // Bq), -(-L // Bk)
    o = np.full_like(q, np.nan)
    lse = np.full((B, Hq, L), np.nan)
    keep = np.full((B, Hq, nq, nk), 255 if sel is not None else 0, dtype=np.uint8)
    if sel is None:
        keep[:] = 0
    margin = np.full((B, Hq, nq, nk), np.nan) if with_margin else None
    kept = np.zeros(B * Hq, dtype=np.int64)
    s, ns = _sel(sel, 3)
    if sel is not None:
        # only legal tiles of selected rows get written; clear them to 0 first
        for (b, hq, qb) in s:
            keep[b, hq, qb] = 0
    _load().oracle_fwd(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), B, Hq, Hkv, L, d, float(scale),
                       float(tau), Bq, Bk, _ptr(s, _i32p), ns, _ptr(o, _dp), _ptr(lse, _dp),
                       _ptr(keep, _u8p), _ptr(margin, _dp), _ptr(kept, _i64p))
    return {"o": o, "lse": lse, "keep": keep, "margin": margin, "kept": kept}


def prefill(q, k, v, scale: float, tau: float, Bq: int, Bk: int,
            sel: Optional[Sequence] = None, with_margin: bool = True):
    """MALA forward of Lq new queries against Lk >= Lq keys (prefill against an
    existing cache). q [B,Lq,Hq,d] holds the queries at positions Lk-Lq ..
    Lk-1; k/v [B,Lk,Hkv,d] (fp64). Query blocks start at the first new query.

    Returns dict with o [B,Lq,Hq,d], lse [B,Hq,Lq], keep [B,Hq,nq,nk]
    (nq = ceil(Lq/Bq), nk = ceil(Lk/Bk)), margin, kept [B*Hq]; ``sel`` as in fwd.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Lq, Hq, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    assert Lk >= Lq
    nq, nk = -(-Lq // Bq), -(-Lk // Bk)
    o = np.full_like(q, np.nan)
    lse = np.full((B, Hq, Lq), np.nan)
    keep = np.full((B, Hq, nq, nk), 255 if sel is not None else 0, dtype=np.uint8)
    margin = np.full((B, Hq, nq, nk), np.nan) if with_margin else None
    kept = np.zeros(B * Hq, dtype=np.int64)
    s, ns = _sel(sel, 3)
    if sel is not None:
        for (b, hq, qb) in s:
            keep[b, hq, qb] = 0
    _load().oracle_prefill(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), B, Hq, Hkv, Lq, Lk, d, float(scale),
                           float(tau), Bq, Bk, _ptr(s, _i32p), ns, _ptr(o, _dp), _ptr(lse, _dp),
                           _ptr(keep, _u8p), _ptr(margin, _dp), _ptr(kept, _i64p))
    return {"o": o, "lse": lse, "keep": keep, "margin": margin, "kept": kept}


def dense_lse(q, k, scale: float):
    q, k = _f64(q), _f64(k)
    B, L, Hq, d = q.shape
    out = np.empty((B, Hq, L))
    _load().oracle_dense_lse(_ptr(q, _dp), _ptr(k, _dp), B, Hq, k.shape[2], L, d, float(scale),
                             _ptr(out, _dp))
    return out


def bwd(q, k, v, o, do, lse, scale: float, tau: float, Bq: int, Bk: int,
        selq: Optional[Sequence] = None, selk: Optional[Sequence] = None,
        with_margin: bool = True):
    """MALA backward. Consumes o and lse as given (fp64).

    Returns dict with dq [B,L,Hq,d], dk/dv [B,L,Hkv,d], keep [B,Hq,nq,nk],
    margin, kept [B*Hq]. With selq / selk, only those query blocks
    ((b, hq, qb)) / key blocks ((b, hkv, kb)) are computed; other rows NaN.
    """
    q, k, v, o, do, lse = map(_f64, (q, k, v, o, do, lse))
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    nq, nk = -(-L // Bq), -(-L // Bk)
    dq = np.full_like(q, np.nan)
    dk = np.full_like(k, np.nan)
    dv = np.full_like(v, np.nan)
    keep = np.zeros((B, Hq, nq, nk), dtype=np.uint8)
    margin = np.full((B, Hq, nq, nk), np.nan) if with_margin else None
    kept = np.zeros(B * Hq, dtype=np.int64)
    sq, nsq = _sel(selq, 3)
    sk, nsk = _sel(selk, 3)
    _load().oracle_bwd(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), _ptr(o, _dp), _ptr(do, _dp),
                       _ptr(lse, _dp), B, Hq, Hkv, L, d, float(scale), float(tau), Bq, Bk,
                       _ptr(sq, _i32p), nsq, _ptr(sk, _i32p), nsk, _ptr(dq, _dp), _ptr(dk, _dp),
                       _ptr(dv, _dp), _ptr(keep, _u8p), _ptr(margin, _dp), _ptr(kept, _i64p))
    return {"dq": dq, "dk": dk, "dv": dv, "keep": keep, "margin": margin, "kept": kept}


def decode_split_range(nk: int, n_splits: int, s: int):
    """Tile range [t0, t1) of split s: T = ceil(nk / n_splits)."""
    T = -(-nk // n_splits)
    return min(s * T, nk), min((s + 1) * T, nk)


def decode(q, kc, vc, scale: float, tau: float, Bk: int, n_splits: int,
           sel: Optional[Sequence] = None, with_parts: bool = False):
    """MALA decode. q [B,Hq,d]; kc/vc [B,Lk,Hkv,d] (fp64).

    Returns dict with o [B,Hq,d], lse [B,Hq], keep [B,Hq,nk], margin,
    kept [B*Hq] and, with ``with_parts``, o_part [B,Hq,S,d] / lse_part [B,Hq,S].
    """
    q, kc, vc = _f64(q), _f64(kc), _f64(vc)
    B, Hq, d = q.shape
    Lk, Hkv = kc.shape[1], kc.shape[2]
    nk = -(-Lk // Bk)
    o = np.full((B, Hq, d), np.nan)
    lse = np.full((B, Hq), np.nan)
    keep = np.zeros((B, Hq, nk), dtype=np.uint8)
    margin = np.full((B, Hq, nk), np.nan)
    kept = np.zeros(B * Hq, dtype=np.int64)
    op = np.zeros((B, Hq, n_splits, d)) if with_parts else None
    lp = np.zeros((B, Hq, n_splits)) if with_parts else None
    s, ns = _sel(sel, 2)
    _load().oracle_decode(_ptr(q, _dp), _ptr(kc, _dp), _ptr(vc, _dp), B, Hq, Hkv, Lk, d,
                          float(scale), float(tau), Bk, n_splits, _ptr(s, _i32p), ns,
                          _ptr(o, _dp), _ptr(lse, _dp), _ptr(keep, _u8p), _ptr(margin, _dp),
                          _ptr(kept, _i64p), _ptr(op, _dp), _ptr(lp, _dp))
    out = {"o": o, "lse": lse, "keep": keep, "margin": margin, "kept": kept}
    if with_parts:
        out["o_part"], out["lse_part"] = op, lp
    return out


# ------------------------------------------------------------------ packed batches
# A packed (variable-length) batch is a set of independent sequences laid end to
# end; MALA's gate never looks across a sequence. These functions are that
# definition written out: each sequence's slice goes through the single-sequence
# routines above, whose arithmetic is pinned on its own.

def _cu(cu):
    cu = np.asarray(cu, dtype=np.int64)
    assert cu.ndim == 1 and cu[0] == 0 and (np.diff(cu) >= 0).all()
    return cu


def varlen_fwd(q, k, v, cu_q, cu_k, scale: float, tau: float, Bq: int, Bk: int, with_margin: bool = True):
    """MALA forward of a packed batch. q [total_q,Hq,d]; k/v [total_k,Hkv,d];
    sequence s owns query rows cu_q[s]:cu_q[s+1] and keys cu_k[s]:cu_k[s+1]
    (Lk_s >= Lq_s: its queries are the last Lq_s of its Lk_s positions, as in
    ``prefill``; Lq_s == Lk_s is the training forward).

    Returns dict with o [total_q,Hq,d], lse [Hq,total_q], keep / margin
    [S,Hq,max_nq,max_nk] (per sequence its [nq_s, nk_s] corner; legal entries
    0/1, the rest 255 / NaN) and kept [S*Hq].
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    cu_q, cu_k = _cu(cu_q), _cu(cu_k)
    S = len(cu_q) - 1
    assert len(cu_k) == S + 1
    Hq, d = q.shape[1], q.shape[2]
    lq, lk = np.diff(cu_q), np.diff(cu_k)
    assert (lk >= lq).all()
    mq = max(1, -(-int(lq.max(initial=0)) // Bq))
    mk = max(1, -(-int(lk.max(initial=0)) // Bk))
    o = np.full_like(q, np.nan)
    lse = np.full((Hq, q.shape[0]), np.nan)
    keep = np.full((S, Hq, mq, mk), 255, dtype=np.uint8)
    margin = np.full((S, Hq, mq, mk), np.nan) if with_margin else None
    kept = np.zeros(S * Hq, dtype=np.int64)
    for s in range(S):
        if lq[s] == 0:
            continue
        r = prefill(q[None, cu_q[s]:cu_q[s + 1]], k[None, cu_k[s]:cu_k[s + 1]], v[None, cu_k[s]:cu_k[s + 1]],
                    scale, tau, Bq, Bk, with_margin=with_margin)
        o[cu_q[s]:cu_q[s + 1]] = r["o"][0]
        lse[:, cu_q[s]:cu_q[s + 1]] = r["lse"][0]
        nq_s, nk_s = r["keep"].shape[2], r["keep"].shape[3]
        legal = _legal(int(lq[s]), int(lk[s]), Bq, Bk)
        blk = keep[s, :, :nq_s, :nk_s]
        blk[:, legal] = r["keep"][0][:, legal]
        if with_margin:
            margin[s, :, :nq_s, :nk_s] = r["margin"][0]
        kept[s * Hq:(s + 1) * Hq] = r["kept"]
    return {"o": o, "lse": lse, "keep": keep, "margin": margin, "kept": kept}


def _legal(Lq: int, Lk: int, Bq: int, Bk: int):
    """[nq, nk] legal-tile mask of Lq queries at positions Lk-Lq.. against Lk keys."""
    P0 = Lk - Lq
    nq, nk = -(-Lq // Bq), -(-Lk // Bk)
    m = np.zeros((nq, nk), dtype=bool)
    for qb in range(nq):
        m[qb, : (P0 + min((qb + 1) * Bq, Lq) - 1) // Bk + 1] = True
    return m


def varlen_bwd(q, k, v, o, do, lse, cu, scale: float, tau: float, Bq: int, Bk: int, with_margin: bool = True):
    """MALA backward of a packed training batch (queries and keys share ``cu``).
    q/o/do [total,Hq,d], k/v [total,Hkv,d], lse [Hq,total] (as ``varlen_fwd``
    returns it). Returns dq, dk, dv (packed like the inputs), keep / margin
    [S,Hq,max_nq,max_nk] (illegal entries 255 / NaN) and kept [S*Hq]."""
    q, k, v, o, do, lse = (_f64(a) for a in (q, k, v, o, do, lse))
    cu = _cu(cu)
    S = len(cu) - 1
    Hq = q.shape[1]
    ln = np.diff(cu)
    mq = max(1, -(-int(ln.max(initial=0)) // Bq))
    mk = max(1, -(-int(ln.max(initial=0)) // Bk))
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    keep = np.full((S, Hq, mq, mk), 255, dtype=np.uint8)
    margin = np.full((S, Hq, mq, mk), np.nan) if with_margin else None
    kept = np.zeros(S * Hq, dtype=np.int64)
    for s in range(S):
        a, b = cu[s], cu[s + 1]
        if b == a:
            continue
        r = bwd(q[None, a:b], k[None, a:b], v[None, a:b], o[None, a:b], do[None, a:b], lse[None, :, a:b],
                scale, tau, Bq, Bk, with_margin=with_margin)
        dq[a:b], dk[a:b], dv[a:b] = r["dq"][0], r["dk"][0], r["dv"][0]
        legal = _legal(int(b - a), int(b - a), Bq, Bk)
        nq_s, nk_s = legal.shape
        blk = keep[s, :, :nq_s, :nk_s]
        blk[:, legal] = r["keep"][0][:, legal]
        if with_margin:
            margin[s, :, :nq_s, :nk_s] = r["margin"][0]
        kept[s * Hq:(s + 1) * Hq] = r["kept"]
    return {"dq": dq, "dk": dk, "dv": dv, "keep": keep, "margin": margin, "kept": kept}


def paged_decode(q, k_pages, v_pages, block_table, seqlens, scale: float, tau: float, n_splits: int,
                 sel: Optional[Sequence] = None):
    """MALA decode against a paged KV cache. q [B,Hq,d]; k_pages/v_pages
    [num_pages,page,Hkv,d]; block_table [B,max_pages] (page ids); seqlens [B].
    Sequence b's keys are rows 0..page-1 of pages block_table[b,0], [b,1], ...,
    cut at seqlens[b]; its key tiles are its pages (Bk = page). Each sequence is
    ``decode`` of its gathered cache with the same n_splits.

    Returns dict with o [B,Hq,d], lse [B,Hq], keep / margin [B,Hq,max_pages]
    (entries past a sequence's tiles 255 / NaN), kept [B*Hq]. ``sel`` lists
    (b, hq) rows to compute; other rows are NaN (keep 255)."""
    q, kp, vp = _f64(q), _f64(k_pages), _f64(v_pages)
    bt = np.asarray(block_table, dtype=np.int64)
    sl = np.asarray(seqlens, dtype=np.int64)
    B, Hq, d = q.shape
    page = kp.shape[1]
    maxp = bt.shape[1]
    o = np.full((B, Hq, d), np.nan)
    lse = np.full((B, Hq), np.nan)
    keep = np.full((B, Hq, maxp), 255, dtype=np.uint8)
    margin = np.full((B, Hq, maxp), np.nan)
    kept = np.zeros(B * Hq, dtype=np.int64)
    rows = None if sel is None else {}
    if sel is not None:
        for (b, hq) in sel:
            rows.setdefault(int(b), []).append(int(hq))
    for b in range(B):
        if rows is not None and b not in rows:
            continue
        Lk = int(sl[b])
        npg = -(-Lk // page)
        kc = kp[bt[b, :npg]].reshape(npg * page, kp.shape[2], d)[:Lk]
        vc = vp[bt[b, :npg]].reshape(npg * page, vp.shape[2], d)[:Lk]
        s = None if rows is None else [(0, hq) for hq in sorted(set(rows[b]))]
        r = decode(q[b:b + 1], kc[None], vc[None], scale, tau, page, n_splits, sel=s)
        hs = range(Hq) if rows is None else sorted(set(rows[b]))
        for hq in hs:
            o[b, hq] = r["o"][0, hq]
            lse[b, hq] = r["lse"][0, hq]
            keep[b, hq, :npg] = r["keep"][0, hq]
            margin[b, hq, :npg] = r["margin"][0, hq]
            kept[b * Hq + hq] = r["kept"][hq]
    return {"o": o, "lse": lse, "keep": keep, "margin": margin, "kept": kept}


def decode_single_pass(q, kc, vc, scale: float, tau: float, Bk: int, sel: Optional[Sequence] = None):
    """Decode as ONE sequential pass over all key tiles (newest to oldest, the
    first kept): ``decode`` with a single split, which equals the forward's last
    query row (pinned in tests/test_oracle.py). A split-independent decode must
    reach exactly these decisions whatever split of the tiles it uses."""
    return decode(q, kc, vc, scale, tau, Bk, 1, sel=sel)
