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
