"""Seeded synthetic inputs for MALA (MassAlloc Attention) workloads.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark. It holds input generation only: no attention arithmetic, no gate, no
softmax. Every tensor is drawn in fp64 and rounded once to bf16
(round-to-nearest-even), and both sides receive the same rounded bits.

The structured generator follows the workload description of the MALA operator
study (agihunt.info "MassAlloc Attention: Let Attention Allocate Its Own
Compute", method paragraphs): attention mass concentrates on local windows,
sink tokens and a sparse retrieval set. Concretely, per (batch b, KV head h):

  * a latent z_t follows AR(1) in every one of the d dimensions,
    z_0 ~ N(0,1), z_t = rho*z_{t-1} + sqrt(1-rho^2)*eps_t, rho = 0.98
    (unit stationary variance);
  * k_t = z_t + 0.5*N(0,1), and for every query head of the group
    q_t = z_t + 0.5*N(0,1) (the latent is shared per KV head so that GQA
    query heads see the same locality);
  * u is a unit vector uniform on the sphere; keys 0..3 get +3u (sinks) and
    every query gets +1.5u;
  * retrieval: per query head, floor(0.01*L) distinct query rows i drawn
    uniformly from {1..L-1}; each gets q_i += 4*k_j for j uniform in
    {0..i-1}, using the final k_j (sink shift included);
  * V ~ N(0,1), dO ~ N(0,1).

Random streams are per slice so that any (b, h) slice can be regenerated on
its own (the oracle's sampled checks at long lengths need single slices):

  kv stream (seed, 0, b, h):  z_0 [d], eps [L-1, d], k noise [L, d],
                              u draw [d], V [L, d]       -- in that order
  q stream  (seed, 1, b, hq): q noise [L, d], retrieval rows, retrieval
                              sources, dO [L, d]         -- in that order

The iid variant draws Q, K, V, dO ~ N(0,1) from the same per-slice streams.

Decode queries (one new token per sequence, all Lk keys visible): for each
(b, hq) q = z_{Lk-1} + 0.5*N(0,1) + 1.5u from stream (seed, 2, b, hq); then
ceil(0.01*B*Hq) distinct (b, hq) pairs, drawn from stream (seed, 3), get
q += 4*k_j with j uniform in {0..Lk-2}.
"""
from __future__ import annotations

import math
import os
from dataclasses import dataclass, field, asdict
from typing import Optional

import numpy as np
from scipy.signal import lfilter

RHO = 0.98
NOISE = 0.5
SINK_K = 3.0
SINK_Q = 1.5
N_SINKS = 4
RETRIEVAL_FRAC = 0.01
RETRIEVAL_GAIN = 4.0


# --------------------------------------------------------------------------
# bf16 rounding (fp64 -> bf16 bits, round to nearest, ties to even)
# --------------------------------------------------------------------------
def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 values once to bf16 and return the 16-bit patterns (uint16).

    Rounds directly from fp64 (no intermediate fp32 rounding, so no double
    rounding): keeps 7 explicit mantissa bits of the fp64 value with
    round-half-to-even, then re-expresses the (now exactly bf16) value as fp32
    and takes its top 16 bits. Values are assumed finite and inside the bf16
    normal range or zero; tiny magnitudes below 2^-126 flush through fp32.
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    bits = x.view(np.uint64)
    drop = np.uint64(45)  # 52 - 7 mantissa bits dropped
    lsb = (bits >> drop) & np.uint64(1)
    rounded = (bits + (np.uint64(1) << np.uint64(44)) - np.uint64(1) + lsb) & ~((np.uint64(1) << drop) - np.uint64(1))
    y = rounded.view(np.float64).astype(np.float32)
    return (y.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact upcast of bf16 bit patterns to fp64."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------
# Workload descriptions
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class TrainWorkload:
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int
    d: int
    Bq: int
    Bk: int
    seed: int
    kind: str = "structured"  # or "iid"
    taus: tuple = (1.0,)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def describe(self) -> dict:
        out = asdict(self)
        out["scale"] = self.scale
        return out


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Lk: int
    d: int
    Bk: int
    seed: int
    taus: tuple = (1.0,)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def describe(self) -> dict:
        out = asdict(self)
        out["scale"] = self.scale
        return out


# The five workloads of the operator study, with their seeds.
C0 = TrainWorkload("mala_fwd_bwd_L1k_h2_d64", 1, 2, 2, 1024, 64, 64, 64, seed=1000, taus=(1.0,))
C1 = TrainWorkload("mala_fwd_bwd_L8k_h16_d128", 1, 16, 16, 8192, 128, 128, 128, seed=1001, taus=(0.0, 1.0))
C1_IID = TrainWorkload("mala_fwd_bwd_L8k_h16_d128_iid", 1, 16, 16, 8192, 128, 128, 128, seed=2001,
                       kind="iid", taus=(0.0, 1.0))
C2 = TrainWorkload("mala_fwd_bwd_L32k_gqa32x8_d128", 1, 32, 8, 32768, 128, 128, 128, seed=1002, taus=(1.0, 0.0))
C3 = TrainWorkload("mala_fwd_bwd_L128k_h8_d128", 1, 8, 8, 131072, 128, 128, 128, seed=1003, taus=(1.0, 0.0))
C4 = DecodeWorkload("mala_decode_B8_Lk128k_gqa32x8_d128", 8, 32, 8, 131072, 128, 128, seed=1004, taus=(1.0, 0.0))

WORKLOADS = {w.name: w for w in (C0, C1, C1_IID, C2, C3, C4)}


@dataclass(frozen=True)
class PackedWorkload:
    """A packed batch of training sequences laid end to end (lengths `lens`)."""
    name: str
    lens: tuple
    Hq: int
    Hkv: int
    d: int
    Bq: int
    Bk: int
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def total(self) -> int:
        return int(sum(self.lens))

    def describe(self) -> dict:
        out = asdict(self)
        out["scale"] = self.scale
        out["total"] = self.total
        return out


# A 32K-token packed batch: nine sequences of mixed, mostly ragged lengths
# (a long document down to a short one), GQA 32/8 as in the 32K workload.
C5 = PackedWorkload("mala_fwd_bwd_varlen_T32k_gqa32x8_d128",
                    (12000, 7300, 4100, 3000, 2600, 1500, 1111, 700, 457), 32, 8, 128, 128, 128, seed=1005)
SUBSET_SEED_OFFSET = 500


# --------------------------------------------------------------------------
# Slice generators
# --------------------------------------------------------------------------
def _stream(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def _ar1(z0: np.ndarray, eps: np.ndarray) -> np.ndarray:
    """z_0 given, z_t = RHO*z_{t-1} + sqrt(1-RHO^2)*eps_t along axis 0."""
    w = np.empty((eps.shape[0] + 1, z0.shape[0]), dtype=np.float64)
    w[0] = z0
    w[1:] = math.sqrt(1.0 - RHO * RHO) * eps
    return lfilter([1.0], [1.0, -RHO], w, axis=0)


def kv_slice(seed: int, b: int, h: int, L: int, d: int, kind: str = "structured"):
    """fp64 (z, k, v, u) for one (batch, KV head); z/u are None for iid."""
    g = _stream(seed, 0, b, h)
    if kind == "iid":
        k = g.standard_normal((L, d))
        v = g.standard_normal((L, d))
        return None, k, v, None
    z0 = g.standard_normal(d)
    eps = g.standard_normal((L - 1, d)) if L > 1 else np.zeros((0, d))
    z = _ar1(z0, eps)
    k = z + NOISE * g.standard_normal((L, d))
    uu = g.standard_normal(d)
    u = uu / np.linalg.norm(uu)
    k[: min(N_SINKS, L)] += SINK_K * u
    v = g.standard_normal((L, d))
    return z, k, v, u


def q_slice(seed: int, b: int, hq: int, L: int, d: int, z, k, u, kind: str = "structured"):
    """fp64 (q, dO) for one (batch, query head) given its KV head's z, k, u."""
    g = _stream(seed, 1, b, hq)
    if kind == "iid":
        q = g.standard_normal((L, d))
        do = g.standard_normal((L, d))
        return q, do
    q = z + NOISE * g.standard_normal((L, d))
    q += SINK_Q * u
    n_ret = int(math.floor(RETRIEVAL_FRAC * L))
    if n_ret > 0 and L > 1:
        rows = g.choice(np.arange(1, L), size=n_ret, replace=False)
        src = g.integers(0, rows)  # j uniform in {0..i-1}
        q[rows] += RETRIEVAL_GAIN * k[src]
    do = g.standard_normal((L, d))
    return q, do


def _train_kv_job(args):
    seed, b, h, L, d, kind, Hq, Hkv = args
    z, k, v, u = kv_slice(seed, b, h, L, d, kind)
    G = Hq // Hkv
    qs, dos = [], []
    for hq in range(h * G, (h + 1) * G):
        q, do = q_slice(seed, b, hq, L, d, z, k, u, kind)
        qs.append(to_bf16_bits(q))
        dos.append(to_bf16_bits(do))
    return b, h, to_bf16_bits(k), to_bf16_bits(v), qs, dos


def make_train_inputs(w: TrainWorkload, workers: int = 1, seed: Optional[int] = None,
                      L: Optional[int] = None):
    """bf16 bit tensors q, k, v, dO in BSHD layout ([B, L, H, d], uint16).

    ``L`` overrides the workload length (used for reduced cases with the same
    recipe); ``workers`` > 1 generates slices in a spawn-context process pool.
    """
    seed = w.seed if seed is None else seed
    L = w.L if L is None else L
    B, Hq, Hkv, d = w.B, w.Hq, w.Hkv, w.d
    q = np.empty((B, L, Hq, d), dtype=np.uint16)
    do = np.empty((B, L, Hq, d), dtype=np.uint16)
    k = np.empty((B, L, Hkv, d), dtype=np.uint16)
    v = np.empty((B, L, Hkv, d), dtype=np.uint16)
    jobs = [(seed, b, h, L, d, w.kind, Hq, Hkv) for b in range(B) for h in range(Hkv)]
    G = Hq // Hkv

    def _store(res):
        b, h, kb, vb, qs, dos = res
        k[b, :, h] = kb
        v[b, :, h] = vb
        for gi in range(G):
            q[b, :, h * G + gi] = qs[gi]
            do[b, :, h * G + gi] = dos[gi]

    if workers > 1 and len(jobs) > 1:
        import multiprocessing as mp
        from concurrent.futures import ProcessPoolExecutor
        with ProcessPoolExecutor(max_workers=min(workers, len(jobs)),
                                 mp_context=mp.get_context("spawn")) as ex:
            for res in ex.map(_train_kv_job, jobs):
                _store(res)
    else:
        for j in jobs:
            _store(_train_kv_job(j))
    return {"q": q, "k": k, "v": v, "do": do}


def make_packed_inputs(w: PackedWorkload, workers: int = 1):
    """bf16 bit tensors of a packed batch: q, dO [total, Hq, d], k, v [total, Hkv, d]
    (uint16) and cu_seqlens [S + 1] (int32). Sequence s is the training recipe for
    one sequence of length lens[s] with seed w.seed * 100 + s."""
    parts = {"q": [], "k": [], "v": [], "do": []}
    for s, L in enumerate(w.lens):
        t = make_train_inputs(TrainWorkload(w.name, 1, w.Hq, w.Hkv, int(L), w.d, w.Bq, w.Bk, seed=w.seed * 100 + s),
                              workers=workers)
        for x in parts:
            parts[x].append(t[x][0])
    out = {x: np.concatenate(v, 0) for x, v in parts.items()}
    out["cu_seqlens"] = np.concatenate([[0], np.cumsum(w.lens)]).astype(np.int32)
    return out


def _decode_kv_job(args):
    seed, b, h, Lk, d = args
    z, k, v, u = kv_slice(seed, b, h, Lk, d, "structured")
    return b, h, to_bf16_bits(k), to_bf16_bits(v), z[-1].copy(), u, k


def make_decode_inputs(w: DecodeWorkload, workers: int = 1, seed: Optional[int] = None,
                       Lk: Optional[int] = None):
    """bf16 bit tensors: q [B, Hq, d], kcache / vcache [B, Lk, Hkv, d]."""
    seed = w.seed if seed is None else seed
    Lk = w.Lk if Lk is None else Lk
    B, Hq, Hkv, d = w.B, w.Hq, w.Hkv, w.d
    G = Hq // Hkv
    kc = np.empty((B, Lk, Hkv, d), dtype=np.uint16)
    vc = np.empty((B, Lk, Hkv, d), dtype=np.uint16)
    q64 = np.empty((B, Hq, d), dtype=np.float64)
    kfull = {}
    jobs = [(seed, b, h, Lk, d) for b in range(B) for h in range(Hkv)]

    def _store(res):
        b, h, kb, vb, zlast, u, k64 = res
        kc[b, :, h] = kb
        vc[b, :, h] = vb
        kfull[(b, h)] = (k64, zlast, u)

    if workers > 1 and len(jobs) > 1:
        import multiprocessing as mp
        from concurrent.futures import ProcessPoolExecutor
        with ProcessPoolExecutor(max_workers=min(workers, len(jobs)),
                                 mp_context=mp.get_context("spawn")) as ex:
            for res in ex.map(_decode_kv_job, jobs):
                _store(res)
    else:
        for j in jobs:
            _store(_decode_kv_job(j))
    for b in range(B):
        for hq in range(Hq):
            h = hq // G
            _, zlast, u = kfull[(b, h)]
            g = _stream(seed, 2, b, hq)
            q64[b, hq] = zlast + NOISE * g.standard_normal(d) + SINK_Q * u
    n_ret = int(math.ceil(RETRIEVAL_FRAC * B * Hq))
    g = _stream(seed, 3)
    if Lk > 1:
        picks = g.choice(B * Hq, size=min(n_ret, B * Hq), replace=False)
        for p in picks:
            b, hq = divmod(int(p), Hq)
            j = int(g.integers(0, Lk - 1))
            q64[b, hq] += RETRIEVAL_GAIN * kfull[(b, hq // G)][0][j]
    return {"q": to_bf16_bits(q64), "kcache": kc, "vcache": vc}


def default_workers() -> int:
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(n, 32))
