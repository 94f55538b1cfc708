"""MALA benchmark: one JSON line on rank 0.

A step is one MALA training pass of the attention operator -- mala_fwd then
mala_bwd -- on the 32K GQA workload (B=1, Hq=32, Hkv=8, L=32768, d=128,
Bq=Bk=128, tau=1) with inputs resident in HBM. The same run also measures
the library's tau=0 path (full attention) on the same inputs and the decode
workload (B=8, Lk=131072, Hq=32, Hkv=8, d=128, Bk=128), reported as
sub-objects of the same line.

  value      effective TFLOP/s, whole job: FLOPs counted as QK over every live
             causal pair plus post-score matmuls over the live pairs of kept
             tiles (fwd 2d*N_legal + 2d*N_f, bwd 2d*N_legal + 8d*N_b), summed
             over ranks, divided by the max-over-ranks device time
  e2e        the same metric through the C ABI starting from pinned host
             buffers: every step's H2D of q, k, v, dO and D2H of dq, dk, dv
             inside the timed region, overlapped with the neighbouring steps'
             compute (two device buffer sets, a copy stream per direction)
  roofline   the dominant kernel's achieved rate against the measured peak

Multi-GPU (torchrun): every rank runs its own copy of the workload (a per-GPU
head slice, as in head-sharded attention); no collective on the data path;
scaling is weak. `--impl reference` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import C1, C1_IID, C2, C3, C4, C5, WORKLOADS, default_workers  # noqa: E402

METRIC = "MALA fwd+bwd ms & eff. TFLOP/s (% bf16 peak) at 32K/128K, τ=1; retained-tile %"
L2_BYTES = 126 * 1024 * 1024


# --------------------------------------------------------------------------
# Work accounting (host logic; unit-tested on CPU)
# --------------------------------------------------------------------------
def live_pairs(L: int, Bq: int, Bk: int) -> np.ndarray:
    """[nq, nk] number of live (i, j <= i) pairs of every tile."""
    nq, nk = -(-L // Bq), -(-L // Bk)
    out = np.zeros((nq, nk), dtype=np.int64)
    for qb in range(nq):
        i = np.arange(qb * Bq, min((qb + 1) * Bq, L))
        for kb in range(nk):
            j0, j1 = kb * Bk, min((kb + 1) * Bk, L)
            out[qb, kb] = np.clip(np.minimum(i, j1 - 1) - j0 + 1, 0, None).sum()
    return out


def train_flops(d: int, B: int, Hq: int, L: int, live: np.ndarray, keep_f, keep_b):
    """Effective FLOPs of one fwd and one bwd (keep maps [B,Hq,nq,nk] or None = all kept)."""
    n_legal = B * Hq * int(live.sum())
    n_f = n_legal if keep_f is None else int(((keep_f == 1) * live).sum())
    n_b = n_legal if keep_b is None else int(((keep_b == 1) * live).sum())
    return {"n_legal": n_legal, "n_f": n_f, "n_b": n_b,
            "fwd": 2 * d * n_legal + 2 * d * n_f, "bwd": 2 * d * n_legal + 8 * d * n_b}


def packed_flops(lens, Hq, d, Bq, Bk, keep_f, keep_b):
    """Effective FLOPs of one fwd and one bwd of a packed training batch: each
    sequence's live pairs with its corner [nq_s, nk_s] of the keep maps
    [S, Hq, max_nq, max_nk] (None = all kept). Also returns the legal-tile count
    and the kept fwd / bwd tiles."""
    fl = {"n_legal": 0, "n_f": 0, "n_b": 0, "fwd": 0, "bwd": 0, "tiles": 0, "kept_f": 0, "kept_b": 0}
    for s_, L in enumerate(lens):
        live = live_pairs(L, Bq, Bk)
        a, b_ = live.shape
        kf = None if keep_f is None else keep_f[s_:s_ + 1, :, :a, :b_]
        kb = None if keep_b is None else keep_b[s_:s_ + 1, :, :a, :b_]
        f1 = train_flops(d, 1, Hq, L, live, kf, kb)
        for key_ in ("n_legal", "n_f", "n_b", "fwd", "bwd"):
            fl[key_] += f1[key_]
        n_t = Hq * int((live > 0).sum())
        fl["tiles"] += n_t
        fl["kept_f"] += n_t if kf is None else int((kf == 1).sum())
        fl["kept_b"] += n_t if kb is None else int((kb == 1).sum())
    return fl


def walked_key_tiles(B: int, Hq: int, L: int, Bk: int) -> int:
    """Key tiles the forward's CTAs walk in a training forward: each CTA owns a
    pair of 128-row query tiles of one (b, hq) and visits key tiles 0 .. the
    tile of the pair's last row."""
    return B * Hq * sum((min(pr * 256 + 256, L) - 1) // Bk + 1 for pr in range(-(-L // 256)))


def pair_v_tiles(km, L: int, Bq: int) -> int:
    """V tiles the default forward loads: a CTA owns a pair of 128-row query
    tiles of one (b, hq) and loads a key tile's V once if some query block of
    the pair keeps it."""
    km = np.asarray(km)
    per = 256 // Bq
    nq = km.shape[2]
    return int(sum((km[:, :, pr * per:min((pr + 1) * per, nq), :] == 1).any(axis=2).sum()
                   for pr in range(-(-L // 256))))


def decode_bytes(B, Hq, Hkv, Lk, d, Bk, keep_map):
    """Algorithmic bytes of one decode step: all K, V of tiles kept by >= 1 head of
    the group, q in and o out (bf16)."""
    nk = -(-Lk // Bk)
    rows = np.array([min((t + 1) * Bk, Lk) - t * Bk for t in range(nk)], dtype=np.int64)
    G = Hq // Hkv
    if keep_map is None:
        v_tiles = np.ones((B, Hkv, nk), dtype=bool)
    else:
        v_tiles = (keep_map.reshape(B, Hkv, G, nk) == 1).any(axis=2)
    k_all = B * Lk * Hkv * d * 2
    v_kept = int((v_tiles * rows[None, None, :]).sum()) * d * 2
    return {"k_all": k_all, "v_kept": v_kept, "qo": 2 * B * Hq * d * 2, "total": k_all + v_kept + 2 * B * Hq * d * 2,
            "v_tile_frac": float(v_tiles.mean())}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# --------------------------------------------------------------------------
# Clock sampling during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", self.gpu_id], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------
# CUDA arm
# --------------------------------------------------------------------------
def bench_config(w, tau, world):
    """The `config` object of the JSON line (identical in both arms)."""
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L, "d": w.d, "Bq": w.Bq, "Bk": w.Bk,
            "tau": tau, "scale": w.scale, "seed": w.seed, "parallelism": f"replicas x{world} (head slices)",
            "l2": "inputs larger than L2 (no flush)"}


def _dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def dist_max(x: float, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def run_cuda(args):
    import torch
    import mass_gated_causal_b200 as mala

    world, rank, local = _dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    barrier = dist_barrier

    def max_over_ranks(x: float) -> float:
        return dist_max(x, dev)

    pk = peaks()
    w = WORKLOADS[args.workload]
    tau = 1.0
    workers = default_workers()
    t_gen = time.time()
    from workloads import make_train_inputs
    inp = make_train_inputs(w, workers=workers)
    t_gen = time.time() - t_gen

    def to_dev(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    q, k, v, do = (to_dev(inp[x]) for x in ("q", "k", "v", "do"))
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    stream = torch.cuda.current_stream(dev)
    # outputs and workspace allocated once
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    kept_f = torch.empty((B * Hq,), dtype=torch.int32, device=dev)
    kept_b = torch.empty((B * Hq,), dtype=torch.int32, device=dev)
    ws_bytes = mala.mala_bwd_workspace_size(B, Hq, L, d)
    ws = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    fws_bytes = mala.mala_fwd_workspace_size(B, Hkv, L, d)
    fws = torch.empty((fws_bytes,), dtype=torch.uint8, device=dev)
    nq, nk = -(-L // w.Bq), -(-L // w.Bk)

    def step(tau_, km_f=None, km_b=None):
        rc = mala.mala_fwd(q, k, v, o, lse, B, Hq, Hkv, L, d, w.scale, tau_, w.Bq, w.Bk, fws, fws_bytes, kept_f, km_f,
                           stream)
        assert rc == 0, mala.mala_status_string(rc)
        rc = mala.mala_bwd(q, k, v, o, do, lse, dq, dk, dv, B, Hq, Hkv, L, d, w.scale, tau_, w.Bq, w.Bk, ws,
                           ws_bytes, kept_b, km_b, stream)
        assert rc == 0, mala.mala_status_string(rc)

    # one diagnostic pass with keep maps: retained tiles and the FLOP count
    live = live_pairs(L, w.Bq, w.Bk)
    km_f = torch.zeros((B, Hq, nq, nk), dtype=torch.uint8, device=dev)
    km_b = torch.zeros((B, Hq, nq, nk), dtype=torch.uint8, device=dev)
    step(tau, km_f, km_b)
    assert mala.mala_check_status(stream) == 0
    kmf, kmb = km_f.cpu().numpy(), km_b.cpu().numpy()
    fl = train_flops(d, B, Hq, L, live, kmf, kmb)
    fl0 = train_flops(d, B, Hq, L, live, None, None)
    legal = (live > 0)
    kept_frac_f = (kmf == 1).reshape(B * Hq, -1).sum(1) / legal.sum()
    kept_frac_b = (kmb == 1).reshape(B * Hq, -1).sum(1) / legal.sum()
    del km_f, km_b

    def timed(fn, steps, warmup):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize(dev)
        barrier()
        torch.cuda.synchronize(dev)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
               torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for e0, e1, e2 in ev:
            e0.record(stream)
            fn(e1)
            e2.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        torch.cuda.synchronize(dev)
        tot = [e0.elapsed_time(e2) for e0, e1, e2 in ev]
        first = [e0.elapsed_time(e1) for e0, e1, e2 in ev]
        second = [e1.elapsed_time(e2) for e0, e1, e2 in ev]
        return tot, first, second

    def train_step(tau_):
        def fn(mid=None):
            rc = mala.mala_fwd(q, k, v, o, lse, B, Hq, Hkv, L, d, w.scale, tau_, w.Bq, w.Bk, fws, fws_bytes, kept_f,
                               None, stream)
            assert rc == 0
            if mid is not None:
                mid.record(stream)
            rc = mala.mala_bwd(q, k, v, o, do, lse, dq, dk, dv, B, Hq, Hkv, L, d, w.scale, tau_, w.Bq, w.Bk, ws,
                               ws_bytes, kept_b, None, stream)
            assert rc == 0
        return fn

    gpu_id = str(local)
    try:
        props = torch.cuda.get_device_properties(dev)
        if getattr(props, "uuid", None) is not None:
            u = str(props.uuid)
            gpu_id = u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        pass

    with ClockSampler(gpu_id) as clk:
        tot1, f1, b1 = timed(train_step(tau), args.steps, args.warmup)
    clocks = clk.summary()
    assert mala.mala_check_status(stream) == 0
    ms = max_over_ranks(float(np.mean(tot1)))
    ms_f = max_over_ranks(float(np.mean(f1)))
    ms_b = max_over_ranks(float(np.mean(b1)))
    step_flops = fl["fwd"] + fl["bwd"]
    value = world * step_flops / (ms * 1e-3) / 1e12

    # tau = 0 (full attention) on the same inputs
    tot0, f0, b0 = timed(train_step(0.0), max(2, args.steps // 2), max(3, args.warmup // 2))
    ms0 = max_over_ranks(float(np.mean(tot0)))
    ms0_f = max_over_ranks(float(np.mean(f0)))
    ms0_b = max_over_ranks(float(np.mean(b0)))
    flops0 = fl0["fwd"] + fl0["bwd"]

    # larger tau on the same inputs: how the step time follows the retained work
    sweep = {}
    km_by_tau = {tau: kmf}
    for tau_s in (4.0, 16.0):
        km_f = torch.zeros((B, Hq, nq, nk), dtype=torch.uint8, device=dev)
        km_b = torch.zeros((B, Hq, nq, nk), dtype=torch.uint8, device=dev)
        step(tau_s, km_f, km_b)
        assert mala.mala_check_status(stream) == 0
        kf_s, kb_s = km_f.cpu().numpy(), km_b.cpu().numpy()
        km_by_tau[tau_s] = kf_s
        del km_f, km_b
        fl_s = train_flops(d, B, Hq, L, live, kf_s, kb_s)
        tot_s, f_s, b_s = timed(train_step(tau_s), 3, 3)
        ms_s = max_over_ranks(float(np.mean(tot_s)))
        sweep[f"tau{int(tau_s)}"] = {
            "ms_per_step": round(ms_s, 3), "fwd_ms": round(max_over_ranks(float(np.mean(f_s))), 3),
            "bwd_ms": round(max_over_ranks(float(np.mean(b_s))), 3),
            "tflops": round(world * (fl_s["fwd"] + fl_s["bwd"]) / (ms_s * 1e-3) / 1e12, 2),
            "retained_tiles_fwd": round(float((kf_s == 1).sum() / (legal.sum() * B * Hq)), 4),
            "retained_tiles_bwd": round(float((kb_s == 1).sum() / (legal.sum() * B * Hq)), 4),
            "speedup_vs_tau0": round(ms0 / ms_s, 3)}
    assert mala.mala_check_status(stream) == 0

    # the opt-in V prefetch (mala_fwd_ex, MALA_FWD_PREFETCH_V: every V tile fetched
    # ahead of the vote) against the default (V requested only for kept tiles):
    # the forward alone, same inputs and decisions
    def fwd_only(tau_, flags):
        def fn(mid=None):
            rc = mala.mala_fwd_ex(q, k, v, o, lse, B, Hq, Hkv, L, d, w.scale, tau_, w.Bq, w.Bk, fws, fws_bytes,
                                  kept_f, None, stream, flags)
            assert rc == 0
            if mid is not None:
                mid.record(stream)
        return fn

    prefetch = {}
    walked = walked_key_tiles(B, Hq, L, w.Bk)
    for tau_p in sorted(km_by_tau):
        t_dem, _, _ = timed(fwd_only(tau_p, 0), 5, 3)
        t_pre, _, _ = timed(fwd_only(tau_p, mala.MALA_FWD_PREFETCH_V), 5, 3)
        ms_dem, ms_pre = max_over_ranks(float(np.mean(t_dem))), max_over_ranks(float(np.mean(t_pre)))
        prefetch[f"tau{tau_p:g}"] = {
            "fwd_ms_v_on_demand": round(ms_dem, 3), "fwd_ms_v_prefetched": round(ms_pre, 3),
            "v_tiles_on_demand_frac": round(pair_v_tiles(km_by_tau[tau_p], L, w.Bq) / walked, 4),
            "v_tiles_prefetched_frac": 1.0}
    assert mala.mala_check_status(stream) == 0

    # matched work (the pages' fidelity comparison) on the CUDA forward's keep map
    mw = matched_work_sample(torch, dev, q, k, v, kmf, w, n_blocks=8, seed=w.seed + 600)

    # e2e through the C ABI from pinned host buffers
    hq_, hk_, hv_, hdo_ = (torch.from_numpy(inp[x].view(np.int16)).view(torch.bfloat16).pin_memory()
                           for x in ("q", "k", "v", "do"))
    hdq = torch.empty(dq.shape, dtype=torch.bfloat16).pin_memory()
    hdk = torch.empty(dk.shape, dtype=torch.bfloat16).pin_memory()
    hdv = torch.empty(dv.shape, dtype=torch.bfloat16).pin_memory()
    h2d = sum(t.numel() * 2 for t in (hq_, hk_, hv_, hdo_))
    d2h = sum(t.numel() * 2 for t in (hdq, hdk, hdv))

    # Each step copies its inputs in and reads its gradients back. Two device
    # buffer sets and one stream per copy direction let the copies of steps
    # n + 1 (in) and n (out) overlap the compute of step n, as a training loop
    # with prefetching would; the timed region spans all K steps' copies and
    # ends once the last gradients are on the host.
    cp_in, cp_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    sets = [(q, k, v, do, dq, dk, dv), tuple(torch.empty_like(t) for t in (q, k, v, do, dq, dk, dv))]
    ev_in = [torch.cuda.Event() for _ in range(2)]   # inputs of set s have landed
    ev_cmp = [torch.cuda.Event() for _ in range(2)]  # the step on set s is done
    ev_out = [torch.cuda.Event() for _ in range(2)]  # gradients of set s are on the host

    def copy_in(s_):
        with torch.cuda.stream(cp_in):
            cp_in.wait_event(ev_cmp[s_])  # the step that last read set s_ is done
            for dst, src in zip(sets[s_][:4], (hq_, hk_, hv_, hdo_)):
                dst.copy_(src, non_blocking=True)
            ev_in[s_].record(cp_in)

    def step_on(s_, tau_):
        q_, k_, v_, do_, dq_, dk_, dv_ = sets[s_]
        stream.wait_event(ev_in[s_])
        stream.wait_event(ev_out[s_])  # its gradient buffers were read back two steps ago
        rc = mala.mala_fwd(q_, k_, v_, o, lse, B, Hq, Hkv, L, d, w.scale, tau_, w.Bq, w.Bk, fws, fws_bytes, kept_f,
                           None, stream)
        assert rc == 0
        rc = mala.mala_bwd(q_, k_, v_, o, do_, lse, dq_, dk_, dv_, B, Hq, Hkv, L, d, w.scale, tau_, w.Bq, w.Bk, ws,
                           ws_bytes, kept_b, None, stream)
        assert rc == 0
        ev_cmp[s_].record(stream)
        with torch.cuda.stream(cp_out):
            cp_out.wait_event(ev_cmp[s_])
            for dst, src in zip((hdq, hdk, hdv), (dq_, dk_, dv_)):
                dst.copy_(src, non_blocking=True)
            ev_out[s_].record(cp_out)

    def e2e_run(nsteps):
        copy_in(0)
        for n_ in range(nsteps):
            if n_ + 1 < nsteps:
                copy_in((n_ + 1) & 1)
            step_on(n_ & 1, tau)
        stream.wait_event(ev_out[(nsteps - 1) & 1])

    # as many steps as the device-timed region: the first input copy and the last
    # gradient read-back are not overlapped with anything and are paid once
    n_e2e = max(3, args.steps)
    e2e_run(max(3, args.warmup))
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    cp_in.wait_event(e_start)  # the first input copy is inside the timed region
    e2e_run(n_e2e)
    e_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    assert mala.mala_check_status(stream) == 0
    ms_e2e = max_over_ranks(e_start.elapsed_time(e_end) / n_e2e)
    del sets

    # the same fwd+bwd step on the 128K workload (the metric is quoted at 32K and 128K)
    long_leg = None
    if not args.no_long and w.name != C3.name:
        long_leg = run_train_leg(C3, mala, torch, dev, stream, pk, workers, timed, max_over_ranks, world,
                                 oracle_seconds=0.0 if (args.no_cpu or rank != 0 or world > 1) else 8.0)

    # a packed batch of mixed lengths (32K tokens in all)
    varlen_leg = None
    if not args.no_varlen:
        varlen_leg = run_varlen_leg(C5, mala, torch, dev, stream, pk, workers, timed, max_over_ranks, world)

    # the 8K workloads (structured and diffuse inputs): gate overhead in the low-skip regime
    legs_8k = None
    if not args.no_8k:
        legs_8k = {x.name: run_train_leg(x, mala, torch, dev, stream, pk, workers, timed, max_over_ranks, world,
                                         oracle_seconds=0.0 if (args.no_cpu or rank != 0 or world > 1) else 3.0)
                   for x in (C1, C1_IID)}

    # decode workload
    dec = None
    if not args.no_decode:
        dec = run_decode(args, mala, torch, dev, stream, pk, workers, timed, max_over_ranks, world,
                         oracle_seconds=0.0 if (args.no_cpu or rank != 0 or world > 1) else 8.0)

    # roofline of the dominant kernel (fwd or bwd call, timed with events on its stream)
    peak_t = pk["bf16_tflops_sustained"]
    t_fwd = fl["fwd"] / (ms_f * 1e-3) / 1e12
    t_bwd = fl["bwd"] / (ms_b * 1e-3) / 1e12
    dom = "mala_bwd_kernel" if ms_b >= ms_f else "mala_fwd_kernel"
    ach = t_bwd if dom == "mala_bwd_kernel" else t_fwd
    traffic = args.traffic if args.traffic is not None else profiled_traffic(dom, w.name)
    roof = {"kernel": dom, "bound": "tensor", "achieved": round(ach, 2), "peak": peak_t, "unit": "TFLOP/s",
            "frac": round(ach / peak_t, 4), "traffic": traffic,
            "peak_kind": f"bf16 dense, {pk['source']} sustained",
            "timed_unit": "mala_bwd call (pre + main + dq convert kernels)" if dom == "mala_bwd_kernel"
            else "mala_fwd call (one kernel)",
            "fwd": {"ms": round(ms_f, 3), "tflops": round(t_fwd, 2), "frac": round(t_fwd / peak_t, 4)},
            "bwd": {"ms": round(ms_b, 3), "tflops": round(t_bwd, 2), "frac": round(t_bwd / peak_t, 4)}}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(w, inp, tau, args.cpu_seconds)

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded structured generator)",
        "config": bench_config(w, tau, world),
        "frac_of_peak": round(value / world / peak_t, 4),
        "retained_tiles": {"fwd_mean": round(float(kept_frac_f.mean()), 4),
                           "fwd_min": round(float(kept_frac_f.min()), 4),
                           "fwd_max": round(float(kept_frac_f.max()), 4),
                           "bwd_mean": round(float(kept_frac_b.mean()), 4),
                           "bwd_min": round(float(kept_frac_b.min()), 4),
                           "bwd_max": round(float(kept_frac_b.max()), 4),
                           "live_pair_frac_fwd": round(fl["n_f"] / fl["n_legal"], 4),
                           "live_pair_frac_bwd": round(fl["n_b"] / fl["n_legal"], 4)},
        "fwd_ms": round(ms_f, 3), "bwd_ms": round(ms_b, 3), "step_tflop": round(step_flops / 1e12, 3),
        "tau0_ms_per_step": round(ms0, 3), "mala_speedup": round(ms0 / ms,  3),
        "tau_sweep": sweep, "fwd_prefetch_v": prefetch, "matched_work": mw,
        "fullattn_tau0": {"ms_per_step": round(ms0, 3), "fwd_ms": round(ms0_f, 3), "bwd_ms": round(ms0_b, 3),
                          "tflops": round(world * flops0 / (ms0 * 1e-3) / 1e12, 3),
                          "frac_of_peak": round(flops0 / (ms0 * 1e-3) / 1e12 / peak_t, 4),
                          "mala_speedup": round(ms0 / ms, 3)},
        "e2e": {"value": round(world * step_flops / (ms_e2e * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_step": round(ms_e2e, 3), "steps": n_e2e, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "copies": "overlapped with compute (two buffer sets, a stream per direction)"},
        "roofline": roof,
        "gpu_launches": 5 * args.steps,
        "clocks": clocks,
        "peaks": pk,
        "input_gen_s": round(t_gen, 1),
    }
    if long_leg is not None:
        line["at_128k"] = long_leg
    if varlen_leg is not None:
        line["varlen"] = varlen_leg
    if legs_8k is not None:
        line["at_8k"] = legs_8k
    if dec is not None:
        line["decode"] = dec
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def run_train_leg(w, mala, torch, dev, stream, pk, workers, timed, max_over_ranks, world, steps=3, warmup=3,
                  oracle_seconds=0.0):
    """fwd+bwd at tau = 1 and tau = 0 on workload `w` (ms, effective TFLOP/s, retained tiles); with
    oracle_seconds > 0 also the CPU oracle on a seeded sample of query blocks, with the full run extrapolated."""
    from workloads import make_train_inputs
    inp = make_train_inputs(w, workers=workers)
    to_dev = lambda bits: torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
    q, k, v, do = (to_dev(inp[x]) for x in ("q", "k", "v", "do"))
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    kept_f = torch.empty((B * Hq,), dtype=torch.int32, device=dev)
    kept_b = torch.empty((B * Hq,), dtype=torch.int32, device=dev)
    ws_bytes = mala.mala_bwd_workspace_size(B, Hq, L, d)
    ws = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    fws_bytes = mala.mala_fwd_workspace_size(B, Hkv, L, d)
    fws = torch.empty((fws_bytes,), dtype=torch.uint8, device=dev)
    nq, nk = -(-L // w.Bq), -(-L // w.Bk)

    def step(tau_, km_f=None, km_b=None, mid=None):
        rc = mala.mala_fwd(q, k, v, o, lse, B, Hq, Hkv, L, d, w.scale, tau_, w.Bq, w.Bk, fws, fws_bytes, kept_f,
                           km_f, stream)
        assert rc == 0, mala.mala_status_string(rc)
        if mid is not None:
            mid.record(stream)
        rc = mala.mala_bwd(q, k, v, o, do, lse, dq, dk, dv, B, Hq, Hkv, L, d, w.scale, tau_, w.Bq, w.Bk, ws,
                           ws_bytes, kept_b, km_b, stream)
        assert rc == 0, mala.mala_status_string(rc)

    live = live_pairs(L, w.Bq, w.Bk)
    km_f = torch.zeros((B, Hq, nq, nk), dtype=torch.uint8, device=dev)
    km_b = torch.zeros((B, Hq, nq, nk), dtype=torch.uint8, device=dev)
    step(1.0, km_f, km_b)
    assert mala.mala_check_status(stream) == 0
    kmf, kmb = km_f.cpu().numpy(), km_b.cpu().numpy()
    del km_f, km_b
    fl = train_flops(d, B, Hq, L, live, kmf, kmb)
    fl0 = train_flops(d, B, Hq, L, live, None, None)
    legal = (live > 0)
    kept_frac_f = (kmf == 1).reshape(B * Hq, -1).sum(1) / legal.sum()
    kept_frac_b = (kmb == 1).reshape(B * Hq, -1).sum(1) / legal.sum()
    out = {"workload": w.name, "B": B, "Hq": Hq, "Hkv": Hkv, "L": L, "d": d, "Bq": w.Bq, "Bk": w.Bk, "steps": steps,
           "warmup": warmup,
           "retained_tiles": {"fwd_mean": round(float(kept_frac_f.mean()), 4),
                              "bwd_mean": round(float(kept_frac_b.mean()), 4),
                              "live_pair_frac_fwd": round(fl["n_f"] / fl["n_legal"], 4),
                              "live_pair_frac_bwd": round(fl["n_b"] / fl["n_legal"], 4)}}
    peak_t = pk["bf16_tflops_sustained"]
    for tau_, flops, key in ((1.0, fl["fwd"] + fl["bwd"], "tau1"), (0.0, fl0["fwd"] + fl0["bwd"], "tau0")):
        tot, f, b_ = timed(lambda mid=None, t_=tau_: step(t_, mid=mid), steps, warmup)
        ms = max_over_ranks(float(np.mean(tot)))
        tf = world * flops / (ms * 1e-3) / 1e12
        out[key] = {"ms_per_step": round(ms, 3), "fwd_ms": round(max_over_ranks(float(np.mean(f))), 3),
                    "bwd_ms": round(max_over_ranks(float(np.mean(b_))), 3), "tflops": round(tf, 2),
                    "frac_of_peak": round(tf / world / peak_t, 4)}
    assert mala.mala_check_status(stream) == 0
    out["mala_speedup"] = round(out["tau0"]["ms_per_step"] / out["tau1"]["ms_per_step"], 3)
    if oracle_seconds > 0:
        out["oracle"] = oracle_subset(w, inp, 1.0, oracle_seconds, fl["fwd"] + fl["bwd"])
    del inp
    return out


def run_varlen_leg(w, mala, torch, dev, stream, pk, workers, timed, max_over_ranks, world, steps=3, warmup=3):
    """fwd+bwd of a packed batch (mala_fwd_varlen + mala_bwd_varlen) at tau = 1 and tau = 0."""
    from workloads import make_packed_inputs
    inp = make_packed_inputs(w, workers=workers)
    to_dev = lambda bits: torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
    q, k, v, do = (to_dev(inp[x]) for x in ("q", "k", "v", "do"))
    cu = torch.from_numpy(inp["cu_seqlens"]).to(dev)
    del inp
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    S, Lmax = len(w.lens), max(w.lens)
    o = torch.empty_like(q)
    lse = torch.empty((Hq, T), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    kept_f = torch.empty((S * Hq,), dtype=torch.int32, device=dev)
    kept_b = torch.empty((S * Hq,), dtype=torch.int32, device=dev)
    ws_bytes = mala.mala_bwd_workspace_size(1, Hq, T, d)
    ws = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    fws_bytes = mala.mala_fwd_workspace_size(1, Hkv, T, d)
    fws = torch.empty((fws_bytes,), dtype=torch.uint8, device=dev)
    nq, nk = -(-Lmax // w.Bq), -(-Lmax // w.Bk)

    def step(tau_, km_f=None, km_b=None, mid=None):
        rc = mala.mala_fwd_varlen(q, k, v, o, lse, cu, cu, S, Lmax, Lmax, T, T, Hq, Hkv, d, w.scale, tau_, w.Bq, w.Bk,
                                  fws, fws_bytes, kept_f, km_f, stream)
        assert rc == 0, mala.mala_status_string(rc)
        if mid is not None:
            mid.record(stream)
        rc = mala.mala_bwd_varlen(q, k, v, o, do, lse, dq, dk, dv, cu, S, Lmax, T, Hq, Hkv, d, w.scale, tau_, w.Bq,
                                  w.Bk, ws, ws_bytes, kept_b, km_b, stream)
        assert rc == 0, mala.mala_status_string(rc)

    km_f = torch.zeros((S, Hq, nq, nk), dtype=torch.uint8, device=dev)
    km_b = torch.zeros((S, Hq, nq, nk), dtype=torch.uint8, device=dev)
    step(1.0, km_f, km_b)
    assert mala.mala_check_status(stream) == 0
    kmf, kmb = km_f.cpu().numpy(), km_b.cpu().numpy()
    del km_f, km_b
    fl = packed_flops(w.lens, Hq, d, w.Bq, w.Bk, kmf, kmb)
    fl0 = packed_flops(w.lens, Hq, d, w.Bq, w.Bk, None, None)
    n_tiles, kept_tf, kept_tb = fl["tiles"], fl["kept_f"], fl["kept_b"]
    out = {"workload": w.name, "lens": list(w.lens), "total": T, "Hq": Hq, "Hkv": Hkv, "d": d, "Bq": w.Bq,
           "Bk": w.Bk, "steps": steps, "warmup": warmup,
           "retained_tiles": {"fwd": round(kept_tf / n_tiles, 4), "bwd": round(kept_tb / n_tiles, 4),
                              "live_pair_frac_fwd": round(fl["n_f"] / fl["n_legal"], 4),
                              "live_pair_frac_bwd": round(fl["n_b"] / fl["n_legal"], 4)}}
    peak_t = pk["bf16_tflops_sustained"]
    for tau_, flops, key in ((1.0, fl["fwd"] + fl["bwd"], "tau1"), (0.0, fl0["fwd"] + fl0["bwd"], "tau0")):
        tot, f, b_ = timed(lambda mid=None, t_=tau_: step(t_, mid=mid), steps, warmup)
        ms = max_over_ranks(float(np.mean(tot)))
        tf = world * flops / (ms * 1e-3) / 1e12
        out[key] = {"ms_per_step": round(ms, 3), "fwd_ms": round(max_over_ranks(float(np.mean(f))), 3),
                    "bwd_ms": round(max_over_ranks(float(np.mean(b_))), 3), "tflops": round(tf, 2),
                    "frac_of_peak": round(tf / world / peak_t, 4)}
    assert mala.mala_check_status(stream) == 0
    out["mala_speedup"] = round(out["tau0"]["ms_per_step"] / out["tau1"]["ms_per_step"], 3)
    return out


def run_paged_decode(args, mala, torch, dev, stream, pk, timed, max_over_ranks, q, kc, vc, w, contiguous):
    """The decode workload's cache scattered into shuffled page pools (page = Bk):
    the same bytes as the contiguous decode, read through the block table."""
    B, Hq, d = q.shape
    Lk, Hkv = kc.shape[1], kc.shape[2]
    page = w.Bk
    npg = -(-Lk // page)
    assert npg * page == Lk
    g = torch.Generator().manual_seed(w.seed + 77)
    perm = torch.randperm(B * npg, generator=g).to(dev)
    kp = torch.empty((B * npg, page, Hkv, d), dtype=kc.dtype, device=dev)
    vp = torch.empty_like(kp)
    kp[perm] = kc.reshape(B * npg, page, Hkv, d)
    vp[perm] = vc.reshape(B * npg, page, Hkv, d)
    table = perm.to(torch.int32).reshape(B, npg).contiguous()
    sl = torch.full((B,), Lk, dtype=torch.int32, device=dev)
    ns = contiguous["n_splits"]
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    kept = torch.empty((B * Hq,), dtype=torch.int32, device=dev)
    wsb = mala.mala_decode_workspace_size(B, Hq, d, ns)
    ws = torch.empty((wsb,), dtype=torch.uint8, device=dev)
    out = {"workload": w.name + "_paged", "page": page, "num_pages": B * npg, "n_splits": ns,
           "layout": "pages shuffled over the pool (seeded permutation)"}
    for tau in (1.0, 0.0):
        km = torch.zeros((B, Hq, npg), dtype=torch.uint8, device=dev)
        rc = mala.mala_decode_paged(q, kp, vp, table, sl, o, lse, B, Hq, Hkv, B * npg, page, npg, d, w.scale, tau, ns,
                                    ws, wsb, kept, km, stream)
        assert rc == 0
        assert mala.mala_check_status(stream) == 0
        by = decode_bytes(B, Hq, Hkv, Lk, d, page, km.cpu().numpy())
        del km

        def fn(mid=None, tau_=tau):
            rc_ = mala.mala_decode_paged(q, kp, vp, table, sl, o, lse, B, Hq, Hkv, B * npg, page, npg, d, w.scale, tau_,
                                         ns, ws, wsb, kept, None, stream)
            assert rc_ == 0
            if mid is not None:
                mid.record(stream)
        tot, _, _ = timed(fn, max(5, args.steps * 2), max(3, args.warmup))
        us = max_over_ranks(float(np.median(tot))) * 1e3
        gbs = by["total"] / (us * 1e-6) / 1e9
        key = f"tau{int(tau)}"
        out[key] = {"us_per_step": round(us, 1), "us_per_token": round(us / B, 2), "GBps": round(gbs, 1),
                    "frac_of_hbm": round(gbs / pk["hbm_gbs"], 4), "bytes_per_step": by["total"],
                    "vs_contiguous": round(contiguous[key]["us_per_step"] / us, 3)}
    assert mala.mala_check_status(stream) == 0
    del kp, vp
    return out


def run_decode(args, mala, torch, dev, stream, pk, workers, timed, max_over_ranks, world, oracle_seconds=0.0):
    from workloads import make_decode_inputs
    w = C4
    inp = make_decode_inputs(w, workers=workers)

    def to_dev(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    q, kc, vc = (to_dev(inp[x]) for x in ("q", "kcache", "vcache"))
    B, Hq, d = q.shape
    Lk, Hkv = kc.shape[1], kc.shape[2]
    ns = mala.mala_decode_default_splits(B, Hkv, Lk, w.Bk)
    nk = -(-Lk // w.Bk)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    kept = torch.empty((B * Hq,), dtype=torch.int32, device=dev)
    wsb = mala.mala_decode_workspace_size(B, Hq, d, ns)
    ws = torch.empty((wsb,), dtype=torch.uint8, device=dev)
    out = {"workload": w.name, "B": B, "Hq": Hq, "Hkv": Hkv, "Lk": Lk, "d": d, "Bk": w.Bk, "n_splits": ns}
    for tau in (1.0, 0.0):
        km = torch.zeros((B, Hq, nk), dtype=torch.uint8, device=dev)
        rc = mala.mala_decode(q, kc, vc, o, lse, B, Hq, Hkv, Lk, d, w.scale, tau, w.Bk, ns, ws, wsb, kept, km, stream)
        assert rc == 0
        assert mala.mala_check_status(stream) == 0
        kmh = km.cpu().numpy()
        by = decode_bytes(B, Hq, Hkv, Lk, d, w.Bk, kmh)
        del km

        def fn(mid=None, tau_=tau):
            rc_ = mala.mala_decode(q, kc, vc, o, lse, B, Hq, Hkv, Lk, d, w.scale, tau_, w.Bk, ns, ws, wsb, kept, None,
                                   stream)
            assert rc_ == 0
            if mid is not None:
                mid.record(stream)
        tot, _, _ = timed(fn, max(5, args.steps * 2), max(3, args.warmup))
        us = max_over_ranks(float(np.median(tot))) * 1e3
        gbs = by["total"] / (us * 1e-6) / 1e9
        out[f"tau{int(tau)}"] = {"us_per_step": round(us, 1), "us_per_token": round(us / B, 2),
                                 "GBps": round(gbs, 1), "frac_of_hbm": round(gbs / pk["hbm_gbs"], 4),
                                 "bytes_per_step": by["total"], "v_tile_frac": round(by["v_tile_frac"], 4),
                                 "retained_tile_frac_per_head": round(float((kmh == 1).mean()), 4)}
    out["mala_speedup"] = round(out["tau0"]["us_per_step"] / out["tau1"]["us_per_step"], 3)
    out["hbm_peak_gbs"] = pk["hbm_gbs"]
    out["paged"] = run_paged_decode(args, mala, torch, dev, stream, pk, timed, max_over_ranks, q, kc, vc, w, out)
    out["exact"] = run_exact_decode(args, mala, torch, dev, stream, pk, timed, max_over_ranks, q, kc, vc, w, out)
    if oracle_seconds > 0:
        out["oracle"] = oracle_decode_subset(w, inp, 1.0, ns, oracle_seconds, out["tau1"]["us_per_step"])
    return out


def run_exact_decode(args, mala, torch, dev, stream, pk, timed, max_over_ranks, q, kc, vc, w, contiguous):
    """mala_decode_exact on the decode workload: the single-pass decisions, the
    same split count for the PV work. Algorithmic bytes as for mala_decode (K,
    V of the kept tiles, q, o); the fp32 scores it writes and reads back are
    reported beside them."""
    B, Hq, d = q.shape
    Lk, Hkv = kc.shape[1], kc.shape[2]
    ns = contiguous["n_splits"]
    nk = -(-Lk // w.Bk)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    kept = torch.empty((B * Hq,), dtype=torch.int32, device=dev)
    wsb = mala.mala_decode_exact_workspace_size(B, Hq, Lk, d, w.Bk, ns)
    ws = torch.empty((wsb,), dtype=torch.uint8, device=dev)
    aux = 2 * B * Hq * nk * w.Bk * 4  # scores written once, read once
    out = {"workload": w.name + "_exact", "n_splits": ns, "scores_bytes_per_step": aux}
    for tau in (1.0, 0.0):
        km = torch.zeros((B, Hq, nk), dtype=torch.uint8, device=dev)
        rc = mala.mala_decode_exact(q, kc, vc, o, lse, B, Hq, Hkv, Lk, d, w.scale, tau, w.Bk, ns, ws, wsb, kept, km,
                                    stream)
        assert rc == 0
        assert mala.mala_check_status(stream) == 0
        kmh = km.cpu().numpy()
        by = decode_bytes(B, Hq, Hkv, Lk, d, w.Bk, kmh)
        del km

        def fn(mid=None, tau_=tau):
            rc_ = mala.mala_decode_exact(q, kc, vc, o, lse, B, Hq, Hkv, Lk, d, w.scale, tau_, w.Bk, ns, ws, wsb, kept,
                                         None, stream)
            assert rc_ == 0
            if mid is not None:
                mid.record(stream)
        tot, _, _ = timed(fn, max(5, args.steps * 2), max(3, args.warmup))
        us = max_over_ranks(float(np.median(tot))) * 1e3
        gbs = by["total"] / (us * 1e-6) / 1e9
        key = f"tau{int(tau)}"
        out[key] = {"us_per_step": round(us, 1), "us_per_token": round(us / B, 2), "GBps": round(gbs, 1),
                    "frac_of_hbm": round(gbs / pk["hbm_gbs"], 4),
                    "frac_of_hbm_with_scores": round((by["total"] + aux) / (us * 1e-6) / 1e9 / pk["hbm_gbs"], 4),
                    "bytes_per_step": by["total"], "v_tile_frac": round(by["v_tile_frac"], 4),
                    "retained_tile_frac_per_head": round(float((kmh == 1).mean()), 4),
                    "vs_split_decode": round(contiguous[key]["us_per_step"] / us, 3)}
    assert mala.mala_check_status(stream) == 0
    return out


def matched_work_sample(torch, dev, q, k, v, keep_map, w, n_blocks, seed):
    """The pages' matched-work comparison (agihunt.info MALA digest, fidelity
    paragraphs) on a seeded sample of query blocks, from the CUDA forward's keep
    map: per row, MALA's key slots (the live keys of its kept tiles), its omitted
    probability mass and output error against dense attention, and the same for
    the reference-mass policy given the same number of slots (the row's largest
    probabilities). MALA's output is the softmax over its retained keys, which is
    what the forward computes up to rounding. fp64 on the GPU with torch: a
    diagnostic beside the measurement, not part of the operator."""
    rng = np.random.default_rng(seed)
    B, L, Hq, d = q.shape
    G = Hq // k.shape[2]
    nq = keep_map.shape[2]
    acc = {x: [] for x in ("slots", "live", "omit_mala", "omit_ref", "err_mala", "err_ref")}
    ar = torch.arange(L, device=dev)
    sample = []
    for _ in range(n_blocks):
        b, h, qb = int(rng.integers(B)), int(rng.integers(Hq)), int(rng.integers(nq))
        sample.append((b, h, qb))
        rows = torch.arange(qb * w.Bq, min((qb + 1) * w.Bq, L), device=dev)
        kk, vv = k[b, :, h // G].double(), v[b, :, h // G].double()
        live = ar[None, :] <= rows[:, None]
        sc = (q[b, rows, h].double() @ kk.T) * w.scale
        p = torch.softmax(sc.masked_fill(~live, float("-inf")), dim=1)
        o_dense = p @ vv
        kept_keys = torch.from_numpy(np.repeat(keep_map[b, h, qb] == 1, w.Bk)[:L].copy()).to(dev)
        ret = live & kept_keys[None, :]
        slots = ret.sum(1)
        pm = p * ret
        omit_mala = 1.0 - pm.sum(1)
        o_mala = (pm @ vv) / pm.sum(1, keepdim=True)
        order = torch.argsort(p, dim=1, descending=True, stable=True)
        rank = torch.empty_like(order)
        rank.scatter_(1, order, ar[None, :].expand(len(rows), L).contiguous())
        pr = torch.where(rank < slots[:, None], p, torch.zeros_like(p))
        omit_ref = 1.0 - pr.sum(1)
        o_ref = (pr @ vv) / pr.sum(1, keepdim=True)
        nrm = o_dense.norm(dim=1)
        for key_, val in (("slots", slots), ("live", live.sum(1)), ("omit_mala", omit_mala), ("omit_ref", omit_ref),
                          ("err_mala", (o_mala - o_dense).norm(dim=1) / nrm),
                          ("err_ref", (o_ref - o_dense).norm(dim=1) / nrm)):
            acc[key_].append(val.double().cpu().numpy())
        del sc, p, pm, pr, order, rank
    r = {x: np.concatenate(v_) for x, v_ in acc.items()}
    return {"rows": int(r["slots"].size), "blocks": n_blocks, "tau": 1.0,
            "slot_frac": round(float(r["slots"].sum() / r["live"].sum()), 4),
            "slots_per_query_mean": round(float(r["slots"].mean()), 1),
            "omitted_mass_mala_mean": float(f"{r['omit_mala'].mean():.4g}"),
            "omitted_mass_ref_mean": float(f"{r['omit_ref'].mean():.4g}"),
            "omitted_mass_mala_max": float(f"{r['omit_mala'].max():.4g}"),
            "out_rel_err_mala_mean": float(f"{r['err_mala'].mean():.4g}"),
            "out_rel_err_ref_mean": float(f"{r['err_ref'].mean():.4g}"),
            "keep_map": "CUDA forward (the diagnostic pass)", "precision": "fp64 (torch on the GPU)",
            "sample": f"{n_blocks} seeded query blocks (b, hq, qb): {sample}"}


# --------------------------------------------------------------------------
# CPU oracle (baseline leg and the reference arm)
# --------------------------------------------------------------------------
def oracle_sample(w, inp, tau, n_blocks, seed):
    """Seeded sample of query blocks; the timed oracle work is forward of those
    blocks plus the dQ part of their backward."""
    rng = np.random.default_rng(seed)
    nq = -(-w.L // w.Bq)
    qb = rng.choice(nq, size=min(n_blocks, nq * w.B * w.Hq), replace=True)
    hq = rng.integers(0, w.Hq, size=qb.shape[0])
    b = rng.integers(0, w.B, size=qb.shape[0])
    return [(int(x), int(y), int(z)) for x, y, z in zip(b, hq, qb)]


def run_oracle_sample(w, qf, kf, vf, dof, tau, sel):
    import oracle
    live = live_pairs(w.L, w.Bq, w.Bk)
    t0 = time.perf_counter()
    f = oracle.fwd(qf, kf, vf, w.scale, tau, w.Bq, w.Bk, sel=sel, with_margin=False)
    o = np.nan_to_num(f["o"])
    lse = np.nan_to_num(f["lse"])
    g = oracle.bwd(qf, kf, vf, o, dof, lse, w.scale, tau, w.Bq, w.Bk, selq=sel, selk=[], with_margin=False)
    dt = time.perf_counter() - t0
    flops = 0
    for (b, h, qb) in sel:
        row_live = live[qb]
        nf = int(((f["keep"][b, h, qb] == 1) * row_live).sum())
        nbk = int(((g["keep"][b, h, qb] == 1) * row_live).sum())
        nl = int(row_live.sum())
        flops += (2 * w.d * nl + 2 * w.d * nf) + (2 * w.d * nl + 4 * w.d * nbk)  # fwd + (QK, dP, dQ)
    return flops, dt


def cpu_baseline(w, inp, tau, seconds):
    import oracle
    from workloads import bf16_bits_to_f64
    qf, kf, vf, dof = (bf16_bits_to_f64(inp[x]) for x in ("q", "k", "v", "do"))
    n = 4
    flops = dt = 0.0
    # grow the sample until it costs about `seconds` of host time
    while True:
        sel = oracle_sample(w, inp, tau, n, seed=w.seed + 500)
        flops, dt = run_oracle_sample(w, qf, kf, vf, dof, tau, sel)
        if dt >= seconds / 4 or n >= 4096:
            break
        n *= 2
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle", "sample": f"{len(sel)} seeded query blocks of {w.name}: forward + dQ part of "
                                        f"the backward, {flops / 1e9:.1f} GFLOP effective in {dt:.1f} s"}


def oracle_subset(w, inp, tau, seconds, full_flops):
    """The oracle on a seeded sample of query blocks (forward + dQ part of the
    backward), grown to about `seconds` of host time; the full fwd+bwd run is
    extrapolated by effective FLOPs (the sample's against the whole step's)."""
    import oracle
    from workloads import bf16_bits_to_f64
    qf, kf, vf, dof = (bf16_bits_to_f64(inp[x]) for x in ("q", "k", "v", "do"))
    n = 2
    while True:
        sel = oracle_sample(w, inp, tau, n, seed=w.seed + 500)
        flops, dt = run_oracle_sample(w, qf, kf, vf, dof, tau, sel)
        if dt >= seconds / 3 or n >= 1024:
            break
        n *= 2
    return {"kind": "oracle", "cores": oracle.num_threads(), "subset_blocks": len(sel),
            "subset_ms": round(dt * 1e3, 1), "subset_gflop": round(flops / 1e9, 2),
            "tflops": round(flops / dt / 1e12, 6),
            "extrapolated_full_step_ms": round(dt * 1e3 * full_flops / flops, 0),
            "sample": f"{len(sel)} seeded query blocks of {w.name}: forward + dQ part of the backward; the full "
                      f"step is extrapolated by effective FLOPs"}


def oracle_decode_subset(w, inp, tau, n_splits, seconds, full_us):
    """The oracle's decode on a seeded sample of (b, query head) rows, grown to
    about `seconds`; the full step is extrapolated by rows."""
    import oracle
    from workloads import bf16_bits_to_f64
    rng = np.random.default_rng(w.seed + 500)
    b0 = int(rng.integers(0, w.B))  # one sequence's cache in fp64 (about 2 GB at 128K) bounds host memory
    qf, kf, vf = (bf16_bits_to_f64(inp[x][b0:b0 + 1]) for x in ("q", "kcache", "vcache"))
    rows_all = [(0, h) for h in range(w.Hq)]
    n = 2
    while True:
        idx = rng.permutation(len(rows_all))[:n]
        sel = [rows_all[i] for i in idx]
        t0 = time.perf_counter()
        oracle.decode(qf, kf, vf, w.scale, tau, w.Bk, n_splits, sel=sel)
        dt = time.perf_counter() - t0
        if dt >= seconds / 3 or n >= len(rows_all):
            break
        n = min(2 * n, len(rows_all))
    full_ms = dt * 1e3 * w.B * w.Hq / len(sel)
    return {"kind": "oracle", "cores": oracle.num_threads(), "subset_rows": len(sel), "subset_ms": round(dt * 1e3, 1),
            "extrapolated_full_step_ms": round(full_ms, 1), "gpu_speedup": round(full_ms * 1e3 / full_us, 1),
            "sample": f"{len(sel)} seeded (b, query head) rows of {w.name} (split decode, same split count); the "
                      f"full step is extrapolated by rows"}


def run_reference(args):
    world, rank, _ = _dist_env()
    if rank != 0:
        return
    import oracle
    from workloads import bf16_bits_to_f64, make_train_inputs
    w = WORKLOADS[args.workload]
    tau = 1.0
    inp = make_train_inputs(w, workers=default_workers())
    qf, kf, vf, dof = (bf16_bits_to_f64(inp[x]) for x in ("q", "k", "v", "do"))
    n = max(4, args.ref_blocks)
    for i in range(args.warmup):
        run_oracle_sample(w, qf, kf, vf, dof, tau, oracle_sample(w, inp, tau, 2, seed=w.seed + 900 + i))
    times, fl = [], []
    for s in range(args.steps):
        sel = oracle_sample(w, inp, tau, n, seed=w.seed + 1000 + s)
        f, dt = run_oracle_sample(w, qf, kf, vf, dof, tau, sel)
        times.append(dt)
        fl.append(f)
    value = sum(fl) / sum(times) / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * float(np.mean(times)), 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded structured generator)",
            "config": bench_config(w, tau, world),
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
                             "kind": "oracle",
                             "sample": f"each step: {n} seeded query blocks of {w.name}, forward + dQ part "
                                       f"of the backward"},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_kernel_case(args):
    """One op on a small case (inputs still larger than L2), for ncu captures:
    fwd / bwd: B=1, Hq=Hkv=16, L=16384, d=128, tau=1; decode and decode_exact:
    B=8, Lk=32768, Hq=32, Hkv=8, d=128. Runs warmup + steps calls and prints the
    mean ms."""
    import torch
    import mass_gated_causal_b200 as mala
    from workloads import TrainWorkload, DecodeWorkload, make_decode_inputs, make_train_inputs
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)

    def to_dev(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    if args.kernel in ("fwd", "bwd"):
        w = TrainWorkload("prof_L16k_h16_d128", 1, 16, 16, 16384, 128, 128, 128, seed=1001)
        inp = make_train_inputs(w, workers=default_workers())
        q, k, v, do = (to_dev(inp[x]) for x in ("q", "k", "v", "do"))
        o, lse, _, _ = mala.forward(q, k, v, w.scale, 1.0, w.Bq, w.Bk)
        if args.kernel == "fwd":
            def fn():
                mala.forward(q, k, v, w.scale, 1.0, w.Bq, w.Bk)
        else:
            ws = torch.empty((mala.mala_bwd_workspace_size(1, 16, 16384, 128),), dtype=torch.uint8, device=dev)

            def fn():
                mala.backward(q, k, v, o, do, lse, w.scale, 1.0, w.Bq, w.Bk, workspace=ws)
    else:
        w = DecodeWorkload("prof_decode_B8_Lk32k", 8, 32, 8, 32768, 128, 128, seed=1004)
        inp = make_decode_inputs(w, workers=default_workers())
        q, kc, vc = (to_dev(inp[x]) for x in ("q", "kcache", "vcache"))

        if args.kernel == "decode":
            def fn():
                mala.decode(q, kc, vc, w.scale, 1.0, w.Bk)
        else:
            def fn():
                mala.decode_exact(q, kc, vc, w.scale, 1.0, w.Bk)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    assert mala.mala_check_status() == 0
    print(json.dumps({"kernel_case": args.kernel, "workload": w.name, "ms_mean": e0.elapsed_time(e1) / args.steps}))


def kernel_sources_sha256(kernel):
    """Hash of the sources that define `kernel` (its header and the shared PTX helpers)."""
    import hashlib
    csrc = os.path.join(ROOT, "mass_gated_causal_b200", "csrc")
    name = {"mala_bwd_kernel": "mala_bwd.cuh", "mala_fwd_kernel": "mala_fwd.cuh",
            "mala_decode_split_kernel": "mala_decode.cuh"}[kernel]
    h = hashlib.sha256()
    for f in (name, "mala_ptx.cuh"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def profiled_traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` on `workload` from a committed ncu summary
    (profiles/<kernel>_<workload>_dram.md), or None when there is none or when the
    kernel's sources have changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}_dram.md")
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as fh:
        for line in fh:
            if ":" in line and line.startswith("- "):
                k, v = line[2:].split(":", 1)
                fields[k.strip()] = v.strip().strip("`")
    if fields.get("sources-sha256") != kernel_sources_sha256(kernel):
        return None
    try:
        return float(fields["dram-bytes-per-launch"])
    except (KeyError, ValueError):
        return None


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("cuda", "reference"), default="cuda")
    ap.add_argument("--workload", default=C2.name, choices=sorted(k for k, v in WORKLOADS.items() if hasattr(v, "L")))
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-long", action="store_true", help="skip the 128K fwd+bwd leg")
    ap.add_argument("--no-varlen", action="store_true", help="skip the packed-batch fwd+bwd leg")
    ap.add_argument("--no-8k", action="store_true", help="skip the 8K structured / diffuse fwd+bwd legs")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--ref-blocks", type=int, default=16)
    ap.add_argument("--kernel", choices=("fwd", "bwd", "decode", "decode_exact"), default=None,
                    help="run one op on a small case (for profiler captures) instead of the benchmark")
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per launch of the dominant kernel from an ncu capture (reported as is)")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "cuda":
        args.warmup = 3
    if args.kernel is not None:
        run_kernel_case(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()
