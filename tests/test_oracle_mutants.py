"""The oracle's pins must catch plausible mistakes.

Each case copies the oracle's C source to a temporary directory, plants one
mistake (a dropped term, a wrong sign, a wrong index, a wrong visit order, a
transposed operand), builds it with gcc and runs a fixed battery of pins
against the mutant. Every mutant must fail at least one pin. The planted
mistakes live only in the temporary copy; the committed oracle is untouched.
"""
import math
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
import mala_bruteforce as bf
from workloads import TrainWorkload, bf16_bits_to_f64, make_train_inputs

MUTANTS = {
    "drop_rescale_of_acc": ("for (int c = 0; c < d; ++c) ar[c] *= alpha;", ""),
    "lq_off_by_one": ("log((double)(P0 + i0 + r + 1))", "log((double)(P0 + i0 + r))"),
    "prefill_lq_ignores_offset": ("log((double)(P0 + i0 + r + 1))", "log((double)(i0 + r + 1))"),
    "prefill_first_tile_ignores_offset": ("const int kb_first = (P0 + i1 - 1) / Bk;",
                                          "const int kb_first = (i1 - 1) / Bk;"),
    "prefill_live_ignores_offset": ("if (j <= P0 + i) sv", "if (j <= i) sv"),
    "visit_order_reversed": ("for (int kb = kb_first; kb >= 0; --kb)", "for (int kb = 0; kb <= kb_first; ++kb)"),
    "gate_uses_max_not_ratio": ("(M[r] - m[r] - log(l[r])) - thr[r]", "(M[r] - m[r]) - thr[r]"),
    "ds_sign": ("const double dS = P * (dP - Di);\n                    for (int c = 0; c < d; ++c) dqi",
                "const double dS = P * (dP + Di);\n                    for (int c = 0; c < d; ++c) dqi"),
    "dq_drops_scale": ("dqi[c] += scale * dS * kj[c];", "dqi[c] += dS * kj[c];"),
    "bwd_gate_sign": ("- LSEi - thr;", "- LSEi + thr;"),
    "gqa_head_map": ("const int hkv = hq / G;\n    const int P0", "const int hkv = hq % Hkv;\n    const int P0"),
    "dk_uses_k_not_q": ("dkj[c] += scale * dS * qi[c];", "dkj[c] += scale * dS * gi[c];"),
    "decode_forces_oldest": ("if (kb == t1 - 1) keep = 1;", "if (kb == t0) keep = 1;"),
    "decode_lq_is_split_length": ("log((double)Lk)", "log((double)(Lk / n_splits + 1))"),
    "dv_transposed": ("dvj[c] += P * gi[c];", "dvj[c] += P * qi[c];"),
}


def _case(L, d, Hq, Hkv, seed, sharpen):
    w = TrainWorkload("tiny", 1, Hq, Hkv, L, d, 8, 8, seed=seed)
    t = make_train_inputs(w)
    q, k, v, do = (bf16_bits_to_f64(t[x]) for x in ("q", "k", "v", "do"))
    return q * sharpen, k, v, do


def _pins_pass() -> bool:
    """Run a compact battery of the oracle pins; True iff all pass."""
    try:
        # tau = 0 forward / backward vs torch fp64
        q, k, v, do = _case(40, 8, 4, 2, 7, 1.0)
        sc = 1 / math.sqrt(8)
        f = oracle.fwd(q, k, v, sc, 0.0, 8, 8)
        g = oracle.bwd(q, k, v, f["o"], do, f["lse"], sc, 0.0, 8, 8)
        qt, kt, vt = (torch.from_numpy(x).requires_grad_() for x in (q, k, v))
        o = torch.nn.functional.scaled_dot_product_attention(
            qt.permute(0, 2, 1, 3), kt.repeat_interleave(2, 2).permute(0, 2, 1, 3),
            vt.repeat_interleave(2, 2).permute(0, 2, 1, 3), is_causal=True, scale=sc).permute(0, 2, 1, 3)
        (o * torch.from_numpy(do)).sum().backward()
        if np.abs(f["o"] - o.detach().numpy()).max() > 1e-10:
            return False
        for name, ref in (("dq", qt.grad), ("dk", kt.grad), ("dv", vt.grad)):
            if not np.isfinite(g[name]).all() or np.abs(g[name] - ref.numpy()).max() > 1e-9:
                return False
        # tau > 0 vs the brute force (GQA case; tau = 4 makes the ln l term decide tiles)
        q, k, v, do = _case(64, 8, 2, 1, 71, 1.0)
        f = oracle.fwd(q, k, v, sc, 4.0, 8, 8)
        ref = bf.bf_forward(q, k, v, sc, 4.0, 8, 8)
        if not (f["keep"] == ref["keep"]).all() or np.abs(f["o"] - ref["o"]).max() > 1e-9:
            return False
        g = oracle.bwd(q, k, v, f["o"], do, f["lse"], sc, 4.0, 8, 8)
        rb = bf.bf_backward(q, k, v, do, sc, 4.0, 8, 8, ref)
        if not (g["keep"] == rb["keep"]).all():
            return False
        for name in ("dq", "dk", "dv"):
            if np.abs(g[name] - rb[name]).max() > 1e-8:
                return False
        # prefill against a cache (offset not a multiple of Bq, Bq != Bk) vs the brute force
        q, k, v, _ = _case(44, 8, 2, 1, 41, 1.5)
        for (tau, Bq, Bk) in ((1.0, 8, 4), (4.0, 4, 8)):
            r = oracle.prefill(q[:, 23:], k, v, sc, tau, Bq, Bk)
            rp = bf.bf_prefill(q[:, 23:], k, v, sc, tau, Bq, Bk)
            if not (r["keep"] == rp["keep"]).all() or np.abs(r["o"] - rp["o"]).max() > 1e-9:
                return False
            if np.abs(r["lse"] - rp["lse"]).max() > 1e-9:
                return False
        # decode vs the brute force
        q, k, v, _ = _case(50, 8, 2, 1, 31, 2.0)
        r = oracle.decode(q[:, -1], k, v, sc, 1.0, 8, 3)
        rd = bf.bf_decode(q[:, -1], k, v, sc, 1.0, 8, 3)
        if not (r["keep"] == rd["keep"]).all() or np.abs(r["o"] - rd["o"]).max() > 1e-9:
            return False
        return True
    except Exception:
        return False


def _build_variant(tmp_path, src_text, name):
    src = tmp_path / f"{name}.c"
    lib = tmp_path / f"lib{name}.so"
    src.write_text(src_text)
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", str(src), "-o", str(lib), "-lm"])
    return str(lib)


def _use(monkeypatch, lib_path):
    monkeypatch.setattr(oracle, "_LIB", lib_path)
    monkeypatch.setattr(oracle, "build", lambda force=False: lib_path)
    monkeypatch.setattr(oracle, "_lib", None)


def test_unmutated_copy_passes_the_battery(tmp_path, monkeypatch):
    text = open(oracle._SRC).read()
    _use(monkeypatch, _build_variant(tmp_path, text, "clean"))
    assert _pins_pass()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, monkeypatch, name):
    old, new = MUTANTS[name]
    text = open(oracle._SRC).read()
    assert text.count(old) == 1, f"mutation site for {name} not unique"
    _use(monkeypatch, _build_variant(tmp_path, text.replace(old, new), name))
    assert not _pins_pass(), f"pins did not catch mutant {name}"
