"""The pins of the oracle's Python compositions must catch plausible mistakes.

Packed batches, the paged decode and the single-pass decode are compositions
(in oracle/__init__.py) of the pinned single-sequence routines. Each case here
executes a copy of that module's source with one planted mistake -- a key
slice taken from the query offsets, queries aligned to the start of their
sequence, an LSE slice without its offset, pages in the wrong order, a last
page not cut at the sequence length, a single pass that splits -- and runs a
compact battery of the pins of tests/test_oracle_varlen.py against it. Every
mutant must fail at least one pin. The planted mistakes live only in the
executed copy; the committed module is untouched.
"""
import math
import types

import numpy as np
import pytest

import oracle
import mala_bruteforce as bf
from test_oracle import case
from test_oracle_varlen import _paged, packed_case

MUTANTS = {
    "varlen_keys_sliced_by_query_offsets": (
        'k[None, cu_k[s]:cu_k[s + 1]], v[None, cu_k[s]:cu_k[s + 1]],',
        'k[None, cu_q[s]:cu_q[s] + lk[s]], v[None, cu_q[s]:cu_q[s] + lk[s]],'),
    "varlen_queries_aligned_to_the_start": (
        'r = prefill(q[None, cu_q[s]:cu_q[s + 1]], k[None, cu_k[s]:cu_k[s + 1]], v[None, cu_k[s]:cu_k[s + 1]],',
        'r = prefill(q[None, cu_q[s]:cu_q[s + 1]], k[None, cu_k[s]:cu_k[s] + lq[s]], '
        'v[None, cu_k[s]:cu_k[s] + lq[s]],'),
    "varlen_bwd_lse_without_offset": ('lse[None, :, a:b],', 'lse[None, :, :b - a],'),
    "paged_pages_reversed": ('kc = kp[bt[b, :npg]]', 'kc = kp[bt[b, :npg][::-1]]'),
    "paged_last_page_not_cut": (
        'kc = kp[bt[b, :npg]].reshape(npg * page, kp.shape[2], d)[:Lk]',
        'kc = kp[bt[b, :npg]].reshape(npg * page, kp.shape[2], d)[:npg * page]'),
    "single_pass_splits": ('return decode(q, kc, vc, scale, tau, Bk, 1, sel=sel)',
                           'return decode(q, kc, vc, scale, tau, Bk, 2, sel=sel)'),
}


def _mutant_module(a, b):
    src = open(oracle.__file__).read()
    assert src.count(a) == 1, a
    mod = types.ModuleType("oracle_mutant")
    mod.__file__ = oracle.__file__  # the same compiled C library
    exec(compile(src.replace(a, b), oracle.__file__, "exec"), mod.__dict__)
    return mod


def _pins_pass(o) -> bool:
    """A compact battery of the composition pins; True iff all pass."""
    try:
        # packed forward with cached prefixes vs the brute force per sequence
        lens_q, lens_k = [5, 12, 9], [21, 12, 30]
        q, k, v, _, cu_q, cu_k = packed_case(lens_q, lens_k, 8, 2, 1, 82, 1.5)
        sc = 1 / math.sqrt(8)
        r = o.varlen_fwd(q, k, v, cu_q, cu_k, sc, 1.0, 4, 8)
        for s in range(3):
            a, b_ = cu_q[s], cu_q[s + 1]
            ref = bf.bf_prefill(q[None, a:b_], k[None, cu_k[s]:cu_k[s + 1]], v[None, cu_k[s]:cu_k[s + 1]], sc, 1.0,
                                4, 8)
            if not np.isfinite(r["o"][a:b_]).all() or np.abs(r["o"][a:b_] - ref["o"][0]).max() > 1e-9:
                return False
            if np.abs(r["lse"][:, a:b_] - ref["lse"][0]).max() > 1e-9:
                return False
        # packed backward vs the brute force per sequence
        lens = [12, 19]
        q, k, v, do, cu, _ = packed_case(lens, lens, 8, 2, 1, 95, 2.0)
        f = o.varlen_fwd(q, k, v, cu, cu, sc, 1.0, 4, 4)
        g = o.varlen_bwd(q, k, v, f["o"], do, f["lse"], cu, sc, 1.0, 4, 4)
        for s in range(2):
            a, b_ = cu[s], cu[s + 1]
            rf = bf.bf_forward(q[None, a:b_], k[None, a:b_], v[None, a:b_], sc, 1.0, 4, 4)
            rb = bf.bf_backward(q[None, a:b_], k[None, a:b_], v[None, a:b_], do[None, a:b_], sc, 1.0, 4, 4, rf)
            for name in ("dq", "dk", "dv"):
                if not np.isfinite(g[name][a:b_]).all() or np.abs(g[name][a:b_] - rb[name][0]).max() > 1e-8:
                    return False
        # paged decode (shuffled pool, partial last pages) vs the brute force
        rng = np.random.default_rng(9)
        plens, page = [37, 20], 8
        qs, kc, vc = [], [], []
        for b_, L in enumerate(plens):
            qq, kk, vv, _ = case(L, 8, 4, 2, seed=170 + b_, sharpen=2.0)
            qs.append(qq[0, -1])
            kc.append(kk[0])
            vc.append(vv[0])
        kp, vp, table = _paged(kc, vc, plens, page, rng)
        qd = np.stack(qs)
        r = o.paged_decode(qd, kp, vp, table, plens, sc, 1.0, 2)
        for b_, L in enumerate(plens):
            ref = bf.bf_decode(qd[b_:b_ + 1], kc[b_][None], vc[b_][None], sc, 1.0, page, 2)
            if np.abs(r["o"][b_] - ref["o"][0]).max() > 1e-9 or np.abs(r["lse"][b_] - ref["lse"][0]).max() > 1e-9:
                return False
        # the single pass is the forward's last query row
        qq, kk, vv, _ = case(48, 8, 2, 1, seed=180, sharpen=2.0)
        rs = o.decode_single_pass(qq[:, -1], kk, vv, sc, 1.0, 8)
        fw = o.fwd(qq, kk, vv, sc, 1.0, 1, 8)
        if np.abs(rs["o"] - fw["o"][:, -1]).max() > 1e-10 or np.abs(rs["lse"] - fw["lse"][:, :, -1]).max() > 1e-10:
            return False
        return True
    except (AssertionError, IndexError, ValueError):
        return False


def test_battery_passes_on_the_committed_oracle():
    assert _pins_pass(oracle)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    a, b = MUTANTS[name]
    assert not _pins_pass(_mutant_module(a, b)), name
