"""Matched-work fidelity report (fp64, CPU): MALA's retained keys vs the
reference-mass policy at the same key slots, on the 1K workload (both heads)
and the 8K workload (4 heads), tau in {0.5, 1, 4, 16}.

Run from the repository root: ``python tests/report_matched_work.py``.
"""
import math
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from oracle.matched_work import matched_work, summary  # noqa: E402
from workloads import C0, C1, bf16_bits_to_f64, make_train_inputs  # noqa: E402


def main():
    for w, heads in ((C0, None), (C1, [(0, h) for h in range(4)])):
        t = make_train_inputs(w)
        q, k, v = (bf16_bits_to_f64(t[x]) for x in ("q", "k", "v"))
        for tau in (0.5, 1.0, 4.0, 16.0):
            s = summary(matched_work(q, k, v, 1 / math.sqrt(w.d), tau, w.Bq, w.Bk, heads=heads))
            print(w.name, "heads", "all" if heads is None else len(heads), "tau", tau,
                  {x: (round(y, 6) if isinstance(y, float) else y) for x, y in s.items()}, flush=True)


if __name__ == "__main__":
    main()
