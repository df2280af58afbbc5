"""Choose the peaking factor alpha of the synthetic inputs (E = alpha*C[t] + noise).

The workloads ask for a peaked softmax whose mean target probability is about
0.3. This script bisects alpha on a 256-row sample using only the fp64 oracle
and prints the value per (D, V, target law); the generator stores the results
as constants. Run: ``python oracle/calibrate_alpha.py``.
"""
from __future__ import annotations

import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from oracle.cce_oracle import forward_rows  # noqa: E402
from linear_cross_entropy_06_b200.inputs import WORKLOADS, make_inputs  # noqa: E402


def mean_target_prob(name: str, alpha: float, rows: int = 256) -> float:
    inp = make_inputs(name, N=rows, alpha=alpha, ignore_frac=0.0)
    _, lse, zt, _, valid = forward_rows(inp.E, inp.C, inp.targets)
    return float(np.exp(zt - lse)[valid].mean())


def calibrate(name: str, target: float = 0.3, lo: float = 4.0, hi: float = 20.0, iters: int = 9) -> float:
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if mean_target_prob(name, mid) < target:
            lo = mid
        else:
            hi = mid
    return round(0.5 * (lo + hi), 2)


if __name__ == "__main__":
    for name in ("llama3.2-1b-head", "gemma2-2b-head-peaked", "llama3.1-8b-head"):
        w = WORKLOADS[name]
        a = calibrate(name)
        print(f"({w.D}, {w.V}, {w.targets!r}): {a},  # mean p_target = {mean_target_prob(name, a):.3f}", flush=True)
