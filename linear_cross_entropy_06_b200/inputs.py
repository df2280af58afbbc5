"""Seeded synthetic inputs shaped like the classifier heads the CCE pages discuss.

This module only draws random numbers: it holds none of the loss arithmetic, and
both the CUDA path's tests and the CPU oracle consume what it makes.

Workloads (mlx-cross-entropy README, "The problem" table and "Performance";
Cut Your Losses abstract; the problem sizes named for each workload below):

* ``tiny``              N=256,   D=128,  V=4096.   E ~ N(0,1), C ~ N(0,1/D), uniform
                        targets, 10% ignore_index.
* ``llama3.2-1b-head``  N=2048,  D=2048, V=128256. Peaked: E = alpha*C[t] + N(0,1),
                        uniform targets, 5% ignore_index.
* ``gemma2-2b-head``    N=2048,  D=2304, V=256000. Flat: E ~ N(0,1), C ~ N(0,1/D),
                        uniform targets; ``gemma2-2b-head-peaked`` is the peaked variant.
* ``llama3.1-8b-head``  N=4096,  D=4096, V=128256. Peaked, Zipf(1.1) targets, 5% ignore.
* ``long-batch``        N=32768, D=4096, V=128256. As llama3.1-8b-head, per-token loss
                        (reduction='none') with grad_out ~ N(0,1).

``alpha`` sets how peaked the softmax is. The values below were chosen with
``oracle/calibrate_alpha.py`` so that the mean softmax probability of the target
token is about 0.3 on a 256-row sample; they are plain constants here.

Random numbers come from numpy's PCG64 (``np.random.default_rng(seed)``), so a
seed gives the same inputs on every machine. bf16 copies are round-to-nearest-
even conversions of the fp32 draws.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

IGNORE_INDEX = -100

# Peaking factor per (D, V, target law), from oracle/calibrate_alpha.py.
ALPHA = {
    (2048, 128256, "uniform"): 11.2,  # mean p_target 0.301
    (2304, 256000, "uniform"): 11.98,  # mean p_target 0.298
    (4096, 128256, "zipf"): 11.27,  # mean p_target 0.300
}


@dataclass(frozen=True)
class Workload:
    name: str
    N: int
    D: int
    V: int
    targets: str = "uniform"  # "uniform" or "zipf"
    zipf_s: float = 1.1
    ignore_frac: float = 0.0
    peaked: bool = False
    reduction: str = "mean"
    grad_out: str = "one"  # "one" (scalar 1.0) or "normal" (per-token N(0,1))
    seed: int = 1234


WORKLOADS = {
    w.name: w
    for w in (
        Workload("tiny", 256, 128, 4096, "uniform", ignore_frac=0.10, seed=1235),
        Workload("llama3.2-1b-head", 2048, 2048, 128256, "uniform", ignore_frac=0.05, peaked=True, seed=1236),
        Workload("gemma2-2b-head", 2048, 2304, 256000, "uniform", seed=1237),
        Workload("gemma2-2b-head-peaked", 2048, 2304, 256000, "uniform", peaked=True, seed=1237),
        Workload("llama3.1-8b-head", 4096, 4096, 128256, "zipf", ignore_frac=0.05, peaked=True, seed=1238),
        Workload("long-batch", 32768, 4096, 128256, "zipf", ignore_frac=0.05, peaked=True,
                 reduction="none", grad_out="normal", seed=1239),
    )
}


@dataclass
class Inputs:
    workload: Workload
    E: torch.Tensor  # [N, D] bf16, CPU
    C: torch.Tensor  # [V, D] bf16, CPU
    targets: torch.Tensor  # [N] int64, CPU
    grad_out: torch.Tensor  # [1] or [N] fp32, CPU
    E32: Optional[torch.Tensor] = None  # fp32 originals (kept for the tiny case only)
    C32: Optional[torch.Tensor] = None
    alpha: float = 0.0
    extra: dict = field(default_factory=dict)


def zipf_targets(rng: np.random.Generator, n: int, V: int, s: float) -> np.ndarray:
    """Token ids with P(id = k-1) proportional to k^-s, k = 1..V (popular ids are small)."""
    w = np.arange(1, V + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    idx = np.searchsorted(cdf, rng.random(n), side="right")
    return np.minimum(idx, V - 1).astype(np.int64)


def make_inputs(name_or_workload, *, N: Optional[int] = None, D: Optional[int] = None,
                V: Optional[int] = None, seed: Optional[int] = None, alpha: Optional[float] = None,
                keep_fp32: Optional[bool] = None, ignore_frac: Optional[float] = None) -> Inputs:
    """Draw one workload's inputs; keyword overrides give ragged or reduced shapes."""
    w = WORKLOADS[name_or_workload] if isinstance(name_or_workload, str) else name_or_workload
    N = w.N if N is None else N
    D = w.D if D is None else D
    V = w.V if V is None else V
    seed = w.seed if seed is None else seed
    ignore_frac = w.ignore_frac if ignore_frac is None else ignore_frac
    if alpha is None:
        alpha = ALPHA.get((D, V, w.targets), 11.27) if w.peaked else 0.0
    keep_fp32 = (w.name == "tiny") if keep_fp32 is None else keep_fp32
    rng = np.random.default_rng(seed)

    C32 = rng.standard_normal((V, D), dtype=np.float32)
    C32 *= np.float32(1.0 / np.sqrt(D))
    if w.targets == "zipf":
        t = zipf_targets(rng, N, V, w.zipf_s)
    else:
        t = rng.integers(0, V, size=N, dtype=np.int64)
    E32 = rng.standard_normal((N, D), dtype=np.float32)
    if w.peaked and N > 0:
        E32 += np.float32(alpha) * C32[t]
    n_ign = int(round(ignore_frac * N))
    if n_ign:
        t[rng.permutation(N)[:n_ign]] = IGNORE_INDEX
    if w.grad_out == "normal":
        g = rng.standard_normal(N, dtype=np.float32)
    else:
        g = np.ones(1, dtype=np.float32)

    E32_t, C32_t = torch.from_numpy(E32), torch.from_numpy(C32)
    inp = Inputs(w, E32_t.to(torch.bfloat16), C32_t.to(torch.bfloat16), torch.from_numpy(t),
                 torch.from_numpy(g), alpha=float(alpha))
    if keep_fp32:
        inp.E32, inp.C32 = E32_t, C32_t
    return inp
