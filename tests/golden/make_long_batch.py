"""Writes long_batch_oracle.npz: the fp64 oracle's per-row LSE and per-token loss, its skip
decision for every tile (and which tiles lie within the oracle's borderline window of ln eps) for
the long-batch workload (N = 32768 tokens, D = 4096, V = 128256, Zipf
targets, 5 % ignored, reduction 'none', skipping at 2^-12 on units of 128 rows x 64 vocabulary
columns).

A full fp64 pass over that problem takes minutes of CPU time, so the GPU parity test reads these
values instead of recomputing them; it evaluates the cheaper parts (dE of whole row blocks, dC of
whole vocabulary tiles from the stored LSE) itself. Calls only the oracle and the seeded input
generator:

    python tests/golden/make_long_batch.py
"""
import hashlib
import math
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from linear_cross_entropy_06_b200.inputs import make_inputs  # noqa: E402
from oracle import cce_oracle as O  # noqa: E402

EPS = 2.0 ** -12
TILE = (128, 64)  # rows x vocabulary columns of the skip rule's unit
WINDOW = 2e-3  # the oracle's borderline window (its default)
OUT = os.path.join(HERE, "long_batch_oracle.npz")


def fingerprint(inp) -> str:
    """Hash of the exact bf16 inputs, so a reader can tell that it regenerated the same problem."""
    h = hashlib.sha256()
    for x in (inp.E, inp.C, inp.targets, inp.grad_out):
        h.update(x.contiguous().view(-1).view(dtype=__import__("torch").uint8).numpy().tobytes())
    return h.hexdigest()


def main():
    t0 = time.time()
    inp = make_inputs("long-batch")
    w = inp.workload
    s = O.sampled(inp.E, inp.C, inp.targets, [], [], inp.grad_out.numpy(), -100, w.reduction, EPS,
                  TILE[0], TILE[1], compute_cols=False)
    skipped = O.filtered_tiles(s.margin, EPS)
    near = np.abs(s.margin - math.log(EPS)) < WINDOW
    np.savez_compressed(OUT, lse=s.lse, nll=s.nll, count=s.count, filtered=s.filtered, borderline=s.borderline,
                        n_tiles=s.margin.size, tile=np.asarray(TILE), eps=EPS, window=WINDOW,
                        grid=np.asarray(s.margin.shape), skipped_bits=np.packbits(skipped.reshape(-1)),
                        borderline_bits=np.packbits(near.reshape(-1)), fingerprint=fingerprint(inp))
    print(f"wrote {OUT}: count {s.count}, skipped {s.filtered} of {s.margin.size} tiles, borderline {s.borderline}, "
          f"{time.time() - t0:.0f} s")


if __name__ == "__main__":
    main()
