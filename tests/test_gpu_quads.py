"""GPU parity on a planted pattern of kept 128 x 64 units of the skip rule.

A bias of +12 on eight tokens makes the same eight 64-column halves kept in every row block and
every other half skipped (its softmax is near exp(-14), far below 2^-12): both halves of
vocabulary tiles 0 and 3, one half of tiles 1, 2, 5 and 7, nothing in tiles 4 and 6. Each row
block then recomputes two items of four halves, [t0 h0, t0 h1, t1 h0, t2 h0] and
[t3 h0, t3 h1, t5 h0, t7 h1], which cross tiles. The dC MMAs read zeros for the skipped half of
tiles 1, 2, 5 and 7, and tiles 4 and 6 have no kept unit (their dC rows come from the empty-tile
fill). The targets are uniform, so most rows' targets lie in skipped halves, some of them in
listed tiles, and their onehot terms are applied row by row. The results are compared with the
fp64 oracle under the same rule (mlx-cross-entropy README, "How it works" item 2), and the skip
decision of every unit with the planted pattern.
"""
import numpy as np
import pytest
import torch

from linear_cross_entropy_06_b200 import ops
from linear_cross_entropy_06_b200.inputs import make_inputs

from test_gpu_bias import check_bias
from test_gpu_parity import EPS

pytestmark = pytest.mark.gpu

HOT = [5, 70, 130, 300, 390, 450, 700, 1000]  # one token in each planted half


def planted_bias(V):
    b = torch.zeros(V, dtype=torch.bfloat16)
    b[HOT] = 12.0
    return b


@pytest.mark.parametrize("reduction", ["mean", "none"])
def test_planted_halves(device, reduction):
    N, D, V = 384, 256, 1024
    inp = make_inputs("tiny", N=N, D=D, V=V, seed=91, ignore_frac=0.1)
    g = torch.from_numpy(np.random.default_rng(92).standard_normal(N).astype(np.float32)) \
        if reduction == "none" else torch.tensor([1.0])
    bias = planted_bias(V)
    r = check_bias(inp, bias, device, reduction, grad_out=g)
    tm, tn = ops.backward_tile_shape()
    kept_units = sorted({v // tn for v in HOT})
    assert r["filtered"] == (N // tm) * (V // tn) - (N // tm) * len(kept_units)

    # the skip map: exactly the planted units kept, in every row block
    E, C, t = inp.E.to(device), inp.C.to(device), inp.targets.to(device)
    gd = g.to(device) if reduction == "none" else g[:1].to(device)
    loss, lse, tmax, count = ops.cce_forward(E, C, t, -100, reduction, bias=bias.to(device))
    smap = ops.cce_backward(E, C, t, lse, tmax, count, gd, EPS, -100, reduction, bias=bias.to(device),
                            skip_map=True)[-1].cpu().numpy()
    want = np.ones((N // tm, V // tn), dtype=np.uint8)
    want[:, kept_units] = 0
    assert (smap == want).all(), smap
