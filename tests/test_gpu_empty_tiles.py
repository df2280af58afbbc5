"""GPU parity of the vocabulary tiles no row block lists ("empty" tiles), against the fp64 oracle.

Every logit of such a tile is skipped, so its rows of dC hold only the target part of the logit
gradient, -scale_r (1 - ls) E_r summed over the rows r whose target is that token, plus the
label-smoothing term shared by every row (Loss functions explainer, "How it works" items 2 and 3;
mlx-cross-entropy README, "How it works" item 2). The library writes them in a kernel of their own
that runs beside the tensor-core kernel; these cases put many targets into one empty tile (longer
lists than the kernel holds at once) and the same token into many rows.

Inputs: the flat "tiny" draw at N=512, D=256, V=16384 with C scaled by 0.1, so every logit is
within a few tenths of 0 while LSE is near ln V: at eps = 2^-12 every tile is skipped and every
vocabulary tile is empty. Targets: rows 0-79 draw tokens of vocabulary tile 5, rows 80-119 all
take token 9 * 128 + 7, rows 120-131 are ignored, the rest stay uniform. Tolerances as in the other
parity tests.
"""
import numpy as np
import pytest
import torch

from linear_cross_entropy_06_b200.inputs import make_inputs

from test_gpu_bias import check_bias, make_bias

pytestmark = pytest.mark.gpu

TILE = 128  # vocabulary tile of the work lists
HALF = 64   # vocabulary columns of a skip-rule unit (half a tile)


def crowded_inputs(seed):
    inp = make_inputs("tiny", N=512, D=256, V=16384, seed=seed, ignore_frac=0.0)
    inp.C = (inp.C.float() * 0.1).to(torch.bfloat16)
    t = inp.targets.clone()
    rng = np.random.default_rng(seed + 1)
    t[:80] = torch.from_numpy(rng.integers(5 * TILE, 6 * TILE, size=80))
    t[80:120] = 9 * TILE + 7
    t[120:132] = -100
    inp.targets = t
    return inp


@pytest.mark.parametrize("variant", ["plain", "bias+smoothing+z-loss"])
@pytest.mark.parametrize("reduction", ["mean", "none"])
def test_empty_tiles_with_long_target_lists(device, variant, reduction):
    inp = crowded_inputs(81)
    N, V = inp.E.shape[0], inp.C.shape[0]
    g = torch.from_numpy(np.random.default_rng(82).standard_normal(N).astype(np.float32)) \
        if reduction == "none" else torch.tensor([1.0])
    if variant == "plain":
        r = check_bias(inp, None, device, reduction, grad_out=g)
    else:
        r = check_bias(inp, make_bias(V, 83, scale=0.05), device, reduction, grad_out=g, ls=0.1, zl=1e-4)
    assert r["filtered"] == (N // TILE) * (V // HALF)  # every half skipped at eps = 2^-12


def test_empty_tiles_fp32_outputs(device):
    inp = crowded_inputs(84)
    r = check_bias(inp, make_bias(inp.C.shape[0], 85, scale=0.05), device, "sum", grad_out=torch.tensor([0.5]),
                   out_fp32=True, ls=0.2)
    assert r["filtered"] == (512 // TILE) * (16384 // HALF)


@pytest.mark.parametrize("D,out_fp32", [(33000, False), (16400, True)])
def test_empty_tiles_wider_than_the_image(device, D, out_fp32):
    """A dC row wider than the kernel's 64 KB shared-memory image (bf16 D > 32768, fp32 D > 16384):
    the constant row goes out in column windows. A bias of 20 on token 5 puts every row's LSE near
    20, so every vocabulary tile but the first is skipped in every row block (the targets elsewhere
    keep their onehot rows), and the first tile keeps only the half that holds token 5 (its other
    half reads as zeros in the dC MMAs), with label smoothing for a non-zero constant row."""
    N, V = 128, 1024
    inp = make_inputs("tiny", N=N, D=D, V=V, seed=86 + D, ignore_frac=0.05)
    bias = torch.zeros(V, dtype=torch.bfloat16)
    bias[5] = 20.0
    r = check_bias(inp, bias, device, "mean", out_fp32=out_fp32, ls=0.1)
    assert r["filtered"] == (N // TILE) * (V // HALF) - 1  # only the half holding token 5 is kept
