"""GPU parity of the loss variants against the fp64 oracle: label smoothing and the z-loss (Loss
functions explainer, "How it works" item 3 and "Implementation notes"), alone and together, with
and without a bias and tile skipping; and the causal token shift of linear_cross_entropy.

Tolerances as in the other parity tests (loss and LSE 2e-3 absolute; dE, dC, dbias relative
Frobenius 1e-2 of the oracle that applies the same tile rule, with the elementwise bound).
"""
import numpy as np
import pytest
import torch

from linear_cross_entropy_06_b200 import ops
from linear_cross_entropy_06_b200.inputs import make_inputs
from oracle import cce_oracle as O

from test_gpu_bias import check_bias, make_bias
from test_gpu_parity import EPS, LOSS_TOL, rel_frob

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("ls,zl", [(0.1, 0.0), (0.0, 1e-4), (0.1, 1e-2), (1.0, 0.0)])
@pytest.mark.parametrize("reduction", ["mean", "none"])
def test_variants_tiny(device, ls, zl, reduction):
    inp = make_inputs("tiny")
    g = torch.from_numpy(np.random.default_rng(5).standard_normal(inp.E.shape[0]).astype(np.float32))
    check_bias(inp, None, device, reduction, grad_out=g if reduction == "none" else torch.tensor([1.0]), ls=ls, zl=zl)


@pytest.mark.parametrize("shape", [(300, 136, 1000), (129, 72, 257), (1, 8, 17)])
def test_variants_ragged_with_bias(device, shape):
    N, D, V = shape
    inp = make_inputs("tiny", N=N, D=D, V=V, seed=50 + N, ignore_frac=0.1)
    check_bias(inp, make_bias(V, 51 + V), device, "sum", grad_out=torch.tensor([0.5]), ls=0.1, zl=1e-3)


def test_variants_on_a_peaked_problem_with_skipping(device):
    inp = make_inputs("llama3.1-8b-head", N=512, D=256, V=16384, alpha=16.0, seed=23)  # tiles skipped
    r = check_bias(inp, make_bias(16384, 5, scale=0.25), device, "mean", ls=0.1, zl=1e-4)
    assert r["filtered"] > 0


def test_variants_fp32_outputs(device):
    inp = make_inputs("tiny", N=256, D=128, V=2048, seed=52)
    check_bias(inp, make_bias(2048, 53), device, "mean", out_fp32=True, ls=0.2, zl=1e-2)


def test_token_shift_through_autograd(device):
    """shift=True: e[b, i] predicts targets[b, i + 1]; the same as the oracle on explicitly shifted
    inputs, with a zero gradient at each sequence's last position."""
    B, T, D, V = 3, 40, 64, 1000
    inp = make_inputs("tiny", N=B * T, D=D, V=V, seed=54, ignore_frac=0.1)
    e = inp.E.to(device).reshape(B, T, D).requires_grad_(True)
    c = inp.C.to(device).requires_grad_(True)
    t = inp.targets.to(device).reshape(B, T)
    loss = ops.linear_cross_entropy(e, c, t, shift=True, label_smoothing=0.1)
    loss.backward()
    Es = inp.E.reshape(B, T, D)[:, :-1].reshape(-1, D)
    ts = inp.targets.reshape(B, T)[:, 1:].reshape(-1)
    f = O.forward(Es, inp.C, ts, label_smoothing=0.1)
    ob = O.backward(Es, inp.C, ts, 1.0, -100, "mean", EPS, *ops.backward_tile_shape(), label_smoothing=0.1)
    assert abs(loss.item() - float(f.loss)) <= LOSS_TOL
    g = e.grad.double().cpu().numpy()
    assert not g[:, -1].any()
    assert rel_frob(g[:, :-1].reshape(-1, D), ob.dE) <= 1e-2
    assert rel_frob(c.grad.double().cpu().numpy(), ob.dC) <= 1e-2
    nll = ops.linear_cross_entropy(e.detach(), c.detach(), t, reduction="none", shift=True)
    assert nll.shape == (B, T - 1)
    fn = O.forward(Es, inp.C, ts, reduction="none")
    assert np.abs(nll.double().cpu().numpy().reshape(-1) - fn.loss).max() <= LOSS_TOL


@pytest.mark.parametrize("ignore_index", [3, 1000])
def test_custom_ignore_index(device, ignore_index):
    """ignore_index inside [0, V) masks exactly the tokens whose target equals it (class 3 is then
    never a target), and one equal to V masks tokens whose target is V; with smoothing and z-loss,
    reduction sum."""
    N, D, V = 300, 136, 1000
    inp = make_inputs("tiny", N=N, D=D, V=V, seed=71, ignore_frac=0.0)
    t = inp.targets.clone()
    t[::7] = ignore_index
    t[1::11] = 3 if ignore_index != 3 else 4
    E, C, tt = inp.E.to(device), inp.C.to(device), t.to(device)
    g = torch.tensor([0.5], device=device)
    loss, lse, tmax, count = ops.cce_forward(E, C, tt, ignore_index, "sum", check=True, label_smoothing=0.1,
                                             z_loss=1e-3)
    dE, dC, filt = ops.cce_backward(E, C, tt, lse, tmax, count, g, EPS, ignore_index, "sum", check=True,
                                    label_smoothing=0.1, z_loss=1e-3)
    f = O.forward(inp.E, inp.C, t, ignore_index, "sum", label_smoothing=0.1, z_loss=1e-3)
    b = O.backward(inp.E, inp.C, t, 0.5, ignore_index, "sum", EPS, *ops.backward_tile_shape(), label_smoothing=0.1,
                   z_loss=1e-3)
    assert int(count.item()) == f.count == int((t != ignore_index).sum())
    assert abs(float(loss.item()) - float(f.loss)) <= LOSS_TOL * f.count
    assert rel_frob(dE.double().cpu().numpy(), b.dE) <= 1e-2
    assert rel_frob(dC.double().cpu().numpy(), b.dC) <= 1e-2
    raw = dE.cpu()[t == ignore_index]
    assert (raw.view(torch.int16) == 0).all(), "dE rows of ignored tokens must be exactly +0"


@pytest.mark.parametrize("shift", [False, True])
def test_perplexity_helper(device, shift):
    """perplexity = exp(mean NLL over non-ignored tokens) (mlx-cross-entropy README, "Computing
    related quantities"), against the oracle's per-token losses; every token ignored gives 1."""
    inp = make_inputs("tiny", N=192, D=128, V=3000, seed=61, ignore_frac=0.1)
    e = inp.E.reshape(4, 48, 128)
    t = inp.targets.reshape(4, 48)
    ppl = ops.perplexity(e.to(device), inp.C.to(device), t.to(device), shift=shift)
    tt = ops.shift_targets(t) if shift else t
    f = O.forward(inp.E, inp.C, tt.reshape(-1), -100, "none")
    want = np.exp(f.nll.sum() / f.count)
    assert abs(float(ppl) - want) <= want * LOSS_TOL
    none = torch.full_like(t, -100)
    assert float(ops.perplexity(e.to(device), inp.C.to(device), none.to(device))) == 1.0
