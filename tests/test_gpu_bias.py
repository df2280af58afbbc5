"""GPU parity of the classifier bias (mlx-cross-entropy README, "API" table: bias [V]) against
the fp64 oracle: logits E C^T + bias in the forward, and dbias = column sums of G in the backward.

Same tolerances as the other parity tests: loss and LSE within 2e-3 absolute; dE, dC and dbias
within a relative Frobenius error of 1e-2 of the oracle that applies the same tile rule, with the
row-wise elementwise bound; ignored rows of dE exactly +0; skipped-tile counts equal.
"""
import ctypes

import numpy as np
import pytest
import torch

from linear_cross_entropy_06_b200 import ops
from linear_cross_entropy_06_b200.inputs import make_inputs
from oracle import cce_oracle as O

from test_gpu_parity import EPS, LOSS_TOL, assert_close_elementwise, assert_count, fp32_floor, frob_ok, rel_frob

pytestmark = pytest.mark.gpu


def make_bias(V, seed, scale=2.0):
    """A bf16 bias [V] (standard normal times `scale`), seeded."""
    b = np.random.default_rng(seed).standard_normal(V).astype(np.float32) * scale
    return torch.from_numpy(b).to(torch.bfloat16)


def run_with_bias(inp, bias, device, filter_eps, reduction, out_fp32=False, grad_out=None, dbias=True, ls=0.0,
                  zl=0.0):
    E, C, t = inp.E.to(device), inp.C.to(device), inp.targets.to(device)
    b = None if bias is None else bias.to(device)
    g = (inp.grad_out if grad_out is None else grad_out).to(device)
    if reduction != "none":
        g = g[:1]
    loss, lse, tmax, count = ops.cce_forward(E, C, t, -100, reduction, check=True, bias=b, label_smoothing=ls,
                                             z_loss=zl)
    dE, dC, filt, db = ops.cce_backward(E, C, t, lse, tmax, count, g, filter_eps, -100, reduction, out_fp32,
                                        check=True, bias=b, dbias=dbias, label_smoothing=ls, z_loss=zl)
    torch.cuda.synchronize()
    return dict(loss=loss.double().cpu().numpy(), lse=lse.double().cpu().numpy(), count=int(count.item()),
                dE=dE.double().cpu().numpy(), dC=dC.double().cpu().numpy(), dbias=db.double().cpu().numpy(),
                filtered=int(filt.item()), dE_raw=dE.cpu())


def check_bias(inp, bias, device, reduction, grad_out=None, out_fp32=False, ls=0.0, zl=0.0):
    tm, tn = ops.backward_tile_shape()
    g = inp.grad_out if grad_out is None else grad_out
    g_or = g.numpy() if reduction == "none" else float(g.reshape(-1)[0])
    ob = None if bias is None else bias
    f = O.forward(inp.E, inp.C, inp.targets, -100, reduction, bias=ob, label_smoothing=ls, z_loss=zl)
    sc = O.row_scale(inp.targets, -100, reduction, g_or, f.count) * (1.0 + 2.0 * zl * np.abs(f.lse).max())
    floors = {"dE": fp32_floor(f.lse, sc, inp.C), "dC": fp32_floor(f.lse, sc, inp.E),
              "dbias": fp32_floor(f.lse, sc, 1.0)}
    for eps in (0.0, EPS):
        b = O.backward(inp.E, inp.C, inp.targets, g_or, -100, reduction, eps, tm, tn,
                       bias=np.zeros(inp.C.shape[0]) if bias is None else ob, label_smoothing=ls, z_loss=zl)
        r = run_with_bias(inp, bias, device, eps, reduction, out_fp32, grad_out, ls=ls, zl=zl)
        if reduction == "sum":
            assert abs(r["loss"][0] - float(f.loss)) <= LOSS_TOL * max(f.count, 1)
        else:
            assert np.abs(r["loss"].reshape(np.asarray(f.loss).shape) - f.loss).max() <= LOSS_TOL
        assert np.abs(r["lse"] - f.lse).max() <= LOSS_TOL
        for name, got, want in (("dE", r["dE"], b.dE), ("dC", r["dC"], b.dC), ("dbias", r["dbias"], b.dbias)):
            assert frob_ok(got, want, 1e-2, floors[name]), f"eps={eps} {name} rel-Frobenius {rel_frob(got, want):.3e}"
            assert_close_elementwise(got.reshape(-1, got.shape[-1]) if got.ndim == 2 else got[None, :],
                                     want.reshape(-1, want.shape[-1]) if want.ndim == 2 else want[None, :],
                                     f"eps={eps} {name}", floors[name])
        ign = (inp.targets == -100)
        if ign.any():
            raw = r["dE_raw"][ign]
            bits = raw.view(torch.int16) if raw.dtype == torch.bfloat16 else raw.view(torch.int32)
            assert (bits == 0).all()
        assert_count(r["filtered"], b.filtered, b.borderline)
    return r


@pytest.mark.parametrize("reduction", ["mean", "sum", "none"])
def test_bias_tiny(device, reduction):
    inp = make_inputs("tiny")
    g = torch.from_numpy(np.random.default_rng(3).standard_normal(inp.E.shape[0]).astype(np.float32))
    check_bias(inp, make_bias(inp.C.shape[0], 1), device, reduction,
               grad_out=g if reduction == "none" else torch.tensor([1.0]))


@pytest.mark.parametrize("shape", [(300, 136, 1000), (129, 72, 257), (5, 64, 130), (1, 8, 17)])
def test_bias_ragged_shapes(device, shape):
    N, D, V = shape
    inp = make_inputs("tiny", N=N, D=D, V=V, seed=11 + N + V, ignore_frac=0.1)
    check_bias(inp, make_bias(V, N + D), device, "mean")


def test_bias_on_a_peaked_problem_with_skipping(device):
    inp = make_inputs("llama3.1-8b-head", N=512, D=256, V=16384, alpha=16.0, seed=23)  # 235 of 512 tiles skipped
    r = check_bias(inp, make_bias(16384, 5, scale=0.25), device, "mean")  # a wide bias would keep every tile
    assert r["filtered"] > 0


def test_bias_fp32_outputs(device):
    inp = make_inputs("tiny", N=256, D=128, V=2048, seed=41)
    check_bias(inp, make_bias(2048, 6), device, "mean", out_fp32=True)


def test_dbias_without_bias_is_the_gradient_of_a_zero_bias(device):
    inp = make_inputs("tiny", N=200, D=96, V=1500, seed=42)
    check_bias(inp, None, device, "mean")


def test_bias_through_autograd(device):
    inp = make_inputs("tiny", N=192, D=128, V=3000, seed=43, ignore_frac=0.1)
    bias = make_bias(3000, 7)
    e = inp.E.to(device).reshape(2, 96, 128).requires_grad_(True)
    c = inp.C.to(device).requires_grad_(True)
    b = bias.to(device).requires_grad_(True)
    t = inp.targets.to(device).reshape(2, 96)
    loss = ops.linear_cross_entropy(e, c, t, bias=b)
    loss.backward()
    f = O.forward(inp.E, inp.C, inp.targets, bias=bias)
    ob = O.backward(inp.E, inp.C, inp.targets, 1.0, -100, "mean", EPS, *ops.backward_tile_shape(), bias=bias)
    assert abs(loss.item() - float(f.loss)) <= LOSS_TOL
    assert rel_frob(b.grad.double().cpu().numpy(), ob.dbias) <= 1e-2
    assert rel_frob(c.grad.double().cpu().numpy(), ob.dC) <= 1e-2
    assert rel_frob(e.grad.double().cpu().numpy().reshape(192, 128), ob.dE) <= 1e-2


def test_noalloc_forward_with_bias(device):
    inp = make_inputs("tiny", N=512, D=256, V=8192, seed=44)
    E, C, t = inp.E.to(device), inp.C.to(device), inp.targets.to(device)
    b = make_bias(8192, 8).to(device)
    ref = ops.cce_forward(E, C, t, -100, "mean", check=True, bias=b)
    lib = ops.load_library()
    p = ops.Problem(512, 256, 8192, -100, ops.REDUCTION_CODES["mean"], 0)
    loss = torch.full((1,), float("nan"), device=device)
    lse = torch.full((512,), float("nan"), device=device)
    tmax = torch.empty(lib.cce_tile_max_len(ctypes.byref(p)), device=device)
    count = torch.empty(1, dtype=torch.int64, device=device)
    st = lib.cce_forward_noalloc(ctypes.byref(p), E.data_ptr(), C.data_ptr(), b.data_ptr(), t.data_ptr(),
                                 loss.data_ptr(), lse.data_ptr(), tmax.data_ptr(), count.data_ptr(),
                                 torch.cuda.current_stream(device).cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    assert abs(float(loss) - float(ref[0])) <= 1e-5
    assert (lse - ref[1]).abs().max().item() <= 1e-5
