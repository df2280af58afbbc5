"""GPU tests of cce_forward_noalloc, the forward for callers that cannot allocate device memory.

Such callers (an embedding host that hands the library only fixed buffers for inputs and outputs,
or a runtime whose allocator must not be re-entered from a loss callback) get a forward whose
scratch lives in a device array the library holds itself. These tests call it through the C ABI
and compare it with cce_forward, which takes a caller-owned workspace, and with the fp64 oracle,
on two calls in a row: the array keeps the previous call's contents, so the second call also
checks that nothing stale leaks into a result. This file sorts last so that a run that stops at
the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from linear_cross_entropy_06_b200 import ops
from linear_cross_entropy_06_b200.inputs import make_inputs
from oracle import cce_oracle as O

pytestmark = pytest.mark.gpu

LOSS_TOL = 2e-3  # the loss / LSE tolerance of the other parity tests


def _noalloc(E, C, t, reduction, bias=None, label_smoothing=0.0, z_loss=0.0, ignore_index=-100):
    lib = ops.load_library()
    N, D = E.shape
    V = C.shape[0]
    p = ops.Problem(N, D, V, ignore_index, ops.REDUCTION_CODES[reduction], 0, label_smoothing, z_loss)
    loss = torch.full((N if reduction == "none" else 1,), float("nan"), device=E.device)
    lse = torch.full((N,), float("nan"), device=E.device)
    tmax = torch.full((max(lib.cce_tile_max_len(ctypes.byref(p)), 1),), float("nan"), device=E.device)
    count = torch.full((1,), -1, dtype=torch.int64, device=E.device)
    st = lib.cce_forward_noalloc(ctypes.byref(p), E.data_ptr(), C.data_ptr(),
                                 None if bias is None else bias.data_ptr(), t.data_ptr(), loss.data_ptr(),
                                 lse.data_ptr(), tmax.data_ptr(), count.data_ptr(),
                                 torch.cuda.current_stream(E.device).cuda_stream)
    return st, loss, lse, tmax, count


VARIANTS = {
    "plain": dict(bias=False, label_smoothing=0.0, z_loss=0.0),
    # the label-smoothing path keeps the column sums of C and each row's sum of logits in the array
    "bias+smoothing+z-loss": dict(bias=True, label_smoothing=0.1, z_loss=1e-4),
}


@pytest.mark.parametrize("variant", list(VARIANTS))
@pytest.mark.parametrize("reduction", ["mean", "none"])
def test_noalloc_forward_matches_workspace_forward_on_two_calls(device, reduction, variant):
    kw = VARIANTS[variant]
    cases = [make_inputs("tiny", N=1024, D=256, V=8192, seed=31),
             make_inputs("llama3.1-8b-head", N=640, D=512, V=20000, seed=32)]
    for inp in cases:  # two calls in a row, different shapes
        V = inp.C.shape[0]
        bias = None
        if kw["bias"]:
            bias = torch.from_numpy(np.random.default_rng(V).standard_normal(V).astype(np.float32)).to(torch.bfloat16)
        E, C, t = inp.E.to(device), inp.C.to(device), inp.targets.to(device)
        b = None if bias is None else bias.to(device)
        ls, zl = kw["label_smoothing"], kw["z_loss"]
        ref_loss, ref_lse, ref_tmax, ref_count = ops.cce_forward(E, C, t, -100, reduction, check=True, bias=b,
                                                                 label_smoothing=ls, z_loss=zl)
        st, loss, lse, tmax, count = _noalloc(E, C, t, reduction, b, ls, zl)
        assert st == 0, ops.load_library().cce_last_error_message()
        torch.cuda.synchronize()
        assert int(count.item()) == int(ref_count.item())
        assert torch.isfinite(loss).all() and torch.isfinite(lse).all()
        assert (loss.double() - ref_loss.double()).abs().max().item() <= LOSS_TOL
        assert (lse.double() - ref_lse.double()).abs().max().item() <= LOSS_TOL
        n = ref_tmax.numel()
        assert (tmax[:n].double() - ref_tmax.double()).abs().max().item() <= LOSS_TOL
        # and against the fp64 oracle on the same inputs
        f = O.forward(inp.E, inp.C, inp.targets, -100, reduction, bias=bias, label_smoothing=ls, z_loss=zl)
        assert int(count.item()) == f.count
        assert np.abs(loss.double().cpu().numpy().reshape(np.shape(f.loss)) - f.loss).max() <= LOSS_TOL
        assert np.abs(lse.double().cpu().numpy() - f.lse).max() <= LOSS_TOL


def test_noalloc_rejects_problems_beyond_its_scratch(device):
    lib = ops.load_library()
    N, D, V = 65536, 128, 128256  # tile sums alone need ceil(V/64) * N * 4 = 525 MB
    p = ops.Problem(N, D, V, -100, 1, 0)
    st = lib.cce_forward_noalloc(ctypes.byref(p), 256, 256, None, 256, 256, 256, 256, 256, None)
    assert st == 2  # CCE_ERR_UNSUPPORTED, before anything is enqueued
    assert b"scratch" in lib.cce_last_error_message()
    torch.cuda.synchronize()


@pytest.mark.parametrize("reduction", ["mean", "none"])
def test_noalloc_device_error_gives_nan_loss_then_recovers(device, reduction):
    """A target outside [0, V) is found on the device, after the call has returned: the loss comes
    back NaN. The next call, on valid targets, clears the array's error word and is correct."""
    inp = make_inputs("tiny", N=256, D=128, V=4096, seed=33)
    E, C = inp.E.to(device), inp.C.to(device)
    bad = inp.targets.clone()
    bad[17] = 4096
    st, loss, *_ = _noalloc(E, C, bad.to(device), reduction)
    assert st == 0
    torch.cuda.synchronize()
    assert torch.isnan(loss).all()
    t = inp.targets.to(device)
    st, loss, lse, _, count = _noalloc(E, C, t, reduction)
    assert st == 0
    torch.cuda.synchronize()
    f = O.forward(inp.E, inp.C, inp.targets, -100, reduction)
    assert np.abs(loss.double().cpu().numpy().reshape(np.shape(f.loss)) - f.loss).max() <= LOSS_TOL
    assert int(count.item()) == f.count


@settings(max_examples=25, derandomize=True, deadline=None,
          suppress_health_check=[HealthCheck.function_scoped_fixture, HealthCheck.too_slow])
@given(N=st.integers(1, 700), D8=st.integers(1, 65), V=st.integers(1, 4000),
       reduction=st.sampled_from(["mean", "sum", "none"]), with_bias=st.booleans(),
       ls=st.sampled_from([0.0, 0.1]), zl=st.sampled_from([0.0, 1e-4]), seed=st.integers(0, 10_000))
def test_noalloc_random_problems_match_the_oracle(device, N, D8, V, reduction, with_bias, ls, zl, seed):
    """Random shapes and options, one call after another on the shared array: the loss, LSE and
    count of each against the fp64 oracle."""
    D = 8 * D8
    inp = make_inputs("tiny", N=N, D=D, V=V, seed=seed, ignore_frac=0.1)
    bias = None
    if with_bias:
        bias = torch.from_numpy(np.random.default_rng(seed + 2).standard_normal(V).astype(np.float32) * 0.5)
        bias = bias.to(torch.bfloat16)
    E, C, t = inp.E.to(device), inp.C.to(device), inp.targets.to(device)
    st_, loss, lse, _, count = _noalloc(E, C, t, reduction, None if bias is None else bias.to(device), ls, zl)
    assert st_ == 0, ops.load_library().cce_last_error_message()
    torch.cuda.synchronize()
    f = O.forward(inp.E, inp.C, inp.targets, -100, reduction, bias=bias, label_smoothing=ls, z_loss=zl)
    assert int(count.item()) == f.count
    tol = LOSS_TOL * (max(f.count, 1) if reduction == "sum" else 1)
    assert np.abs(loss.double().cpu().numpy().reshape(np.shape(f.loss)) - f.loss).max() <= tol
    assert np.abs(lse.double().cpu().numpy() - f.lse).max() <= LOSS_TOL
