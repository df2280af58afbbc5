"""GPU tests of cce_forward_noalloc, the forward for callers that cannot allocate device memory.

Such callers (code under CUDA graph capture, or an embedding that only hands the library fixed
buffers) get a forward whose scratch lives in a device array the library holds itself. These
tests call it through the C ABI and compare it with cce_forward, which takes a caller-owned
workspace, on two calls in a row: the array keeps the previous call's contents, so the second
call also checks that nothing stale leaks into a result. This file sorts last so that a run that
stops at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from linear_cross_entropy_06_b200 import ops
from linear_cross_entropy_06_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

LOSS_TOL = 2e-3  # the loss / LSE tolerance of the other parity tests


def _noalloc(E, C, t, reduction, ignore_index=-100):
    lib = ops.load_library()
    N, D = E.shape
    V = C.shape[0]
    p = ops.Problem(N, D, V, ignore_index, ops.REDUCTION_CODES[reduction], 0)
    loss = torch.full((N if reduction == "none" else 1,), float("nan"), device=E.device)
    lse = torch.full((N,), float("nan"), device=E.device)
    tmax = torch.full((max(lib.cce_tile_max_len(ctypes.byref(p)), 1),), float("nan"), device=E.device)
    count = torch.full((1,), -1, dtype=torch.int64, device=E.device)
    st = lib.cce_forward_noalloc(ctypes.byref(p), E.data_ptr(), C.data_ptr(), None, t.data_ptr(), loss.data_ptr(),
                                 lse.data_ptr(), tmax.data_ptr(), count.data_ptr(),
                                 torch.cuda.current_stream(E.device).cuda_stream)
    return st, loss, lse, tmax, count


@pytest.mark.parametrize("reduction", ["mean", "none"])
def test_noalloc_forward_matches_workspace_forward_on_two_calls(device, reduction):
    cases = [make_inputs("tiny", N=1024, D=256, V=8192, seed=31),
             make_inputs("llama3.1-8b-head", N=640, D=512, V=20000, seed=32)]
    for inp in cases:  # two calls in a row, different shapes
        E, C, t = inp.E.to(device), inp.C.to(device), inp.targets.to(device)
        ref_loss, ref_lse, ref_tmax, ref_count = ops.cce_forward(E, C, t, -100, reduction, check=True)
        st, loss, lse, tmax, count = _noalloc(E, C, t, reduction)
        assert st == 0, ops.load_library().cce_last_error_message()
        torch.cuda.synchronize()
        assert int(count.item()) == int(ref_count.item())
        assert torch.isfinite(loss).all() and torch.isfinite(lse).all()
        assert (loss.double() - ref_loss.double()).abs().max().item() <= LOSS_TOL
        assert (lse.double() - ref_lse.double()).abs().max().item() <= LOSS_TOL
        n = ref_tmax.numel()
        assert (tmax[:n].double() - ref_tmax.double()).abs().max().item() <= LOSS_TOL


def test_noalloc_rejects_problems_beyond_its_scratch(device):
    lib = ops.load_library()
    N, D, V = 65536, 128, 128256  # tile sums alone need ceil(V/128) * N * 4 = 263 MB
    p = ops.Problem(N, D, V, -100, 1, 0)
    st = lib.cce_forward_noalloc(ctypes.byref(p), 256, 256, None, 256, 256, 256, 256, 256, None)
    assert st == 2  # CCE_ERR_UNSUPPORTED, before anything is enqueued
    assert b"scratch" in lib.cce_last_error_message()
    torch.cuda.synchronize()


def test_noalloc_forward_replays_in_a_cuda_graph(device):
    """The caller this entry point serves: the forward captured in a CUDA graph (no allocation
    during capture), replayed on new inputs copied into the captured buffers."""
    N, D, V = 512, 256, 8192
    first = make_inputs("tiny", N=N, D=D, V=V, seed=61)
    second = make_inputs("llama3.1-8b-head", N=N, D=D, V=V, seed=62)
    E = first.E.to(device).clone()
    C = first.C.to(device).clone()
    t = first.targets.to(device).clone()
    # warm-up call outside capture: resolves the scratch address and the driver entry point
    st, *_ = _noalloc(E, C, t, "mean")
    assert st == 0
    torch.cuda.synchronize()
    lib = ops.load_library()
    p = ops.Problem(N, D, V, -100, ops.REDUCTION_CODES["mean"], 0)
    loss = torch.empty(1, device=device)
    lse = torch.empty(N, device=device)
    tmax = torch.empty(lib.cce_tile_max_len(ctypes.byref(p)), device=device)
    count = torch.empty(1, dtype=torch.int64, device=device)
    graph = torch.cuda.CUDAGraph()
    stream = torch.cuda.Stream(device)
    stream.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            st = lib.cce_forward_noalloc(ctypes.byref(p), E.data_ptr(), C.data_ptr(), None, t.data_ptr(),
                                         loss.data_ptr(), lse.data_ptr(), tmax.data_ptr(), count.data_ptr(),
                                         stream.cuda_stream)
    assert st == 0
    for inp in (second, first):
        E.copy_(inp.E.to(device))
        C.copy_(inp.C.to(device))
        t.copy_(inp.targets.to(device))
        graph.replay()
        torch.cuda.synchronize()
        ref_loss, ref_lse, _, ref_count = ops.cce_forward(inp.E.to(device), inp.C.to(device),
                                                          inp.targets.to(device), check=True)
        assert abs(float(loss) - float(ref_loss)) <= 1e-5
        assert (lse - ref_lse).abs().max().item() <= 1e-5
        assert int(count) == int(ref_count)
