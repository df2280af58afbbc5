"""The forward and backward captured into a CUDA graph and replayed.

Every operation the library enqueues is stream-ordered (kernel launches, including the cooperative
planning launch and the launches that may overlap their predecessor, and memsets), and it neither
allocates device memory nor waits for the GPU inside a call, so a training loop can capture the
loss once and replay it. The replays must give the eager results: the loss, dC and the skipped
count exactly, dE to the rounding of its fp32 reduce-adds across vocabulary chunks, whose order
is not fixed.
"""
import pytest
import torch

from linear_cross_entropy_06_b200 import ops
from linear_cross_entropy_06_b200.inputs import make_inputs

from test_gpu_parity import EPS

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("reduction", ["mean", "none"])
def test_graph_replay_matches_eager(device, reduction):
    N, D, V = 640, 256, 20000  # several vocabulary tiles and row blocks, a ragged last tile
    inp = make_inputs("llama3.1-8b-head", N=N, D=D, V=V, alpha=20.0, seed=97)  # most units skipped
    E, C, t = inp.E.to(device), inp.C.to(device), inp.targets.to(device)
    g = torch.linspace(-1.0, 1.0, N, device=device) if reduction == "none" else torch.ones(1, device=device)

    def step():
        loss, lse, tmax, count = ops.cce_forward(E, C, t, -100, reduction)
        dE, dC, filt = ops.cce_backward(E, C, t, lse, tmax, count, g, EPS, -100, reduction)
        return loss, dE, dC, filt

    ref = [x.clone() for x in step()]
    torch.cuda.synchronize()
    side = torch.cuda.Stream()  # warm-up on a side stream before capture, as torch recommends
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(2):
            step()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        out = step()
    for _ in range(3):
        graph.replay()
        torch.cuda.synchronize()
        loss, dE, dC, filt = out
        assert torch.equal(loss, ref[0])
        assert torch.equal(dC, ref[2])
        assert int(filt.item()) == int(ref[3].item()) > 0
        rel = (dE.float() - ref[1].float()).norm() / ref[1].float().norm()
        assert rel <= 1e-3, float(rel)
