"""Failure detection on the GPU without a fault: a bounded wait that runs out is reported.

Forward: the kernel's producer is told (through a test-only environment switch, read at call
time) to issue no loads, so the MMA warp's wait on the first stage gives up after
CCE_WAIT_TIMEOUT_MS. Backward: the dE items of the first vocabulary chunk are told to wait for
one gradient half more than the recompute stores, so their wait on a counter raised by other
CTAs gives up; the other CTAs see the recorded error and stop too. Planning: one block of the
cooperative planning launch leaves before the first grid barrier, so the other blocks' wait there
gives up. In every case the kernel records CCE_ERR_DEVICE_TIMEOUT and exits cleanly; the test
checks the status and that the same process then computes correct results again. Run in a child
process so that the environment switches cannot leak into other tests.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import os, sys
sys.path.insert(0, os.environ["CCE_ROOT"])
import torch
from linear_cross_entropy_06_b200 import ops
from linear_cross_entropy_06_b200.inputs import make_inputs
from oracle import cce_oracle as O
inp = make_inputs("tiny", N=256, D=128, V=4096)
E, C, t = inp.E.cuda(), inp.C.cuda(), inp.targets.cuda()
os.environ["CCE_TEST_INJECT_STALL"] = "1"
try:
    ops.cce_forward(E, C, t, check=True)
    print("NO-ERROR")
except ops.CCEError as e:
    print("STATUS", e.status)
os.environ["CCE_TEST_INJECT_STALL"] = "0"
loss, *_ = ops.cce_forward(E, C, t, check=True)
ref = float(O.forward(inp.E, inp.C, inp.targets).loss)
print("RECOVERED", abs(float(loss.item()) - ref) <= 2e-3)
"""


def test_bounded_wait_timeout_is_reported_and_context_survives():
    env = dict(os.environ, CCE_ROOT=ROOT, CCE_WAIT_TIMEOUT_MS="200")
    out = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert "STATUS 5" in out.stdout, out.stdout  # CCE_ERR_DEVICE_TIMEOUT
    assert "RECOVERED True" in out.stdout, out.stdout


CHILD_BWD = r"""
import os, sys
sys.path.insert(0, os.environ["CCE_ROOT"])
import numpy as np
import torch
from linear_cross_entropy_06_b200 import ops
from linear_cross_entropy_06_b200.inputs import make_inputs
from oracle import cce_oracle as O
inp = make_inputs("tiny", N=512, D=128, V=8192)
E, C, t = inp.E.cuda(), inp.C.cuda(), inp.targets.cuda()
g = torch.ones(1, device="cuda")
loss, lse, tmax, count = ops.cce_forward(E, C, t, check=True)
os.environ["CCE_TEST_INJECT_STALL"] = "2"
try:
    ops.cce_backward(E, C, t, lse, tmax, count, g, 0.0, check=True)
    print("NO-ERROR")
except ops.CCEError as e:
    print("STATUS", e.status)
os.environ["CCE_TEST_INJECT_STALL"] = "0"
dE, dC, _ = ops.cce_backward(E, C, t, lse, tmax, count, g, 0.0, check=True)
ref = O.backward(inp.E, inp.C, inp.targets, 1.0, -100, "mean", 0.0, 128, 128)
rel = np.linalg.norm(dE.double().cpu().numpy() - ref.dE) / np.linalg.norm(ref.dE)
print("RECOVERED", rel <= 1e-2)
"""


def test_backward_dependency_wait_timeout_is_reported_and_context_survives():
    env = dict(os.environ, CCE_ROOT=ROOT, CCE_WAIT_TIMEOUT_MS="200")
    out = subprocess.run([sys.executable, "-c", CHILD_BWD], env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert "STATUS 5" in out.stdout, out.stdout  # CCE_ERR_DEVICE_TIMEOUT
    assert "RECOVERED True" in out.stdout, out.stdout


CHILD_PLAN = CHILD_BWD.replace('os.environ["CCE_TEST_INJECT_STALL"] = "2"', 'os.environ["CCE_TEST_INJECT_STALL"] = "3"')


def test_planning_barrier_timeout_is_reported_and_context_survives():
    """The planning launch's first grid barrier: one block leaves before it (test hook), so the
    others' bounded wait runs out and records CCE_ERR_DEVICE_TIMEOUT; the tensor-core kernel then
    hands out no work from the unfinished plan, and the next backward on the same context is
    correct."""
    assert CHILD_PLAN != CHILD_BWD
    env = dict(os.environ, CCE_ROOT=ROOT, CCE_WAIT_TIMEOUT_MS="200")
    out = subprocess.run([sys.executable, "-c", CHILD_PLAN], env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert "STATUS 5" in out.stdout, out.stdout  # CCE_ERR_DEVICE_TIMEOUT
    assert "RECOVERED True" in out.stdout, out.stdout
