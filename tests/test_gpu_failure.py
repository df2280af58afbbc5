"""Failure detection on the GPU without a fault: a bounded wait that runs out is reported.

The forward kernel's producer is told (through a test-only environment switch, read at call
time) to issue no loads, so the MMA warp's wait on the first stage gives up after
CCE_WAIT_TIMEOUT_MS. The kernel records CCE_ERR_DEVICE_TIMEOUT and exits cleanly; the test
checks the status and that the same process then computes a correct loss again. Run in a child
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
