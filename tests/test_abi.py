"""Host-side checks of libcce.so that need no GPU: exports, sizes, argument validation."""
import ctypes
import os
import re

import pytest

from linear_cross_entropy_06_b200 import ops
from linear_cross_entropy_06_b200.build import LIB, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return ops.load_library()


def declared_symbols():
    with open(os.path.join(ROOT, "include", "cce.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"CCE_API\s+[\w\s\*]*?\b(cce_\w+)\s*\(", text)))


def test_header_declares_the_documented_calls():
    names = declared_symbols()
    for n in ("cce_forward", "cce_backward", "cce_forward_workspace_size", "cce_backward_workspace_size",
              "cce_check_device_error", "cce_status_string", "cce_tile_max_len"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert name in ops.SIGNATURES, f"binding lacks {name}"
    assert set(ops.SIGNATURES) == set(declared_symbols())


def test_library_has_no_link_time_cuda_dependency():
    """libcce.so links the CUDA runtime statically and looks the driver up at run time, so it loads
    on a machine without a driver: its dynamic section names neither libcuda nor libcudart."""
    import shutil
    import subprocess

    build()
    ctypes.CDLL(LIB)
    readelf = shutil.which("readelf")
    if readelf is None:
        pytest.skip("readelf not available")
    out = subprocess.run([readelf, "-d", LIB], check=True, capture_output=True, text=True).stdout
    needed = re.findall(r"\(NEEDED\)\s+Shared library: \[([^\]]+)\]", out)
    assert needed, out
    assert not [n for n in needed if n.startswith(("libcuda.", "libcudart.", "libtorch", "libc10"))], needed


def _p(N=256, D=128, V=4096, red=1, ignore=-100, reserved=0):
    return ops.Problem(N, D, V, ignore, red, reserved)


def test_sizes(lib):
    p = _p(N=300, D=136, V=1000)
    T = -(-1000 // 64)  # saved maxima per 64 vocabulary columns
    assert lib.cce_tile_max_len(ctypes.byref(p)) == T * 300
    fw = lib.cce_forward_workspace_size(ctypes.byref(p))
    # header, tile sums [T, N], target logits, row losses, and for label smoothing the column
    # sums of C [D + 1] and the row sums of the logits [N]; 256-byte alignment of each
    assert 0 < fw < 256 + 4 * (T * 300 + 900 + 137) + 6 * 256
    bw32 = lib.cce_backward_workspace_size(ctypes.byref(p), 1)
    bw16 = lib.cce_backward_workspace_size(ctypes.byref(p), 0)
    assert bw16 - bw32 >= 4 * 300 * 136  # the fp32 dE accumulator (dC is summed on chip)
    # nothing of size N*V: the workspaces of a Llama-3 head are far below N*V*2 bytes
    big = _p(N=32768, D=4096, V=128256, red=0)
    assert lib.cce_forward_workspace_size(ctypes.byref(big)) < 32768 * 128256 * 2 // 8
    assert lib.cce_tile_max_len(ctypes.byref(big)) * 4 < 32768 * 128256 * 2 // 8
    r, c = ops.backward_tile_shape()
    assert (r, c) == (128, 64)


@pytest.mark.parametrize("bad", [dict(D=7), dict(D=0), dict(V=0), dict(N=-1), dict(red=3), dict(reserved=1)])
def test_bad_problems_are_rejected_before_any_cuda_call(lib, bad):
    p = _p(**bad)
    assert lib.cce_tile_max_len(ctypes.byref(p)) == -1
    assert lib.cce_forward_workspace_size(ctypes.byref(p)) == 0
    st = lib.cce_forward(ctypes.byref(p), 16, 16, None, 16, 16, 16, 16, 16, 16, 1 << 20, None)
    assert st == 1  # CCE_ERR_INVALID_ARG
    assert lib.cce_last_error_message()


def test_null_and_misaligned_pointers_are_rejected(lib):
    p = _p()
    assert lib.cce_forward(ctypes.byref(p), None, 16, None, 16, 16, 16, 16, 16, 16, 1 << 20, None) == 1
    assert lib.cce_forward(ctypes.byref(p), 18, 16, None, 16, 16, 16, 16, 16, 16, 1 << 20, None) == 1
    assert b"aligned" in lib.cce_last_error_message()
    # a bias that is not 16-byte aligned
    assert lib.cce_forward(ctypes.byref(p), 16, 16, 24, 16, 16, 16, 16, 16, 16, 1 << 20, None) == 1
    assert b"aligned" in lib.cce_last_error_message()
    assert lib.cce_backward(ctypes.byref(p), 16, 16, None, 16, 16, 16, 16, 16, float("nan"), 16, 16, None, 0, 16,
                            16, 1 << 40, None) == 1
    assert lib.cce_backward(ctypes.byref(p), 16, 16, None, 16, 16, 16, 16, 16, 0.5, 16, 16, 40, 0, 16, 16,
                            1 << 40, None) == 1  # misaligned dbias


@pytest.mark.parametrize("field,value", [("label_smoothing", -0.1), ("label_smoothing", 1.5),
                                         ("label_smoothing", float("nan")), ("z_loss", -1.0), ("z_loss", float("inf"))])
def test_bad_loss_variants_are_rejected(lib, field, value):
    p = _p()
    setattr(p, field, value)
    assert lib.cce_tile_max_len(ctypes.byref(p)) == -1
    assert lib.cce_forward(ctypes.byref(p), 16, 16, None, 16, 16, 16, 16, 16, 16, 1 << 20, None) == 1
    assert field.encode() in lib.cce_last_error_message()


def test_small_workspace_is_rejected(lib):
    p = _p()
    need = lib.cce_forward_workspace_size(ctypes.byref(p))
    assert lib.cce_forward(ctypes.byref(p), 16, 16, None, 16, 16, 16, 16, 16, 16, need - 1, None) == 3


def test_status_strings(lib):
    for code in range(7):
        assert lib.cce_status_string(code)
    assert lib.cce_version() >= 300


def test_plain_c_caller_compiles_links_and_runs():
    """include/cce.h is valid C99 and libcce.so serves a C caller that has no Python or torch."""
    import shutil
    import subprocess
    import tempfile

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(LIB)
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "abi_example")
        subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(root, "include"),
                        os.path.join(root, "tests", "c", "abi_example.c"), "-o", exe, "-L", libdir, "-lcce",
                        "-Wl,-rpath," + libdir], check=True, capture_output=True, text=True)
        out = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=60).stdout
    vals = dict(line.split(" ", 1) for line in out.strip().splitlines())
    assert int(vals["version"]) >= 300
    assert vals["tile"] == "128 64"
    assert int(vals["tile_max_len"]) == 4096 * ((128256 + 63) // 64)
    assert int(vals["fwd_ws"]) > 0 and int(vals["bwd_ws"]) > 0
    assert vals["bad_status"].startswith("1 ")  # CCE_ERR_INVALID_ARG
    assert "multiple of 8" in vals["message"]


def test_backward_scratch_grows_with_tokens_not_vocabulary(lib):
    """The gradient-tile scratch is max(128 MiB, 4 MiB per 128 rows): doubling V adds only the
    tile plan (tens of bytes per 128 x 128 tile), while going from 4096 to 32768 tokens adds the
    scratch of 224 more row blocks besides the fp32 dE accumulator."""
    def bw(N, V, D=4096, out_fp32=1):
        p = _p(N=N, D=D, V=V, red=0)
        return lib.cce_backward_workspace_size(ctypes.byref(p), out_fp32)

    small, wide = bw(4096, 64128), bw(4096, 128256)
    tiles_added = (4096 // 128) * (128256 // 128 - 64128 // 128)
    assert 0 < wide - small <= 48 * tiles_added + (1 << 20)
    big = bw(32768, 128256)
    assert big - wide >= 224 * (4 << 20)
    # nothing of size N*V: at the long-batch shape far below the bf16 logits (8.4 GB)
    assert big < 32768 * 128256 * 2 // 4


def _operands(N=256, D=128, V=1000, e_dtype=None, t_dtype=None):
    import torch
    E = torch.zeros(N, D, dtype=e_dtype or torch.bfloat16)
    C = torch.zeros(V, D, dtype=torch.bfloat16)
    t = torch.zeros(N, dtype=t_dtype or torch.int64)
    return E, C, t


@pytest.mark.parametrize("case,needle", [
    (dict(e_dtype="float32"), "bfloat16"),
    (dict(e_dtype="float16"), "bfloat16"),
    (dict(t_dtype="int32"), "int64"),
])
def test_binding_rejects_wrong_dtypes_before_the_library(lib, case, needle):
    """The kernels read bf16 operands and int64 targets through raw pointers: any other dtype would
    be read as the wrong type (int32 targets: past the end of their buffer), so the binding refuses."""
    import torch
    kw = {k: getattr(torch, v) for k, v in case.items()}
    E, C, t = _operands(**kw)
    with pytest.raises(ops.CCEError, match=needle) as ei:
        ops.cce_forward(E, C, t)
    assert ei.value.status == 1


def test_binding_rejects_mismatched_shapes(lib):
    import torch
    E, C, t = _operands()
    with pytest.raises(ops.CCEError, match="must be \\[V, 128\\]"):
        ops.cce_forward(E, C[:, :64].contiguous(), t)
    with pytest.raises(ops.CCEError, match="N=256 entries"):
        ops.cce_forward(E, C, t[:255])
    with pytest.raises(ops.CCEError, match="2-D"):
        ops.cce_forward(E.reshape(2, 128, 128), C, t)


def test_binding_checks_the_saved_forward_state_in_the_backward(lib):
    """lse, tile_max and count are read in full by the backward's kernels: a short or mistyped buffer
    is refused on the host (here on CPU tensors, which would be refused next anyway)."""
    import torch
    E, C, t = _operands()
    p = _p(N=256, D=128, V=1000)
    tm_len = lib.cce_tile_max_len(ctypes.byref(p))
    lse = torch.zeros(256)
    tmax = torch.zeros(tm_len)
    count = torch.zeros(1, dtype=torch.int64)
    g = torch.ones(())
    with pytest.raises(ops.CCEError, match="tile_max"):
        ops.cce_backward(E, C, t, lse, tmax[:-1], count, g)
    with pytest.raises(ops.CCEError, match="lse"):
        ops.cce_backward(E, C, t, lse.double(), tmax, count, g)
    with pytest.raises(ops.CCEError, match="count"):
        ops.cce_backward(E, C, t, lse, tmax, count.int(), g)
    with pytest.raises(ops.CCEError, match="grad_out must have 256"):
        ops.cce_backward(E, C, t, lse, tmax, count, g, reduction="none")
    # well-formed CPU tensors reach the device check: there is no CPU path
    with pytest.raises(ops.CCEError, match="no CPU path"):
        ops.cce_backward(E, C, t, lse, tmax, count, g)
