"""Thin ctypes binding of libcce.so and the autograd wrapper ``linear_cross_entropy``.

Argument marshalling only: every step of the forward and the backward runs in the
library's CUDA kernels. torch provides device memory and the current stream.
The library is loaded on first use; a missing library or a machine without a
CUDA device raises ``CCEError`` (there is no fallback of any kind).

API shape follows the mlx-cross-entropy README ("API" table and "Usage"):
``linear_cross_entropy(e, c, targets, bias=None, reduction="mean", ignore_index=-100)`` with
``[..., D]`` hidden states flattened to ``[N, D]`` and, for ``reduction="none"``,
the per-token loss returned in the targets' shape.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcce.so")

REDUCTION_CODES = {"none": 0, "mean": 1, "sum": 2}
STATUS_NAMES = {
    0: "CCE_OK",
    1: "CCE_ERR_INVALID_ARG",
    2: "CCE_ERR_UNSUPPORTED",
    3: "CCE_ERR_WORKSPACE",
    4: "CCE_ERR_TARGET_RANGE",
    5: "CCE_ERR_DEVICE_TIMEOUT",
    6: "CCE_ERR_CUDA",
}
DEFAULT_FILTER_EPS = 2.0 ** -12


class CCEError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class Problem(ctypes.Structure):
    _fields_ = [
        ("N", ctypes.c_int64),
        ("D", ctypes.c_int64),
        ("V", ctypes.c_int64),
        ("ignore_index", ctypes.c_int64),
        ("reduction", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
        ("label_smoothing", ctypes.c_float),
        ("z_loss", ctypes.c_float),
        ("vocab_start", ctypes.c_int64),
        ("vocab_total", ctypes.c_int64),
    ]


# Every symbol include/cce.h declares, with its ctypes signature.
_VP, _SZ, _I32, _I64, _F32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
_PP = ctypes.POINTER(Problem)
SIGNATURES = {
    "cce_tile_max_len": (_I64, [_PP]),
    "cce_backward_tile_shape": (None, [ctypes.POINTER(_I32), ctypes.POINTER(_I32)]),
    "cce_forward_workspace_size": (_SZ, [_PP]),
    "cce_backward_workspace_size": (_SZ, [_PP, _I32]),
    "cce_forward": (_I32, [_PP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "cce_backward": (_I32, [_PP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _F32, _VP, _VP, _VP, _I32, _VP, _VP, _SZ,
                            _VP]),
    "cce_check_device_error": (_I32, [_VP, _VP]),
    "cce_status_string": (ctypes.c_char_p, [_I32]),
    "cce_last_error_message": (ctypes.c_char_p, []),
    "cce_version": (_I32, []),
    "cce_set_kernel_events": (None, [_VP, _VP, _VP, _VP]),
    "cce_kernel_launch_count": (_I64, []),
    "cce_forward_noalloc": (_I32, [_PP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "cce_backward_skip_map": (_I32, [_PP, _VP, _SZ, _VP, _VP]),
    "cce_forward_partial": (_I32, [_PP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "cce_forward_merge": (_I32, [_PP, _VP, _I32, _VP, _VP, _VP, _VP, _VP]),
}

OUT_BF16, OUT_FP32, OUT_DE_FP32 = 0, 1, 2  # cce_backward's output dtype modes

_lib: Optional[ctypes.CDLL] = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libcce.so (once) and declare its signatures. Raises CCEError if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise CCEError(6, f"{path} not found: build it with `python -m linear_cross_entropy_06_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != 0:
        msg = _lib.cce_last_error_message().decode() if _lib is not None else ""
        raise CCEError(status, msg)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _problem(N: int, D: int, V: int, ignore_index: int, reduction: str, label_smoothing: float = 0.0,
             z_loss: float = 0.0, vocab_start: int = 0, vocab_total: int = 0) -> Problem:
    if reduction not in REDUCTION_CODES:
        raise ValueError(f"reduction must be one of {tuple(REDUCTION_CODES)}, got {reduction!r}")
    return Problem(N, D, V, ignore_index, REDUCTION_CODES[reduction], 0, float(label_smoothing), float(z_loss),
                   int(vocab_start), int(vocab_total))


def _require_cuda(*tensors: torch.Tensor) -> torch.device:
    dev = tensors[0].device
    if dev.type != "cuda":
        raise CCEError(1, "inputs must be CUDA tensors: there is no CPU path")
    for t in tensors:
        if t.device != dev:
            raise CCEError(1, "all inputs must be on the same device")
    return dev


def _require(cond: bool, message: str) -> None:
    if not cond:
        raise CCEError(1, message)


def _check_operands(E: torch.Tensor, C: torch.Tensor, targets: torch.Tensor) -> Tuple[int, int, int]:
    """Dtype and shape checks of E [N, D] bf16, C [V, D] bf16 and targets [N] int64 before any pointer
    reaches the library: the kernels read exactly N*D, V*D and N elements of those types."""
    _require(E.dim() == 2 and C.dim() == 2, f"E and C must be 2-D, got {tuple(E.shape)} and {tuple(C.shape)}")
    _require(E.dtype == torch.bfloat16 and C.dtype == torch.bfloat16,
             f"E and C must be bfloat16, got {E.dtype} and {C.dtype}")
    N, D = E.shape
    V = C.shape[0]
    _require(C.shape[1] == D, f"C must be [V, {D}], got {tuple(C.shape)}")
    _require(targets.dtype == torch.int64, f"targets must be int64, got {targets.dtype}")
    _require(targets.numel() == N, f"targets must have N={N} entries, got {targets.numel()}")
    return N, D, V


def backward_tile_shape() -> Tuple[int, int]:
    lib = load_library()
    r, c = _I32(), _I32()
    lib.cce_backward_tile_shape(ctypes.byref(r), ctypes.byref(c))
    return r.value, c.value


def _bias_arg(bias: Optional[torch.Tensor], V: int, dev: torch.device) -> Optional[torch.Tensor]:
    if bias is None:
        return None
    if bias.device != dev:
        raise CCEError(1, "bias must be on the same device as E and C")
    if bias.numel() != V:
        raise CCEError(1, f"bias must have V={V} entries, got {bias.numel()}")
    return bias.reshape(-1).to(torch.bfloat16).contiguous()


def cce_forward(E: torch.Tensor, C: torch.Tensor, targets: torch.Tensor, ignore_index: int = -100,
                reduction: str = "mean", check: bool = False, bias: Optional[torch.Tensor] = None,
                label_smoothing: float = 0.0, z_loss: float = 0.0):
    """Run the forward (logits E C^T + bias). Returns (loss, lse, tile_max, count) as device tensors."""
    lib = load_library()
    N, D, V = _check_operands(E, C, targets)
    dev = _require_cuda(E, C, targets)
    E, C, targets = E.contiguous(), C.contiguous(), targets.contiguous()
    bias = _bias_arg(bias, V, dev)
    p = _problem(N, D, V, ignore_index, reduction, label_smoothing, z_loss)
    loss = torch.empty(N if reduction == "none" else 1, device=dev, dtype=torch.float32)
    lse = torch.empty(N, device=dev, dtype=torch.float32)
    tm_len = lib.cce_tile_max_len(ctypes.byref(p))
    if tm_len < 0:
        raise CCEError(1, f"bad problem N={N} D={D} V={V}")
    tile_max = torch.empty(max(tm_len, 1), device=dev, dtype=torch.float32)
    count = torch.empty(1, device=dev, dtype=torch.int64)
    ws_bytes = lib.cce_forward_workspace_size(ctypes.byref(p))
    ws = torch.empty(max(ws_bytes, 1), device=dev, dtype=torch.uint8)
    with torch.cuda.device(dev):
        _check(lib.cce_forward(ctypes.byref(p), _ptr(E), _ptr(C), _ptr(bias), _ptr(targets), _ptr(loss), _ptr(lse),
                               _ptr(tile_max), _ptr(count), _ptr(ws), ws_bytes, _stream(dev)))
        if check:
            _check(lib.cce_check_device_error(_ptr(ws), _stream(dev)))
    return loss, lse, tile_max, count


def cce_backward(E: torch.Tensor, C: torch.Tensor, targets: torch.Tensor, lse: torch.Tensor,
                 tile_max: torch.Tensor, count: torch.Tensor, grad_out: torch.Tensor,
                 filter_eps: float = DEFAULT_FILTER_EPS, ignore_index: int = -100,
                 reduction: str = "mean", out_fp32=False, check: bool = False,
                 bias: Optional[torch.Tensor] = None, dbias: Optional[bool] = None,
                 label_smoothing: float = 0.0, z_loss: float = 0.0, skip_map: bool = False,
                 vocab_start: int = 0, vocab_total: int = 0):
    """Run the backward. Returns (dE, dC, filtered_tiles) as device tensors, then dbias when it is
    computed (``dbias``; by default whenever ``bias`` is given), then, with ``skip_map``, the uint8
    [ceil(N / tile_rows), ceil(V / tile_cols)] map of the skip rule's units (1 skipped, 0 kept).
    ``out_fp32``: False / OUT_BF16, True / OUT_FP32, or OUT_DE_FP32 (dE fp32, dC and dbias bf16).
    ``vocab_start`` / ``vocab_total``: C is rows [vocab_start, vocab_start + V) of a classifier of
    vocab_total rows (0: not sharded); lse and count are then the merged ones."""
    lib = load_library()
    N, D, V = _check_operands(E, C, targets)
    p = _problem(N, D, V, ignore_index, reduction, label_smoothing, z_loss, vocab_start, vocab_total)
    tm_len = lib.cce_tile_max_len(ctypes.byref(p))
    _require(tm_len >= 0, f"bad problem N={N} D={D} V={V}: {lib.cce_last_error_message().decode()}")
    # the saved forward state, read in full by the backward's kernels
    _require(lse.dtype == torch.float32 and lse.numel() == N, f"lse must be float32 with N={N} entries")
    _require(tile_max.dtype == torch.float32 and tile_max.numel() >= tm_len,
             f"tile_max must be float32 with at least {tm_len} entries")
    _require(count.dtype == torch.int64 and count.numel() >= 1, "count must be an int64 tensor of one entry")
    _require(grad_out.numel() == (N if reduction == "none" else 1),
             f"grad_out must have {N if reduction == 'none' else 1} entries for reduction={reduction!r}")
    dev = _require_cuda(E, C, targets, lse, tile_max, count)
    E, C, targets = E.contiguous(), C.contiguous(), targets.contiguous()
    lse, tile_max, count = lse.contiguous(), tile_max.contiguous(), count.contiguous()
    bias = _bias_arg(bias, V, dev)
    want_dbias = (bias is not None) if dbias is None else bool(dbias)
    g = grad_out.to(device=dev, dtype=torch.float32).reshape(-1).contiguous()
    mode = int(out_fp32)
    _require(mode in (OUT_BF16, OUT_FP32, OUT_DE_FP32), f"out_fp32 must be 0, 1 or 2, got {out_fp32!r}")
    de_dtype = torch.float32 if mode in (OUT_FP32, OUT_DE_FP32) else torch.bfloat16
    dc_dtype = torch.float32 if mode == OUT_FP32 else torch.bfloat16
    dE = torch.empty(N, D, device=dev, dtype=de_dtype)
    dC = torch.empty(V, D, device=dev, dtype=dc_dtype)
    db = torch.empty(V, device=dev, dtype=dc_dtype) if want_dbias else None
    filtered = torch.empty(1, device=dev, dtype=torch.int64)
    ws_bytes = lib.cce_backward_workspace_size(ctypes.byref(p), mode)
    _require(ws_bytes > 0, f"bad problem: {lib.cce_last_error_message().decode()}")
    ws = torch.empty(max(ws_bytes, 1), device=dev, dtype=torch.uint8)
    with torch.cuda.device(dev):
        _check(lib.cce_backward(ctypes.byref(p), _ptr(E), _ptr(C), _ptr(bias), _ptr(targets), _ptr(lse),
                                _ptr(tile_max), _ptr(count), _ptr(g), float(filter_eps), _ptr(dE), _ptr(dC), _ptr(db),
                                mode, _ptr(filtered), _ptr(ws), ws_bytes, _stream(dev)))
        smap = None
        if skip_map:
            tr, tc = backward_tile_shape()
            smap = torch.empty(-(-N // tr), -(-V // tc), device=dev, dtype=torch.uint8)
            _check(lib.cce_backward_skip_map(ctypes.byref(p), _ptr(ws), ws_bytes, _ptr(smap), _stream(dev)))
        if check:
            _check(lib.cce_check_device_error(_ptr(ws), _stream(dev)))
    out = (dE, dC, filtered) + ((db,) if want_dbias else ())
    return out + (smap,) if skip_map else out


def cce_forward_partial(E: torch.Tensor, C: torch.Tensor, targets: torch.Tensor, vocab_start: int, vocab_total: int,
                        ignore_index: int = -100, bias: Optional[torch.Tensor] = None, label_smoothing: float = 0.0,
                        check: bool = False):
    """Forward of one vocabulary shard: C is rows [vocab_start, vocab_start + V) of a classifier of
    vocab_total rows. Returns (partial [3, N] fp32, tile_max) as device tensors: per row the shard's
    log-sum-exp, the correct-token logit when the target lies in the shard (else 0), and the sum of
    the shard's logits (label smoothing only; else 0)."""
    lib = load_library()
    N, D, V = _check_operands(E, C, targets)
    dev = _require_cuda(E, C, targets)
    E, C, targets = E.contiguous(), C.contiguous(), targets.contiguous()
    bias = _bias_arg(bias, V, dev)
    p = _problem(N, D, V, ignore_index, "none", label_smoothing, 0.0, vocab_start, vocab_total)
    tm_len = lib.cce_tile_max_len(ctypes.byref(p))
    _require(tm_len >= 0, f"bad problem: {lib.cce_last_error_message().decode()}")
    partial = torch.empty(3, N, device=dev, dtype=torch.float32)
    tile_max = torch.empty(max(tm_len, 1), device=dev, dtype=torch.float32)
    ws_bytes = lib.cce_forward_workspace_size(ctypes.byref(p))
    ws = torch.empty(max(ws_bytes, 1), device=dev, dtype=torch.uint8)
    with torch.cuda.device(dev):
        _check(lib.cce_forward_partial(ctypes.byref(p), _ptr(E), _ptr(C), _ptr(bias), _ptr(targets), _ptr(partial),
                                       _ptr(tile_max), _ptr(ws), ws_bytes, _stream(dev)))
        if check:
            _check(lib.cce_check_device_error(_ptr(ws), _stream(dev)))
    return partial, tile_max


def cce_forward_merge(partials: torch.Tensor, targets: torch.Tensor, V: int, D: int, ignore_index: int = -100,
                      reduction: str = "mean", label_smoothing: float = 0.0, z_loss: float = 0.0):
    """Loss, LSE over the whole vocabulary of V entries, and count, from every shard's partial
    results stacked as [shards, 3, N]. Returns (loss, lse, count) as device tensors."""
    lib = load_library()
    _require(partials.dim() == 3 and partials.shape[1] == 3 and partials.dtype == torch.float32,
             f"partials must be float32 [shards, 3, N], got {partials.dtype} {tuple(partials.shape)}")
    shards, _, N = partials.shape
    _require(targets.dtype == torch.int64 and targets.numel() == N, f"targets must be int64 with N={N} entries")
    dev = _require_cuda(partials, targets)
    partials, targets = partials.contiguous(), targets.contiguous()
    p = _problem(N, D, V, ignore_index, reduction, label_smoothing, z_loss)
    loss = torch.empty(N if reduction == "none" else 1, device=dev, dtype=torch.float32)
    lse = torch.empty(N, device=dev, dtype=torch.float32)
    count = torch.empty(1, device=dev, dtype=torch.int64)
    with torch.cuda.device(dev):
        _check(lib.cce_forward_merge(ctypes.byref(p), _ptr(partials), shards, _ptr(targets), _ptr(loss), _ptr(lse),
                                     _ptr(count), _stream(dev)))
    return loss, lse, count


class _LinearCrossEntropy(torch.autograd.Function):
    @staticmethod
    def forward(ctx, E, C, bias, targets, ignore_index, reduction, filter_eps, label_smoothing, z_loss):
        loss, lse, tile_max, count = cce_forward(E, C, targets, ignore_index, reduction, bias=bias,
                                                 label_smoothing=label_smoothing, z_loss=z_loss)
        ctx.save_for_backward(E, C, bias, targets, lse, tile_max, count)
        ctx.cfg = (ignore_index, reduction, filter_eps, label_smoothing, z_loss)
        return loss if reduction == "none" else loss.reshape(())

    @staticmethod
    def backward(ctx, grad_loss):
        E, C, bias, targets, lse, tile_max, count = ctx.saved_tensors
        ignore_index, reduction, filter_eps, label_smoothing, z_loss = ctx.cfg
        want_db = bias is not None and ctx.needs_input_grad[2]
        out = cce_backward(E, C, targets, lse, tile_max, count, grad_loss, filter_eps, ignore_index, reduction,
                           out_fp32=False, bias=bias, dbias=want_db, label_smoothing=label_smoothing, z_loss=z_loss)
        dbias = out[3].to(bias.dtype) if want_db else None
        return out[0].to(E.dtype), out[1].to(C.dtype), dbias, None, None, None, None, None, None


def shift_targets(targets: torch.Tensor, ignore_index: int = -100) -> torch.Tensor:
    """Causal-LM targets for hidden states of shape [..., T, D]: position i predicts token i + 1,
    and the last position of each sequence has no target (``ignore_index``)."""
    out = torch.full_like(targets, ignore_index)
    out[..., :-1] = targets[..., 1:]
    return out


def linear_cross_entropy(e: torch.Tensor, c: torch.Tensor, targets: torch.Tensor,
                         bias: Optional[torch.Tensor] = None, reduction: str = "mean", ignore_index: int = -100,
                         filter_eps: float = DEFAULT_FILTER_EPS, label_smoothing: float = 0.0, z_loss: float = 0.0,
                         shift: bool = False) -> torch.Tensor:
    """Cross-entropy of softmax(e @ c.T + bias) at ``targets`` without materialising the logits.

    e: [..., D] bf16 hidden states; c: [V, D] bf16 classifier; targets: [...] int64; bias: optional
    [V] classifier bias (mlx-cross-entropy README, "API" table). ``label_smoothing`` and ``z_loss``
    select the smoothed target and the z-loss of the Loss functions explainer (0 and 0: plain
    cross-entropy). ``shift`` makes e[..., i, :] predict targets[..., i + 1] (causal language
    modelling over a trailing sequence axis); the last position of each sequence is then ignored.
    Returns a scalar (mean/sum) or the per-token loss in the shape of ``targets`` (none; with
    ``shift``, one position shorter along the sequence axis).
    """
    if e.shape[:-1] != targets.shape:
        raise ValueError(f"targets shape {tuple(targets.shape)} must equal e.shape[:-1] {tuple(e.shape[:-1])}")
    if shift:
        if targets.dim() < 1 or targets.shape[-1] < 1:
            raise ValueError("shift needs a sequence axis of length >= 1")
        targets = shift_targets(targets, ignore_index)
    lead = targets.shape
    E = e.reshape(-1, e.shape[-1])
    t = targets.reshape(-1).to(torch.int64)
    out = _LinearCrossEntropy.apply(E, c, bias, t, ignore_index, reduction, filter_eps, label_smoothing, z_loss)
    if reduction != "none":
        return out
    out = out.reshape(lead)
    return out[..., :-1] if shift else out


def perplexity(e: torch.Tensor, c: torch.Tensor, targets: torch.Tensor, bias: Optional[torch.Tensor] = None,
               ignore_index: int = -100, shift: bool = False) -> torch.Tensor:
    """Perplexity exp(mean NLL) of the classifier on ``targets``, the mean taken over non-ignored
    tokens (mlx-cross-entropy README, "Computing related quantities": the exponential of the mean
    per-token negative log-likelihood). The mean NLL is the library's forward with reduction
    "mean" (computed in its kernels, no logits stored); only the exponential of that one number is
    taken here. With every token ignored the mean is 0 and the perplexity 1. No gradient flows."""
    with torch.no_grad():
        nll = linear_cross_entropy(e, c, targets, bias=bias, reduction="mean", ignore_index=ignore_index,
                                   shift=shift)
    return torch.exp(nll)
