"""Vocabulary-parallel linear cross-entropy: the classifier split by rows over the ranks of a group.

Every rank holds the same hidden states E [N, D] and targets, and one contiguous range of the
classifier's rows, C[vocab_start : vocab_start + V_r] of vocab_total rows. The loss of each token
needs the log-sum-exp over the whole vocabulary (Loss functions explainer, "How it works" item 1),
which the shards' partial log-sum-exps give exactly, as the tiles of one GPU do (mlx-cross-entropy
README, "How it works" item 1: partial maxima and sums combine into a stable log-sum-exp).

Forward, on every rank:
  1. cce_forward_partial on its shard: per row the shard's log-sum-exp, the correct-token logit when
     the target lies in the shard (else 0), and the shard's logit sum (label smoothing only);
  2. one all-gather of those 3N floats from every rank;
  3. cce_forward_merge: the loss, the LSE over the whole vocabulary and the count, identical on
     every rank.
Backward, on every rank: cce_backward on its shard with the merged LSE and count gives the shard's
rows of dC (and dbias) and the shard's part of dE (fp32); one all-reduce (sum) of N x D fp32 values
gives dE. Tile skipping works per shard: a tile's decision reads only its own rows and columns.

The shards' compute runs in the library's CUDA kernels; this module holds the partition of the
vocabulary and the two collectives of torch.distributed (NCCL on GPUs). ``shard_ops`` replaces the
three per-shard calls (used by CPU tests of the collective logic).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional, Tuple

import torch
import torch.distributed as dist

from . import ops

TILE_ROWS = 128  # shard boundaries fall on multiples of the kernels' 128-row vocabulary tiles


def shard_range(vocab_total: int, world: int, rank: int, align: int = TILE_ROWS) -> Tuple[int, int]:
    """(vocab_start, rows) of rank `rank`'s shard: contiguous ranges covering [0, vocab_total) in rank
    order, boundaries on multiples of `align`, sizes differing by at most one `align` block."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a group of {world}")
    blocks = -(-vocab_total // align)
    lo = blocks * rank // world
    hi = blocks * (rank + 1) // world
    start, stop = min(lo * align, vocab_total), min(hi * align, vocab_total)
    return start, stop - start


@dataclass
class ShardOps:
    """The three per-shard computations (defaults: the library's kernels)."""
    forward_partial: Callable = ops.cce_forward_partial
    merge: Callable = ops.cce_forward_merge
    backward: Callable = ops.cce_backward


def _world(group) -> Tuple[int, int]:
    return dist.get_world_size(group), dist.get_rank(group)


class _VocabParallelCrossEntropy(torch.autograd.Function):
    @staticmethod
    def forward(ctx, E, C, bias, targets, vocab_start, vocab_total, group, ignore_index, reduction, filter_eps,
                label_smoothing, z_loss, shard_ops):
        partial, tile_max = shard_ops.forward_partial(E, C, targets, vocab_start, vocab_total, ignore_index,
                                                      bias=bias, label_smoothing=label_smoothing)
        world, _ = _world(group)
        parts = [torch.empty_like(partial) for _ in range(world)]
        dist.all_gather(parts, partial.contiguous(), group=group)
        loss, lse, count = shard_ops.merge(torch.stack(parts), targets, vocab_total, E.shape[1], ignore_index,
                                           reduction, label_smoothing, z_loss)
        ctx.save_for_backward(E, C, bias, targets, lse, tile_max, count)
        ctx.cfg = (vocab_start, vocab_total, group, ignore_index, reduction, filter_eps, label_smoothing, z_loss,
                   shard_ops)
        return loss if reduction == "none" else loss.reshape(())

    @staticmethod
    def backward(ctx, grad_loss):
        E, C, bias, targets, lse, tile_max, count = ctx.saved_tensors
        vocab_start, vocab_total, group, ignore_index, reduction, filter_eps, ls, zl, shard_ops = ctx.cfg
        want_db = bias is not None and ctx.needs_input_grad[2]
        out = shard_ops.backward(E, C, targets, lse, tile_max, count, grad_loss, filter_eps, ignore_index, reduction,
                                 out_fp32=ops.OUT_DE_FP32, bias=bias, dbias=want_db, label_smoothing=ls, z_loss=zl,
                                 vocab_start=vocab_start, vocab_total=vocab_total)
        dE = out[0]
        dist.all_reduce(dE, op=dist.ReduceOp.SUM, group=group)  # every shard's part of dE
        dbias = out[3].to(bias.dtype) if want_db else None
        return (dE.to(E.dtype), out[1].to(C.dtype), dbias) + (None,) * 10


def linear_cross_entropy_vocab_parallel(e: torch.Tensor, c_shard: torch.Tensor, targets: torch.Tensor,
                                        vocab_start: int, vocab_total: int, group=None,
                                        bias_shard: Optional[torch.Tensor] = None, reduction: str = "mean",
                                        ignore_index: int = -100, filter_eps: float = ops.DEFAULT_FILTER_EPS,
                                        label_smoothing: float = 0.0, z_loss: float = 0.0,
                                        shard_ops: Optional[ShardOps] = None) -> torch.Tensor:
    """Cross-entropy of softmax(e @ C.T + bias) at ``targets`` with C split by rows over ``group``.

    e: [..., D] hidden states (the same on every rank); c_shard: this rank's rows
    [vocab_start, vocab_start + V_r) of the classifier; targets: [...] ids in [0, vocab_total);
    bias_shard: this rank's entries of the bias, or None. Returns the loss of the whole vocabulary,
    identical on every rank: a scalar (mean / sum) or the per-token loss in the targets' shape
    (none). Gradients: e gets the full dE on every rank, c_shard and bias_shard their own rows."""
    if e.shape[:-1] != targets.shape:
        raise ValueError(f"targets shape {tuple(targets.shape)} must equal e.shape[:-1] {tuple(e.shape[:-1])}")
    if not 0 <= vocab_start <= vocab_total - c_shard.shape[0]:
        raise ValueError("the shard's rows must lie inside [0, vocab_total)")
    lead = targets.shape
    E = e.reshape(-1, e.shape[-1])
    t = targets.reshape(-1).to(torch.int64)
    out = _VocabParallelCrossEntropy.apply(E, c_shard, bias_shard, t, int(vocab_start), int(vocab_total), group,
                                           ignore_index, reduction, filter_eps, label_smoothing, z_loss,
                                           shard_ops or ShardOps())
    return out if reduction != "none" else out.reshape(lead)
