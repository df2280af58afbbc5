"""The collective logic of the vocabulary-parallel loss on CPU: two and three gloo ranks.

linear_cross_entropy_vocab_parallel splits the classifier by rows (shard_range), runs three
per-shard computations and joins them with two collectives: an all-gather of every shard's
partial results in the forward and an all-reduce (sum) of dE in the backward. On the GPU the
per-shard computations are the library's kernels (tests/test_gpu_vocab_parallel.py checks them
against the oracle). Here, without a GPU, they are replaced by a float64 restatement of the same
definitions, so that what is tested is the partition, the collectives and the autograd plumbing:
every rank must end with the oracle's loss and dE on the whole vocabulary, and the ranks' dC and
dbias rows, put together, must be the oracle's.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem():
    rng = np.random.default_rng(81)
    N, D, V = 24, 16, 700
    C = rng.standard_normal((V, D)) / 4.0
    t = rng.integers(0, V, N)
    t[[2, 9]] = -100
    E = rng.standard_normal((N, D)) + 3.0 * C[np.where(t >= 0, t, 0)]
    bias = rng.standard_normal(V) * 0.2
    g = rng.standard_normal(N)
    return E, C, t, bias, g


def _fake_ops(ls, zl):
    """float64 stand-ins for the three per-shard kernels (definitions of the Loss functions
    explainer, How it works items 1-3; no tile skipping: the test runs with filter_eps = 0)."""
    from linear_cross_entropy_06_b200.vocab_parallel import ShardOps

    def forward_partial(E, C, targets, vs, vtot, ignore_index, bias=None, label_smoothing=0.0):
        z = E.detach() @ C.detach().T + (0.0 if bias is None else bias.detach()[None, :])
        lse = torch.logsumexp(z, dim=1)
        tl = targets - vs
        local = (targets != ignore_index) & (tl >= 0) & (tl < C.shape[0])
        zt = torch.where(local, z.gather(1, tl.clamp(0, C.shape[0] - 1)[:, None])[:, 0], torch.zeros_like(lse))
        zs = z.sum(1) if label_smoothing else torch.zeros_like(lse)
        return torch.stack([lse, zt, zs]), None

    def merge(parts, targets, V, D, ignore_index, reduction, label_smoothing, z_loss):
        L = torch.logsumexp(parts[:, 0], dim=0)
        zt, zs = parts[:, 1].sum(0), parts[:, 2].sum(0)
        valid = targets != ignore_index
        rows = torch.where(valid, L - (1 - label_smoothing) * zt - label_smoothing / V * zs + z_loss * L * L,
                           torch.zeros_like(L))
        count = valid.sum().reshape(1)
        loss = {"none": rows, "sum": rows.sum().reshape(1),
                "mean": (rows.sum() / count.clamp(min=1)).reshape(1)}[reduction]
        return loss, L, count

    def backward(E, C, targets, lse, tile_max, count, grad, eps, ignore_index, reduction, out_fp32=None, bias=None,
                 dbias=False, label_smoothing=0.0, z_loss=0.0, vocab_start=0, vocab_total=0):
        assert eps == 0.0 and tile_max is None
        z = E @ C.T + (0.0 if bias is None else bias[None, :])
        p = torch.exp(z - lse[:, None])
        valid = targets != ignore_index
        g = grad.reshape(-1)
        scale = {"mean": g[0] / count.clamp(min=1), "sum": g[0] + 0 * lse, "none": g}[reduction] * valid
        G = (scale * (1 + 2 * z_loss * lse))[:, None] * p - (scale * label_smoothing / vocab_total)[:, None]
        tl = targets - vocab_start
        local = valid & (tl >= 0) & (tl < C.shape[0])
        G[local, tl[local]] -= scale[local] * (1 - label_smoothing)
        out = (G @ C, G.T @ E, None)
        return out + ((G.sum(0),) if dbias else ())

    return ShardOps(forward_partial, merge, backward)


def _worker(rank, world, port, reduction, ls, zl, out):
    import sys

    sys.path.insert(0, ROOT)
    from linear_cross_entropy_06_b200.vocab_parallel import linear_cross_entropy_vocab_parallel, shard_range

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        E, C, t, bias, g = _problem()
        V = C.shape[0]
        vs, n = shard_range(V, world, rank)
        e = torch.tensor(E).reshape(4, 6, -1).requires_grad_(True)
        c = torch.tensor(C[vs:vs + n]).requires_grad_(True)
        b = torch.tensor(bias[vs:vs + n]).requires_grad_(True)
        tt = torch.tensor(t).reshape(4, 6)
        loss = linear_cross_entropy_vocab_parallel(e, c, tt, vs, V, bias_shard=b, reduction=reduction,
                                                   filter_eps=0.0, label_smoothing=ls, z_loss=zl,
                                                   shard_ops=_fake_ops(ls, zl))
        gl = torch.tensor(g).reshape(4, 6) if reduction == "none" else torch.tensor(1.0, dtype=torch.float64)
        loss.backward(gl)
        out[rank] = (vs, n, loss.detach().numpy(), e.grad.reshape(24, -1).numpy(), c.grad.numpy(), b.grad.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("reduction,ls,zl", [("mean", 0.0, 0.0), ("none", 0.1, 1e-3)])
def test_gloo_ranks_reproduce_the_whole_vocabulary(world, reduction, ls, zl):
    import sys

    sys.path.insert(0, ROOT)
    from oracle import cce_oracle as O

    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, reduction, ls, zl, out), nprocs=world, join=True,
                           start_method="spawn")
        res = [out[r] for r in range(world)]
    E, C, t, bias, g = _problem()
    V = C.shape[0]
    g_or = g if reduction == "none" else 1.0
    f = O.forward(E, C, t, -100, reduction, bias=bias, label_smoothing=ls, z_loss=zl)
    b = O.backward(E, C, t, g_or, -100, reduction, 0.0, 8, 64, bias=bias, label_smoothing=ls, z_loss=zl)
    starts = [r[0] for r in res]
    assert starts == sorted(starts) and starts[0] == 0 and sum(r[1] for r in res) == V
    assert all(s % 128 == 0 for s in starts)  # shard boundaries on the kernels' vocabulary tiles
    for vs, n, loss, dE, dC, db in res:
        np.testing.assert_allclose(loss.reshape(np.shape(f.loss)), f.loss, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dE, b.dE, rtol=1e-9, atol=1e-12)  # the all-reduce of the shards' parts
        np.testing.assert_allclose(dC, b.dC[vs:vs + n], rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(db, b.dbias[vs:vs + n], rtol=1e-9, atol=1e-12)


def test_shard_range_partition():
    import sys

    sys.path.insert(0, ROOT)
    from linear_cross_entropy_06_b200.vocab_parallel import shard_range

    for V, world in [(128256, 8), (256000, 8), (1000, 3), (100, 4), (5000, 2)]:
        ranges = [shard_range(V, world, r) for r in range(world)]
        assert ranges[0][0] == 0 and sum(n for _, n in ranges) == V
        for (s0, n0), (s1, _) in zip(ranges, ranges[1:]):
            assert s0 + n0 == s1 and s1 % 128 == 0
        sizes = [n for _, n in ranges if n]
        assert max(sizes) - min(sizes) <= 128 + (V % 128)
    with pytest.raises(ValueError):
        shard_range(1000, 2, 2)
