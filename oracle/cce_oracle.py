"""fp64 CPU oracle for linear cross-entropy, the computation Cut Cross-Entropy performs.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. The CUDA library never calls it, and it never calls the CUDA library:
the two share no code.

What it computes, and where that is stated:

* Cut Your Losses in Large-Vocabulary Language Models (paper-index page,
  abstract): the loss is the ordinary cross-entropy of ``softmax(E @ C.T)`` at the
  correct tokens. CCE only avoids materialising the logits. This oracle
  materialises them (in row groups), in float64.
* Cut Cross Entropy from first principles (blog, first paragraph): per token,
  ``loss = LSE - z_correct``.
* Loss functions (explainer), "How it works" items 1, 2 and 4: the stable
  log-sum-exp ``m + log sum exp(z - m)``; the logit gradient ``p - y``; the mean
  over non-ignored tokens only.
* mlx-cross-entropy README, "API" table: ``reduction`` in {mean, sum, none},
  ``ignore_index`` (default -100) masks a token, and an optional classifier bias
  ``[V]`` is added to every row of logits: ``z = E @ C.T + bias``. Its gradient is
  the column sum of the logit gradient, ``dbias = sum_r G[r, :]``.
* mlx-cross-entropy README, "How it works" item 2: the backward skips tiles
  whose softmax is below ``2**-12``. The rule here, per tile of ``tile_m`` rows by
  ``tile_n`` vocabulary columns: the tile is skipped when every non-ignored row
  ``r`` in it, at every column ``v`` in it, has ``z[r, v] - LSE[r] < ln(eps)``.
  A tile with no non-ignored row is skipped. ``eps <= 0`` turns skipping off.
  The onehot term of the gradient is never skipped.

* Loss functions (explainer), "How it works" item 3 and its listing: label
  smoothing replaces the one-hot target with ``(1 - ls) * onehot + ls / V``; the
  loss is ``-sum_v target_v * log p_v`` and the gradient stays ``p - target``.
  Per row that is ``LSE - (1 - ls) * z_t - (ls / V) * sum_v z_v``.
* Loss functions (explainer), "Implementation notes": the z-loss adds
  ``zl * LSE**2`` per token (PaLM uses zl = 1e-4); its logit gradient is
  ``2 * zl * LSE * p``.

Readings where the pages leave a step open:

* ``mean`` with every token ignored gives loss 0 and a zero gradient: the sum
  is divided by ``max(count, 1)``, as the explainer's listing does. PyTorch
  returns NaN in this case.
* With ``reduction='none'`` an ignored token's loss is exactly 0.
* The gradient's upstream factor ``grad_out`` is a scalar for mean/sum and a
  per-token vector for none. The scale of row ``r`` is ``g / max(count, 1)``
  (mean), ``g`` (sum) or ``g[r]`` (none), and 0 for ignored rows.
* Tile skipping drops only the softmax part of the gradient,
  ``(1 + 2 zl LSE) * p``; the target part ``(1 - ls) * onehot + ls / V`` is
  never skipped (it does not depend on the logits).

Every function is pinned by ``tests/test_oracle_pins.py`` against closed forms,
values the pages print, finite differences, brute force and an independent
library routine (``torch.nn.functional.cross_entropy`` in float64).
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Iterator, Optional, Sequence

import numpy as np

REDUCTIONS = ("mean", "sum", "none")

# Row-group size used when the logits are materialised piecewise. The rows of
# the loss are independent, so evaluating them group by group is the same
# definition; only sums over rows (dC, the reductions) see a different order.
ROW_GROUP = 512


def _f64(x) -> np.ndarray:
    """Exact float64 copy of a numpy array or a torch tensor (bf16 included)."""
    try:
        import torch  # local: the oracle itself needs only numpy

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def _i64(x) -> np.ndarray:
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.int64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.int64)


def validate_targets(targets: np.ndarray, V: int, ignore_index: int) -> None:
    """Each target is a class index in [0, V) or ``ignore_index``.

    mlx-cross-entropy README, "API" table (``targets``: target indices;
    ``ignore_index``: target index to mask).
    """
    t = _i64(targets)
    bad = (t != ignore_index) & ((t < 0) | (t >= V))
    if bad.any():
        r = int(np.flatnonzero(bad)[0])
        raise ValueError(f"target {int(t[r])} at row {r} is outside [0, {V}) and is not ignore_index")


def _bias64(bias, V: int) -> Optional[np.ndarray]:
    if bias is None:
        return None
    b = _f64(bias).reshape(-1)
    if b.shape[0] != V:
        raise ValueError(f"bias must have {V} entries, got {b.shape[0]}")
    return b


def logits(E: np.ndarray, C: np.ndarray, bias=None) -> np.ndarray:
    """z = E @ C.T (+ bias) in float64 (mlx-cross-entropy README, "How it works" item 1: e @ c.T;
    "API" table: classifier bias [V])."""
    z = _f64(E) @ _f64(C).T
    b = _bias64(bias, z.shape[1])
    return z if b is None else z + b[None, :]


def log_sum_exp_rows(z: np.ndarray) -> np.ndarray:
    """Stable per-row log-sum-exp: m + log(sum(exp(z - m))), m the row max.

    Loss functions explainer, "How it works" item 1.
    """
    m = z.max(axis=1)
    return m + np.log(np.exp(z - m[:, None]).sum(axis=1))


def softmax_rows(z: np.ndarray, lse: np.ndarray) -> np.ndarray:
    """p = exp(z - LSE) per row (the normaliser shared by softmax and the loss)."""
    return np.exp(z - lse[:, None])


def _row_groups(n: int, group: Optional[int] = None) -> Iterator[slice]:
    group = ROW_GROUP if group is None else group  # read at call time (tests shrink it)
    for r0 in range(0, n, group):
        yield slice(r0, min(r0 + group, n))


@dataclass
class ForwardResult:
    loss: np.ndarray  # shape [] for mean/sum, [N] for none
    lse: np.ndarray  # [N]
    z_target: np.ndarray  # [N]; 0 for ignored rows
    nll: np.ndarray  # [N] per-token loss; 0 for ignored rows
    count: int  # number of non-ignored rows


def reduce_loss(nll: np.ndarray, count: int, reduction: str) -> np.ndarray:
    """Reduction over tokens.

    mlx-cross-entropy README, "API" table (mean / sum / none); Loss functions
    explainer, "How it works" item 4 (average over non-ignored tokens).
    """
    if reduction == "mean":
        return np.asarray(nll.sum() / max(count, 1))
    if reduction == "sum":
        return np.asarray(nll.sum())
    if reduction == "none":
        return nll.copy()
    raise ValueError(f"reduction must be one of {REDUCTIONS}, got {reduction!r}")


def row_loss(lse, z_target, z_sum, V: int, valid, label_smoothing: float = 0.0, z_loss: float = 0.0):
    """Per-token loss: LSE - (1 - ls) z_t - (ls / V) sum_v z_v + zl LSE^2; 0 for ignored tokens.

    Cut Cross Entropy from first principles (loss = -correct_token + LSE); Loss
    functions explainer, "How it works" item 3 (smoothed target) and "Implementation
    notes" (z-loss).
    """
    nll = lse - (1.0 - label_smoothing) * z_target - (label_smoothing / V) * z_sum + z_loss * lse * lse
    return np.where(valid, nll, 0.0)


def logit_grad(p, lse, targets, valid, scale, label_smoothing: float = 0.0, z_loss: float = 0.0):
    """G = scale_r * ((1 + 2 zl LSE_r) * p - (1 - ls) * onehot - ls / V) for the rows given.

    ``p`` may have skipped tiles already set to 0 (only the softmax part is skipped).
    Loss functions explainer, "How it works" items 2 and 3: the gradient is p - target.
    """
    V = p.shape[1]
    G = (scale * (1.0 + 2.0 * z_loss * lse))[:, None] * p
    rv = np.flatnonzero(valid)
    G[rv, targets[rv]] -= scale[rv] * (1.0 - label_smoothing)
    if label_smoothing:
        G[rv] -= (scale[rv] * (label_smoothing / V))[:, None]
    return G


def forward_rows(E, C, targets, rows: Optional[Sequence[int]] = None, ignore_index: int = -100, bias=None,
                 label_smoothing: float = 0.0, z_loss: float = 0.0):
    """Per-row LSE, correct-token logit and loss for a subset of rows.

    Each row of the loss depends only on its own hidden state, so any subset of
    rows can be evaluated exactly. Returns (rows, lse, z_target, nll, valid).
    """
    E64, C64, t = _f64(E), _f64(C), _i64(targets)
    V = C64.shape[0]
    b = _bias64(bias, V)
    validate_targets(t, V, ignore_index)
    rows = np.arange(E64.shape[0]) if rows is None else np.asarray(rows, dtype=np.int64)
    lse = np.empty(len(rows))
    zt = np.zeros(len(rows))
    zs = np.zeros(len(rows))
    for g in _row_groups(len(rows)):
        rr = rows[g]
        z = E64[rr] @ C64.T
        if b is not None:
            z += b[None, :]
        lse[g] = log_sum_exp_rows(z)
        zs[g] = z.sum(axis=1)
        tr = t[rr]
        ok = tr != ignore_index
        zt[g] = np.where(ok, z[np.arange(len(rr)), np.where(ok, tr, 0)], 0.0)
    valid = t[rows] != ignore_index
    nll = row_loss(lse, zt, zs, V, valid, label_smoothing, z_loss)
    return rows, lse, zt, nll, valid


def forward(E, C, targets, ignore_index: int = -100, reduction: str = "mean", bias=None,
            label_smoothing: float = 0.0, z_loss: float = 0.0) -> ForwardResult:
    """Loss and per-row LSE of linear cross-entropy (the forward the CUDA path computes)."""
    if reduction not in REDUCTIONS:
        raise ValueError(f"reduction must be one of {REDUCTIONS}, got {reduction!r}")
    _, lse, zt, nll, valid = forward_rows(E, C, targets, None, ignore_index, bias, label_smoothing, z_loss)
    count = int(valid.sum())
    return ForwardResult(reduce_loss(nll, count, reduction), lse, zt, nll, count)


def row_scale(targets, ignore_index: int, reduction: str, grad_out, count: int) -> np.ndarray:
    """Factor multiplying row r of the logit gradient (p - y).

    Loss functions explainer, "How it works" items 2 and 4, and its listing's
    ``(p - target) / count``. Ignored rows get 0.
    """
    t = _i64(targets)
    valid = t != ignore_index
    g = _f64(grad_out)
    if reduction == "mean":
        s = np.full(t.shape[0], float(g.reshape(-1)[0]) / max(count, 1))
    elif reduction == "sum":
        s = np.full(t.shape[0], float(g.reshape(-1)[0]))
    elif reduction == "none":
        s = g.reshape(-1).astype(np.float64).copy()
        if s.shape[0] != t.shape[0]:
            raise ValueError("grad_out must have one entry per token for reduction='none'")
    else:
        raise ValueError(f"reduction must be one of {REDUCTIONS}, got {reduction!r}")
    return np.where(valid, s, 0.0)


def tile_log_margin(z_minus_lse: np.ndarray, valid: np.ndarray, tile_m: int, tile_n: int) -> np.ndarray:
    """max over the tile's non-ignored rows and its columns of (z - LSE); -inf if no row is valid.

    Shape [ceil(n/tile_m), ceil(V/tile_n)] for the n rows given.
    """
    n, V = z_minus_lse.shape
    nb, nt = -(-n // tile_m), -(-V // tile_n)
    out = np.full((nb, nt), -np.inf)
    masked = np.where(valid[:, None], z_minus_lse, -np.inf)
    for b in range(nb):
        blk = masked[b * tile_m:(b + 1) * tile_m]
        for t in range(nt):
            out[b, t] = blk[:, t * tile_n:(t + 1) * tile_n].max()
    return out


def filtered_tiles(margin: np.ndarray, filter_eps: float) -> np.ndarray:
    """True where the tile is skipped: every valid softmax entry in it is below eps.

    mlx-cross-entropy README, "How it works" item 2 (skip tiles where softmax <
    2^-12). Compared in log space, strict: skipped iff max(z - LSE) < ln(eps).
    ``filter_eps <= 0`` skips nothing.
    """
    if filter_eps <= 0:
        return np.zeros(margin.shape, dtype=bool)
    return margin < math.log(filter_eps)


@dataclass
class BackwardResult:
    dE: np.ndarray  # [N, D]
    dC: np.ndarray  # [V, D]
    filtered: int  # number of skipped tiles
    borderline: int  # tiles whose margin is within `window` of ln(eps)
    n_tiles: int
    dbias: Optional[np.ndarray] = None  # [V] when a bias is given
    margin: Optional[np.ndarray] = None  # [ceil(N/tile_m), ceil(V/tile_n)] max over valid rows of z - LSE


def backward(E, C, targets, grad_out=1.0, ignore_index: int = -100, reduction: str = "mean",
             filter_eps: float = 2.0 ** -12, tile_m: int = 128, tile_n: int = 256,
             window: float = 2e-3, bias=None, label_smoothing: float = 0.0, z_loss: float = 0.0) -> BackwardResult:
    """dE, dC (and dbias) of linear cross-entropy, with the tile-skipping rule applied.

    G = scale_r * (p~ - onehot), p~ = softmax with skipped tiles set to 0;
    dE = G @ C, dC = G.T @ E, dbias = column sums of G (Loss functions explainer,
    "How it works" item 2: the logit gradient is p - y; mlx-cross-entropy README,
    "How it works" item 2: skipped tiles contribute nothing).
    """
    E64, C64, t = _f64(E), _f64(C), _i64(targets)
    N, V = E64.shape[0], C64.shape[0]
    validate_targets(t, V, ignore_index)
    valid = t != ignore_index
    count = int(valid.sum())
    scale = row_scale(t, ignore_index, reduction, grad_out, count)

    z = logits(E64, C64, bias)
    lse = log_sum_exp_rows(z)
    p = softmax_rows(z, lse)
    margin = tile_log_margin(z - lse[:, None], valid, tile_m, tile_n)
    skip = filtered_tiles(margin, filter_eps)
    for b, tt in zip(*np.nonzero(skip)):
        p[b * tile_m:(b + 1) * tile_m, tt * tile_n:(tt + 1) * tile_n] = 0.0
    G = logit_grad(p, lse, t, valid, scale, label_smoothing, z_loss)
    borderline = 0
    if filter_eps > 0:
        borderline = int((np.abs(margin - math.log(filter_eps)) < window).sum())
    return BackwardResult(G @ C64, G.T @ E64, int(skip.sum()), borderline, skip.size,
                          None if bias is None else G.sum(axis=0), margin)


@dataclass
class SampledResult:
    lse: np.ndarray  # [N], every row
    nll: np.ndarray  # [N]
    count: int
    loss: np.ndarray
    margin: np.ndarray  # [ceil(N/tile_m), ceil(V/tile_n)]
    filtered: int
    borderline: int
    rows: np.ndarray
    dE_rows: np.ndarray  # [len(rows), D]
    cols: np.ndarray
    dC_cols: np.ndarray  # [len(cols), D]
    dbias: Optional[np.ndarray] = None  # [V] when a bias is given and compute_cols


def sampled(E, C, targets, rows: Sequence[int], cols: Sequence[int], grad_out=1.0,
            ignore_index: int = -100, reduction: str = "mean", filter_eps: float = 2.0 ** -12,
            tile_m: int = 128, tile_n: int = 256, window: float = 2e-3,
            compute_cols: bool = True, bias=None, label_smoothing: float = 0.0,
            z_loss: float = 0.0) -> SampledResult:
    """The same definitions as ``forward``/``backward``, evaluated for large problems.

    The logits are materialised one row group at a time (rows are independent),
    so memory stays at ``ROW_GROUP * V`` doubles. Every row's LSE, every tile's
    skip decision and the loss are exact; dE is returned for the rows ``rows``
    and dC for the vocabulary rows ``cols`` (dC needs every row's softmax at those
    columns, so ``compute_cols`` makes this a full pass over all rows; with a bias
    that pass also gives every entry of dbias).
    """
    E64, C64, t = _f64(E), _f64(C), _i64(targets)
    N, V = E64.shape[0], C64.shape[0]
    bv = _bias64(bias, V)
    validate_targets(t, V, ignore_index)
    valid = t != ignore_index
    count = int(valid.sum())
    scale = row_scale(t, ignore_index, reduction, grad_out, count)
    rows = np.asarray(rows, dtype=np.int64)
    cols = np.asarray(cols, dtype=np.int64)
    if ROW_GROUP % tile_m:
        raise ValueError("ROW_GROUP must be a multiple of tile_m")

    lse = np.empty(N)
    zt = np.zeros(N)
    zs = np.zeros(N)
    nb, nt = -(-N // tile_m), -(-V // tile_n)
    margin = np.full((nb, nt), -np.inf)
    dE_rows = np.zeros((len(rows), E64.shape[1]))
    dC_cols = np.zeros((len(cols), E64.shape[1]))
    dbias = np.zeros(V) if (bv is not None and compute_cols) else None
    row_pos = {int(r): i for i, r in enumerate(rows)}
    ln_eps = math.log(filter_eps) if filter_eps > 0 else -math.inf

    for g in _row_groups(N):
        z = E64[g] @ C64.T
        if bv is not None:
            z += bv[None, :]
        l = log_sum_exp_rows(z)
        lse[g] = l
        zs[g] = z.sum(axis=1)
        tg, vg = t[g], valid[g]
        zt[g] = np.where(vg, z[np.arange(z.shape[0]), np.where(vg, tg, 0)], 0.0)
        m = tile_log_margin(z - l[:, None], vg, tile_m, tile_n)
        b0 = g.start // tile_m
        margin[b0:b0 + m.shape[0]] = m
        need_rows = [i for i in range(g.start, g.stop) if i in row_pos]
        if not compute_cols and not need_rows:
            continue
        p = softmax_rows(z, l)
        skip = filtered_tiles(m, filter_eps)
        for b, tt in zip(*np.nonzero(skip)):
            p[b * tile_m:(b + 1) * tile_m, tt * tile_n:(tt + 1) * tile_n] = 0.0
        G = logit_grad(p, l, tg, vg, scale[g], label_smoothing, z_loss)
        for i in need_rows:
            dE_rows[row_pos[i]] = G[i - g.start] @ C64
        if compute_cols:
            dC_cols += G[:, cols].T @ E64[g]
            if dbias is not None:
                dbias += G.sum(axis=0)
        del z, p, G

    nll = row_loss(lse, zt, zs, V, valid, label_smoothing, z_loss)
    skip_all = filtered_tiles(margin, filter_eps)
    borderline = int((np.abs(margin - ln_eps) < window).sum()) if filter_eps > 0 else 0
    return SampledResult(lse, nll, count, reduce_loss(nll, count, reduction), margin,
                         int(skip_all.sum()), borderline, rows, dE_rows, cols, dC_cols, dbias)


@dataclass
class RowBlockResult:
    rows: np.ndarray  # every row of the chosen blocks, ascending
    lse: np.ndarray
    nll: np.ndarray
    margin: np.ndarray  # [len(blocks), ceil(V/tile_n)]
    filtered: int  # skipped tiles among the chosen blocks
    dE: np.ndarray  # [len(rows), D]


def row_blocks(E, C, targets, blocks: Sequence[int], grad_out=1.0, ignore_index: int = -100,
               reduction: str = "mean", filter_eps: float = 2.0 ** -12, tile_m: int = 128,
               tile_n: int = 256, bias=None, label_smoothing: float = 0.0, z_loss: float = 0.0) -> RowBlockResult:
    """Exact results for whole row blocks of the tile grid.

    A tile's skip decision depends only on the rows of its own row block, and a
    row's dE depends only on its own logits and those decisions, so evaluating
    complete blocks gives their LSE, loss, decisions and dE exactly. The row
    count used by ``mean`` comes from all targets.
    """
    E64, C64, t = _f64(E), _f64(C), _i64(targets)
    N, V = E64.shape[0], C64.shape[0]
    bv = _bias64(bias, V)
    validate_targets(t, V, ignore_index)
    count = int((t != ignore_index).sum())
    scale_all = row_scale(t, ignore_index, reduction, grad_out, count)
    rows = np.concatenate([np.arange(b * tile_m, min((b + 1) * tile_m, N)) for b in sorted(blocks)])
    lse = np.empty(len(rows))
    nll = np.empty(len(rows))
    margins = []
    dE = np.zeros((len(rows), E64.shape[1]))
    filtered = 0
    pos = 0
    for b in sorted(blocks):
        rr = np.arange(b * tile_m, min((b + 1) * tile_m, N))
        z = E64[rr] @ C64.T
        if bv is not None:
            z += bv[None, :]
        l = log_sum_exp_rows(z)
        tb = t[rr]
        vb = tb != ignore_index
        m = tile_log_margin(z - l[:, None], vb, tile_m, tile_n)
        skip = filtered_tiles(m, filter_eps)
        filtered += int(skip.sum())
        p = softmax_rows(z, l)
        for tt in np.flatnonzero(skip[0]):
            p[:, tt * tile_n:(tt + 1) * tile_n] = 0.0
        G = logit_grad(p, l, tb, vb, scale_all[rr], label_smoothing, z_loss)
        zt = np.where(vb, z[np.arange(len(rr)), np.where(vb, tb, 0)], 0.0)
        lse[pos:pos + len(rr)] = l
        nll[pos:pos + len(rr)] = row_loss(l, zt, z.sum(axis=1), V, vb, label_smoothing, z_loss)
        dE[pos:pos + len(rr)] = G @ C64
        margins.append(m[0])
        pos += len(rr)
    return RowBlockResult(rows, lse, nll, np.array(margins), filtered, dE)


@dataclass
class VocabTileResult:
    tiles: np.ndarray  # the vocabulary tiles evaluated, ascending
    cols: np.ndarray  # their columns, tile after tile
    margin: np.ndarray  # [ceil(N/tile_m), len(tiles)]
    filtered: int  # skipped (row block, tile) pairs among the chosen tiles
    dC: np.ndarray  # [len(cols), D]
    dbias: Optional[np.ndarray] = None  # [len(cols)] when a bias is given


def vocab_tiles(E, C, targets, lse, tiles: Sequence[int], grad_out=1.0, ignore_index: int = -100,
                reduction: str = "mean", filter_eps: float = 2.0 ** -12, tile_m: int = 128, tile_n: int = 256,
                bias=None, label_smoothing: float = 0.0, z_loss: float = 0.0) -> VocabTileResult:
    """Exact dC (and dbias) rows of whole vocabulary tiles, given every row's LSE.

    Column v of the logit gradient G needs only z[:, v], each row's LSE and the skip
    decisions of the tiles that hold v; a tile's decision reads only its own rows and
    columns (mlx-cross-entropy README, "How it works" item 2). So dC = G^T E and
    dbias = sum_r G[r, :] restricted to whole tiles follow from E, the rows of C in
    those tiles and the LSE vector of the same problem (from ``forward`` or
    ``sampled``), with the per-row G of ``logit_grad`` (Loss functions explainer,
    "How it works" items 2 and 3):
    G[r, v] = scale_r ((1 + 2 zl LSE_r) p~[r, v] - (1 - ls) [v = t_r] - ls / V).
    """
    E64, C64, t = _f64(E), _f64(C), _i64(targets)
    N, V = E64.shape[0], C64.shape[0]
    bv = _bias64(bias, V)
    validate_targets(t, V, ignore_index)
    lse = _f64(lse).reshape(-1)
    if lse.shape[0] != N:
        raise ValueError(f"lse must have {N} entries, got {lse.shape[0]}")
    tiles = np.asarray(sorted(set(int(x) for x in tiles)), dtype=np.int64)
    nt = -(-V // tile_n)
    if tiles.size and (tiles[0] < 0 or tiles[-1] >= nt):
        raise ValueError(f"vocabulary tiles must lie in [0, {nt})")
    if ROW_GROUP % tile_m:
        raise ValueError("ROW_GROUP must be a multiple of tile_m")
    cols = np.concatenate([np.arange(k * tile_n, min((k + 1) * tile_n, V)) for k in tiles]) if tiles.size \
        else np.zeros(0, dtype=np.int64)
    valid = t != ignore_index
    count = int(valid.sum())
    scale = row_scale(t, ignore_index, reduction, grad_out, count)
    Cc = C64[cols]
    nb = -(-N // tile_m)
    margin = np.full((nb, len(tiles)), -np.inf)
    dC = np.zeros((len(cols), E64.shape[1]))
    dbias = np.zeros(len(cols)) if bv is not None else None
    col_of = {int(v): j for j, v in enumerate(cols)}
    for g in _row_groups(N):
        z = E64[g] @ Cc.T
        if bv is not None:
            z += bv[cols][None, :]
        l = lse[g]
        vg, tg = valid[g], t[g]
        m = tile_log_margin(z - l[:, None], vg, tile_m, tile_n)
        b0 = g.start // tile_m
        margin[b0:b0 + m.shape[0]] = m
        p = softmax_rows(z, l)
        skip = filtered_tiles(m, filter_eps)
        for b, k in zip(*np.nonzero(skip)):
            p[b * tile_m:(b + 1) * tile_m, k * tile_n:(k + 1) * tile_n] = 0.0
        sc = scale[g]
        G = (sc * (1.0 + 2.0 * z_loss * l))[:, None] * p
        for i in np.flatnonzero(vg):
            j = col_of.get(int(tg[i]))
            if j is not None:
                G[i, j] -= sc[i] * (1.0 - label_smoothing)
        if label_smoothing:
            G[vg] -= (sc[vg] * (label_smoothing / V))[:, None]
        dC += G.T @ E64[g]
        if dbias is not None:
            dbias += G.sum(axis=0)
        del z, p, G
    skip_all = filtered_tiles(margin, filter_eps)
    return VocabTileResult(tiles, cols, margin, int(skip_all.sum()), dC, dbias)
