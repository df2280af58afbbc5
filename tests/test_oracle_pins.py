"""Pins of the fp64 oracle to facts fixed by the pages and by the mathematics (CPU only).

Each test is chosen so that a plausible slip in the oracle (a dropped max shift,
a wrong sign, a missing onehot, a transposed operand, a wrong normaliser, a wrong
skip rule) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import cce_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand_problem(N=24, D=16, V=200, seed=0, ignore=(3, 7), scale=1.0):
    rng = np.random.default_rng(seed)
    E = rng.standard_normal((N, D))
    C = rng.standard_normal((V, D)) * scale
    t = rng.integers(0, V, N)
    for r in ignore:
        t[r] = -100
    return E, C, t


# --- values the pages print -------------------------------------------------------------------

def test_zero_logits_give_ln_classes():
    g = _golden("zero_logits_1000_classes.json")
    K = g["classes"]
    E = np.zeros((1, 8))
    C = np.zeros((K, 8))  # C = 0 -> every logit is 0
    t = np.array([g["target"]])
    f = O.forward(E, C, t)
    assert abs(float(f.loss) - math.log(K)) < 1e-12
    assert round(float(f.loss), 4) == g["printed_value_4dp"]
    # gradient of uniform softmax: scale * (1/K - onehot), here via dC = G^T E = 0 and dE = G C = 0,
    # so check the logit gradient through an identity classifier instead
    E2 = np.zeros((1, K))
    C2 = np.eye(K)
    b = O.backward(E2, C2, t, filter_eps=0.0)
    expect = np.full(K, 1.0 / K)
    expect[g["target"]] -= 1.0
    np.testing.assert_allclose(b.dE[0], expect, rtol=0, atol=1e-15)


def test_large_logit_stays_finite():
    g = _golden("large_logit_stays_finite.json")
    z = np.array([g["logits"]])
    f = O.forward(z, np.eye(z.shape[1]), np.array([g["target"]]))
    assert np.isfinite(f.loss) and float(f.loss) == g["expected_loss"]
    b = O.backward(z, np.eye(z.shape[1]), np.array([g["target"]]), filter_eps=0.0)
    assert np.isfinite(b.dE).all()
    # p = [1, e^-1e4]: gradient at the logits is [1, -1] (target 1) up to e^-1e4
    np.testing.assert_allclose(b.dE[0], [1.0, -1.0], atol=1e-300)


@pytest.mark.parametrize("smoothing", ["page", 0.0])
def test_explainer_worked_example_finite_differences(smoothing):
    g = _golden("explainer_worked_logits.json")
    ls = g["label_smoothing"] if smoothing == "page" else smoothing
    n, k = g["n"], g["k"]
    z = np.array([((i * 37 % 13) - 6) * 0.8 for i in range(n * k)], dtype=np.float64).reshape(n, k)
    t = np.array(g["targets"])
    C = np.eye(k)  # E @ C.T = E, so E plays the logits
    b = O.backward(z, C, t, ignore_index=g["ignore_index"], filter_eps=0.0, label_smoothing=ls)
    h, tol = g["fd_step"], g["fd_tolerance"]
    for i in g["fd_entries"]:
        zp, zm = z.copy(), z.copy()
        zp.flat[i] += h
        zm.flat[i] -= h
        lp = float(O.forward(zp, C, t, g["ignore_index"], label_smoothing=ls).loss)
        lm = float(O.forward(zm, C, t, g["ignore_index"], label_smoothing=ls).loss)
        assert abs((lp - lm) / (2 * h) - b.dE.flat[i]) < tol
    # the ignored row has zero gradient and the mean divides by 3 non-ignored rows
    assert (b.dE[2] == 0).all()
    f = O.forward(z, C, t)
    assert f.count == 3


# --- closed forms and invariants ----------------------------------------------------------------

def test_softmax_rows_sum_to_one():
    E, C, t = _rand_problem(scale=3.0)
    z = O.logits(E, C)
    p = O.softmax_rows(z, O.log_sum_exp_rows(z))
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)


def test_lse_matches_direct_definition_and_is_shift_stable():
    E, C, t = _rand_problem()
    z = O.logits(E, C)
    direct = np.log(np.exp(z).sum(axis=1))
    np.testing.assert_allclose(O.log_sum_exp_rows(z), direct, rtol=1e-13)
    np.testing.assert_allclose(O.log_sum_exp_rows(z + 800.0), direct + 800.0, rtol=1e-13)


def test_loss_is_lse_minus_target_logit():
    E, C, t = _rand_problem()
    f = O.forward(E, C, t, reduction="none")
    z = E @ C.T
    for r in range(len(t)):
        if t[r] == -100:
            assert f.loss[r] == 0.0
        else:
            lse = math.log(sum(math.exp(v) for v in z[r]))
            assert abs(f.loss[r] - (lse - z[r, t[r]])) < 1e-11


def test_ignored_rows_exact_zero_and_independent():
    E, C, t = _rand_problem()
    for red in ("mean", "sum", "none"):
        g = np.random.default_rng(1).standard_normal(len(t)) if red == "none" else 1.0
        b = O.backward(E, C, t, grad_out=g, reduction=red, filter_eps=2.0 ** -12, tile_m=8, tile_n=32)
        for r in (3, 7):
            assert (b.dE[r] == 0.0).all() and not np.signbit(b.dE[r]).any()
        E2 = E.copy()
        E2[3] = 1e3 * np.random.default_rng(2).standard_normal(E.shape[1])
        b2 = O.backward(E2, C, t, grad_out=g, reduction=red, filter_eps=2.0 ** -12, tile_m=8, tile_n=32)
        f, f2 = O.forward(E, C, t, reduction=red), O.forward(E2, C, t, reduction=red)
        assert np.array_equal(f.loss, f2.loss)
        assert np.array_equal(b.dC, b2.dC)
        assert b.filtered == b2.filtered


@pytest.mark.parametrize("reduction", ["mean", "sum", "none"])
def test_finite_differences(reduction):
    N, D, V = 8, 16, 64
    E, C, t = _rand_problem(N, D, V, seed=3, ignore=(5,))
    g = np.random.default_rng(4).standard_normal(N) if reduction == "none" else 1.0

    def L(E_, C_):
        f = O.forward(E_, C_, t, reduction=reduction)
        return float(np.sum(np.asarray(f.loss) * g)) if reduction == "none" else float(f.loss)

    b = O.backward(E, C, t, grad_out=g, reduction=reduction, filter_eps=0.0)
    h = 1e-5
    rng = np.random.default_rng(5)
    for _ in range(12):
        i, j = rng.integers(0, N), rng.integers(0, D)
        Ep, Em = E.copy(), E.copy()
        Ep[i, j] += h
        Em[i, j] -= h
        fd = (L(Ep, C) - L(Em, C)) / (2 * h)
        assert abs(fd - b.dE[i, j]) <= 1e-6 * max(1.0, abs(fd))
        v, j = rng.integers(0, V), rng.integers(0, D)
        Cp, Cm = C.copy(), C.copy()
        Cp[v, j] += h
        Cm[v, j] -= h
        fd = (L(E, Cp) - L(E, Cm)) / (2 * h)
        assert abs(fd - b.dC[v, j]) <= 1e-6 * max(1.0, abs(fd))


@pytest.mark.parametrize("reduction", ["mean", "sum", "none"])
def test_matches_torch_cross_entropy_float64(reduction):
    """Library special case: materialised logits + F.cross_entropy with autograd (filter off)."""
    E, C, t = _rand_problem(N=40, D=24, V=300, seed=6, ignore=(0, 11, 39))
    Et = torch.tensor(E, requires_grad=True)
    Ct = torch.tensor(C, requires_grad=True)
    tt = torch.tensor(t)
    out = torch.nn.functional.cross_entropy(Et @ Ct.T, tt, ignore_index=-100, reduction=reduction)
    g = np.random.default_rng(7).standard_normal(len(t)) if reduction == "none" else 1.0
    (out * torch.tensor(g)).sum().backward()
    f = O.forward(E, C, t, reduction=reduction)
    b = O.backward(E, C, t, grad_out=g, reduction=reduction, filter_eps=0.0)
    np.testing.assert_allclose(np.asarray(f.loss), out.detach().numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(b.dE, Et.grad.numpy(), rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(b.dC, Ct.grad.numpy(), rtol=1e-10, atol=1e-14)


def test_mean_with_every_row_ignored_is_zero():
    E, C, t = _rand_problem(N=4, ignore=())
    t[:] = -100
    f = O.forward(E, C, t)
    b = O.backward(E, C, t)
    assert float(f.loss) == 0.0 and f.count == 0
    assert not b.dE.any() and not b.dC.any()


def test_reduction_relations_and_linearity():
    E, C, t = _rand_problem(seed=8)
    fm, fs, fn = (O.forward(E, C, t, reduction=r) for r in ("mean", "sum", "none"))
    assert abs(float(fm.loss) - float(fs.loss) / fm.count) < 1e-12
    assert abs(float(fn.loss.sum()) - float(fs.loss)) < 1e-12
    b1 = O.backward(E, C, t, grad_out=1.0, reduction="sum", filter_eps=0.0)
    b3 = O.backward(E, C, t, grad_out=-2.5, reduction="sum", filter_eps=0.0)
    np.testing.assert_allclose(b3.dE, -2.5 * b1.dE, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(b3.dC, -2.5 * b1.dC, rtol=1e-13, atol=1e-15)
    bm = O.backward(E, C, t, grad_out=1.0, reduction="mean", filter_eps=0.0)
    np.testing.assert_allclose(bm.dE * fm.count, b1.dE, rtol=1e-12, atol=1e-15)
    ones = np.ones(len(t))
    bn = O.backward(E, C, t, grad_out=ones, reduction="none", filter_eps=0.0)
    np.testing.assert_allclose(bn.dC, b1.dC, rtol=1e-12, atol=1e-15)


def test_targets_outside_vocabulary_are_rejected():
    E, C, t = _rand_problem()
    t[4] = C.shape[0]
    with pytest.raises(ValueError):
        O.forward(E, C, t)
    t[4] = -7
    with pytest.raises(ValueError):
        O.backward(E, C, t)


# --- the skip rule -------------------------------------------------------------------------------

def _brute_force_skipped(E, C, t, eps, tm, tn, ignore=-100):
    """Tile skipped iff every non-ignored softmax entry in it is below eps (pure Python)."""
    N, V = len(t), len(C)
    probs = []
    for r in range(N):
        z = [sum(E[r][d] * C[v][d] for d in range(len(E[r]))) for v in range(V)]
        m = max(z)
        s = sum(math.exp(x - m) for x in z)
        probs.append([math.exp(x - m) / s for x in z])
    skipped = 0
    for b0 in range(0, N, tm):
        for v0 in range(0, V, tn):
            keep = any(probs[r][v] >= eps for r in range(b0, min(b0 + tm, N)) if t[r] != ignore
                       for v in range(v0, min(v0 + tn, V)))
            skipped += not keep
    return skipped


@pytest.mark.parametrize("eps", [2.0 ** -12, 2.0 ** -6, 0.02])
def test_skip_count_matches_brute_force(eps):
    E, C, t = _rand_problem(N=21, D=6, V=90, seed=9, ignore=(2, 3, 4, 5, 6))
    E = E * 2.5  # spread the softmax so that tiles fall on both sides of eps
    b = O.backward(E, C, t, filter_eps=eps, tile_m=4, tile_n=16)
    assert b.filtered == _brute_force_skipped(E.tolist(), C.tolist(), t.tolist(), eps, 4, 16)
    assert 0 < b.filtered < b.n_tiles


def test_skip_rule_limits_and_monotonicity():
    E, C, t = _rand_problem(N=32, D=8, V=256, seed=10)
    E = E * 2.0
    full = O.backward(E, C, t, filter_eps=0.0, tile_m=8, tile_n=32)
    assert full.filtered == 0
    ref = O.backward(E, C, t, filter_eps=-1.0, tile_m=8, tile_n=32)
    assert np.array_equal(full.dE, ref.dE)
    counts = [O.backward(E, C, t, filter_eps=e, tile_m=8, tile_n=32).filtered
              for e in (1e-9, 2.0 ** -12, 1e-3, 1e-2, 0.1, 0.5)]
    assert counts == sorted(counts)
    # eps above 1 skips every tile: only the onehot term is left
    allskip = O.backward(E, C, t, filter_eps=2.0, tile_m=8, tile_n=32)
    assert allskip.filtered == allskip.n_tiles
    valid = t != -100
    scale = np.where(valid, 1.0 / valid.sum(), 0.0)
    dE = np.zeros_like(E)
    dC = np.zeros_like(C)
    for r in np.flatnonzero(valid):
        dE[r] = -scale[r] * C[t[r]]
        dC[t[r]] -= scale[r] * E[r]
    np.testing.assert_allclose(allskip.dE, dE, rtol=1e-13, atol=1e-16)
    np.testing.assert_allclose(allskip.dC, dC, rtol=1e-13, atol=1e-16)


def test_skipping_changes_gradient_by_at_most_the_skipped_mass():
    E, C, t = _rand_problem(N=32, D=8, V=256, seed=11)
    E = E * 2.0
    eps = 2.0 ** -6
    full = O.backward(E, C, t, filter_eps=0.0, tile_m=8, tile_n=32)
    filt = O.backward(E, C, t, filter_eps=eps, tile_m=8, tile_n=32)
    assert filt.filtered > 0
    # each skipped entry had p < eps, so |dE_r difference| <= scale * eps * sum_v |C_v|
    valid = t != -100
    bound = (1.0 / valid.sum()) * eps * np.abs(C).sum(axis=0)
    assert (np.abs(full.dE - filt.dE) <= bound[None, :] + 1e-15).all()


def test_vocab_tile_relabelling_permutes_dC():
    E, C, t = _rand_problem(N=16, D=8, V=128, seed=12, ignore=(1,))
    E = E * 2.0
    tn = 32
    perm_tiles = [2, 0, 3, 1]
    perm = np.concatenate([np.arange(p * tn, (p + 1) * tn) for p in perm_tiles])
    inv = np.argsort(perm)
    t2 = np.where(t == -100, -100, inv[np.where(t == -100, 0, t)])
    C2 = C[perm]
    a = O.backward(E, C, t, filter_eps=2.0 ** -8, tile_m=8, tile_n=tn)
    b = O.backward(E, C2, t2, filter_eps=2.0 ** -8, tile_m=8, tile_n=tn)
    assert a.filtered == b.filtered
    np.testing.assert_allclose(b.dE, a.dE, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(b.dC, a.dC[perm], rtol=1e-12, atol=1e-15)
    fa, fb = O.forward(E, C, t), O.forward(E, C2, t2)
    assert abs(float(fa.loss) - float(fb.loss)) < 1e-13


def test_sampled_evaluation_agrees_with_full(monkeypatch):
    monkeypatch.setattr(O, "ROW_GROUP", 16)
    E, C, t = _rand_problem(N=50, D=12, V=300, seed=13, ignore=(0, 17, 18))
    E = E * 2.0
    rows, cols = [0, 5, 17, 49], [0, 7, 150, 299]
    for red in ("mean", "none"):
        g = np.random.default_rng(14).standard_normal(50) if red == "none" else 0.7
        full_f = O.forward(E, C, t, reduction=red)
        full_b = O.backward(E, C, t, grad_out=g, reduction=red, filter_eps=2.0 ** -8, tile_m=8, tile_n=64)
        s = O.sampled(E, C, t, rows, cols, grad_out=g, reduction=red, filter_eps=2.0 ** -8, tile_m=8, tile_n=64)
        np.testing.assert_allclose(s.lse, full_f.lse, rtol=1e-13)
        np.testing.assert_allclose(np.asarray(s.loss), np.asarray(full_f.loss), rtol=1e-12, atol=1e-14)
        assert s.filtered == full_b.filtered
        np.testing.assert_allclose(s.dE_rows, full_b.dE[rows], rtol=1e-11, atol=1e-14)
        np.testing.assert_allclose(s.dC_cols, full_b.dC[cols], rtol=1e-11, atol=1e-14)


def test_row_block_evaluation_agrees_with_full():
    E, C, t = _rand_problem(N=40, D=12, V=300, seed=15, ignore=(0, 17, 18))
    E = E * 2.0
    full = O.backward(E, C, t, grad_out=0.5, reduction="mean", filter_eps=2.0 ** -8, tile_m=8, tile_n=64)
    f = O.forward(E, C, t)
    rb = O.row_blocks(E, C, t, [4, 1], grad_out=0.5, reduction="mean", filter_eps=2.0 ** -8, tile_m=8, tile_n=64)
    assert list(rb.rows) == list(range(8, 16)) + list(range(32, 40))
    np.testing.assert_allclose(rb.lse, f.lse[rb.rows], rtol=1e-13)
    np.testing.assert_allclose(rb.nll, f.nll[rb.rows], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(rb.dE, full.dE[rb.rows], rtol=1e-11, atol=1e-14)
    margin = O.tile_log_margin(O.logits(E, C) - f.lse[:, None], t != -100, 8, 64)
    assert rb.filtered == int(O.filtered_tiles(margin[[1, 4]], 2.0 ** -8).sum())


# --- classifier bias (mlx-cross-entropy README, "API" table: bias [V]) -------------------------

@pytest.mark.parametrize("reduction", ["mean", "sum", "none"])
def test_bias_matches_torch_linear_cross_entropy_float64(reduction):
    """Library special case: F.linear(e, c, bias) + F.cross_entropy with autograd (filter off)."""
    E, C, t = _rand_problem(N=40, D=24, V=300, seed=21, ignore=(0, 11, 39))
    bias = np.random.default_rng(22).standard_normal(300) * 2.0
    Et = torch.tensor(E, requires_grad=True)
    Ct = torch.tensor(C, requires_grad=True)
    bt = torch.tensor(bias, requires_grad=True)
    tt = torch.tensor(t)
    out = torch.nn.functional.cross_entropy(torch.nn.functional.linear(Et, Ct, bt), tt, ignore_index=-100,
                                            reduction=reduction)
    g = np.random.default_rng(23).standard_normal(len(t)) if reduction == "none" else 1.0
    (out * torch.tensor(g)).sum().backward()
    f = O.forward(E, C, t, reduction=reduction, bias=bias)
    b = O.backward(E, C, t, grad_out=g, reduction=reduction, filter_eps=0.0, bias=bias)
    np.testing.assert_allclose(np.asarray(f.loss), out.detach().numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(b.dE, Et.grad.numpy(), rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(b.dC, Ct.grad.numpy(), rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(b.dbias, bt.grad.numpy(), rtol=1e-10, atol=1e-14)


def test_bias_finite_differences():
    N, D, V = 8, 16, 64
    E, C, t = _rand_problem(N, D, V, seed=24, ignore=(2,))
    bias = np.random.default_rng(25).standard_normal(V)
    b = O.backward(E, C, t, filter_eps=0.0, bias=bias)
    h = 1e-5
    for v in (0, 5, 31, 63, int(t[0])):
        bp, bm = bias.copy(), bias.copy()
        bp[v] += h
        bm[v] -= h
        fd = (float(O.forward(E, C, t, bias=bp).loss) - float(O.forward(E, C, t, bias=bm).loss)) / (2 * h)
        assert abs(fd - b.dbias[v]) <= 1e-7 * max(1.0, abs(fd))


def test_bias_shift_invariance_and_zero_sum_gradient():
    """Softmax is shift invariant: a constant added to every bias entry changes neither the loss
    nor any gradient, and with filtering off dbias sums to zero (each row of p - y sums to 0)."""
    E, C, t = _rand_problem(N=20, D=8, V=96, seed=26, ignore=(4,))
    bias = np.random.default_rng(27).standard_normal(96)
    f0 = O.forward(E, C, t, bias=bias)
    f1 = O.forward(E, C, t, bias=bias + 3.5)
    b0 = O.backward(E, C, t, filter_eps=0.0, bias=bias)
    b1 = O.backward(E, C, t, filter_eps=0.0, bias=bias + 3.5)
    assert abs(float(f0.loss) - float(f1.loss)) < 1e-12
    np.testing.assert_allclose(b0.dE, b1.dE, atol=1e-13)
    np.testing.assert_allclose(b0.dbias, b1.dbias, atol=1e-13)
    assert abs(b0.dbias.sum()) < 1e-12
    # and a zero bias is the same as no bias
    fz = O.forward(E, C, t, bias=np.zeros(96))
    assert float(fz.loss) == float(O.forward(E, C, t).loss)


def test_bias_only_model_has_closed_form():
    """E = 0: every row's logits are the bias, so each row's loss is log-sum-exp(bias) - bias[t_r]
    (computed here with math.fsum, not the oracle's routine) and dbias sums softmax(bias) - onehot
    over the valid rows, divided by their count."""
    V = 50
    bias = np.random.default_rng(28).standard_normal(V) * 3.0
    t = np.array([3, 3, 17, -100, 49])
    E = np.zeros((5, 4))
    C = np.random.default_rng(29).standard_normal((V, 4))
    m = max(bias)
    lse = m + math.log(math.fsum(math.exp(x - m) for x in bias))
    want = math.fsum(lse - bias[k] for k in (3, 3, 17, 49)) / 4
    assert abs(float(O.forward(E, C, t, bias=bias).loss) - want) < 1e-12
    p = [math.exp(x - lse) for x in bias]
    want_db = [(4 * p[v] - sum(1 for k in (3, 3, 17, 49) if k == v)) / 4 for v in range(V)]
    np.testing.assert_allclose(O.backward(E, C, t, filter_eps=0.0, bias=bias).dbias, want_db, atol=1e-13)


def test_bias_sampled_and_row_blocks_agree_with_full(monkeypatch):
    monkeypatch.setattr(O, "ROW_GROUP", 16)
    E, C, t = _rand_problem(N=48, D=12, V=256, seed=30, ignore=(0, 17))
    E = E * 2.0
    bias = np.random.default_rng(31).standard_normal(256)
    full_f = O.forward(E, C, t, bias=bias)
    full_b = O.backward(E, C, t, grad_out=0.7, filter_eps=2.0 ** -8, tile_m=8, tile_n=64, bias=bias)
    s = O.sampled(E, C, t, [1, 40], [0, 200], grad_out=0.7, filter_eps=2.0 ** -8, tile_m=8, tile_n=64, bias=bias)
    np.testing.assert_allclose(s.lse, full_f.lse, rtol=1e-13)
    np.testing.assert_allclose(s.dE_rows, full_b.dE[[1, 40]], rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(s.dC_cols, full_b.dC[[0, 200]], rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(s.dbias, full_b.dbias, rtol=1e-11, atol=1e-14)
    rb = O.row_blocks(E, C, t, [2], grad_out=0.7, filter_eps=2.0 ** -8, tile_m=8, tile_n=64, bias=bias)
    np.testing.assert_allclose(rb.dE, full_b.dE[16:24], rtol=1e-11, atol=1e-14)


def test_sampled_with_skips_in_every_row_group(monkeypatch):
    """Several row groups, each with skipped tiles, with and without a bias: the group loop's
    per-tile bookkeeping must not disturb the next group."""
    monkeypatch.setattr(O, "ROW_GROUP", 16)
    rng = np.random.default_rng(32)
    N, D, V = 64, 32, 2048
    C = rng.standard_normal((V, D)) / np.sqrt(D)
    t = rng.integers(0, V, N)
    t[5] = -100
    E = 24.0 * C[np.where(t >= 0, t, 0)] + rng.standard_normal((N, D))  # peaked: most tiles skipped
    for bias in (None, np.random.default_rng(33).standard_normal(V) * 0.5):
        full = O.backward(E, C, t, filter_eps=2.0 ** -12, tile_m=8, tile_n=64, bias=bias)
        lse = O.forward(E, C, t, bias=bias).lse
        skip = O.filtered_tiles(O.tile_log_margin(O.logits(E, C, bias) - lse[:, None], t != -100, 8, 64), 2.0 ** -12)
        assert all(skip[2 * k:2 * k + 2].any() for k in range(4)), "every 16-row group must hold a skipped tile"
        s = O.sampled(E, C, t, [3, 60], [1, 2000], filter_eps=2.0 ** -12, tile_m=8, tile_n=64, bias=bias)
        assert s.filtered == full.filtered
        np.testing.assert_allclose(s.lse, lse, rtol=1e-13)
        np.testing.assert_allclose(s.dE_rows, full.dE[[3, 60]], rtol=1e-11, atol=1e-14)
        np.testing.assert_allclose(s.dC_cols, full.dC[[1, 2000]], rtol=1e-11, atol=1e-14)



# --- label smoothing and z-loss (Loss functions explainer: How it works item 3; Implementation
# notes: z-loss) ---------------------------------------------------------------------------------

@pytest.mark.parametrize("reduction", ["mean", "sum", "none"])
def test_smoothing_and_z_loss_match_torch_float64(reduction):
    """Library special case: F.cross_entropy(label_smoothing=ls) (torch spreads ls over all V
    classes, the page's definition) plus zl * logsumexp^2 per non-ignored token, with autograd."""
    E, C, t = _rand_problem(N=40, D=24, V=300, seed=41, ignore=(0, 11, 39))
    bias = np.random.default_rng(42).standard_normal(300)
    ls, zl = 0.1, 1e-2
    Et = torch.tensor(E, requires_grad=True)
    Ct = torch.tensor(C, requires_grad=True)
    bt = torch.tensor(bias, requires_grad=True)
    tt = torch.tensor(t)
    z = torch.nn.functional.linear(Et, Ct, bt)
    ce = torch.nn.functional.cross_entropy(z, tt, ignore_index=-100, reduction="none", label_smoothing=ls)
    valid = (tt != -100).double()
    per_tok = (ce + zl * torch.logsumexp(z, dim=1) ** 2) * valid
    out = {"mean": per_tok.sum() / valid.sum(), "sum": per_tok.sum(), "none": per_tok}[reduction]
    g = np.random.default_rng(43).standard_normal(len(t)) if reduction == "none" else 1.0
    (out * torch.tensor(g)).sum().backward()
    f = O.forward(E, C, t, reduction=reduction, bias=bias, label_smoothing=ls, z_loss=zl)
    b = O.backward(E, C, t, grad_out=g, reduction=reduction, filter_eps=0.0, bias=bias, label_smoothing=ls,
                   z_loss=zl)
    np.testing.assert_allclose(np.asarray(f.loss), out.detach().numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(b.dE, Et.grad.numpy(), rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(b.dC, Ct.grad.numpy(), rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(b.dbias, bt.grad.numpy(), rtol=1e-10, atol=1e-14)


@pytest.mark.parametrize("reduction", ["mean", "none"])
def test_smoothing_and_z_loss_finite_differences(reduction):
    N, D, V = 8, 16, 64
    E, C, t = _rand_problem(N, D, V, seed=44, ignore=(5,))
    ls, zl = 0.2, 0.05
    g = np.random.default_rng(45).standard_normal(N) if reduction == "none" else 1.0

    def L(E_, C_):
        f = O.forward(E_, C_, t, reduction=reduction, label_smoothing=ls, z_loss=zl)
        return float(np.sum(np.asarray(f.loss) * g)) if reduction == "none" else float(f.loss)

    b = O.backward(E, C, t, grad_out=g, reduction=reduction, filter_eps=0.0, label_smoothing=ls, z_loss=zl)
    h = 1e-5
    rng = np.random.default_rng(46)
    for _ in range(10):
        i, j = rng.integers(0, N), rng.integers(0, D)
        Ep, Em = E.copy(), E.copy()
        Ep[i, j] += h
        Em[i, j] -= h
        assert abs((L(Ep, C) - L(Em, C)) / (2 * h) - b.dE[i, j]) <= 1e-6 * max(1.0, abs(b.dE[i, j]))
        v, j = rng.integers(0, V), rng.integers(0, D)
        Cp, Cm = C.copy(), C.copy()
        Cp[v, j] += h
        Cm[v, j] -= h
        assert abs((L(E, Cp) - L(E, Cm)) / (2 * h) - b.dC[v, j]) <= 1e-6 * max(1.0, abs(b.dC[v, j]))


def test_full_smoothing_and_pure_z_loss_closed_forms():
    """ls = 1: the target is uniform, so each token's loss is LSE - mean_v z_v; zl alone adds
    zl * LSE^2. Both written out with math.fsum over the logits."""
    E, C, t = _rand_problem(N=6, D=5, V=40, seed=47, ignore=(2,))
    z = E @ C.T
    want_u, want_z = [], []
    for r in range(6):
        if t[r] == -100:
            continue
        m = max(z[r])
        lse = m + math.log(math.fsum(math.exp(x - m) for x in z[r]))
        want_u.append(lse - math.fsum(z[r]) / 40)
        want_z.append(lse - z[r][t[r]] + 0.3 * lse * lse)
    assert abs(float(O.forward(E, C, t, label_smoothing=1.0).loss) - math.fsum(want_u) / 5) < 1e-12
    assert abs(float(O.forward(E, C, t, z_loss=0.3).loss) - math.fsum(want_z) / 5) < 1e-12


def test_skipping_keeps_the_smoothing_term():
    """Tile skipping removes only (1 + 2 zl LSE) p; the ls / V part of the target, which does not
    depend on the logits, survives in every tile: a fully skipped problem still carries it."""
    E, C, t = _rand_problem(N=16, D=8, V=128, seed=48, ignore=())
    ls, zl = 0.1, 1e-3
    b_all = O.backward(E, C, t, filter_eps=2.0, tile_m=8, tile_n=64, label_smoothing=ls, z_loss=zl)  # eps > 1
    assert b_all.filtered == b_all.n_tiles
    scale = 1.0 / 16
    # G = -scale ((1 - ls) onehot + ls / V) exactly, so dC_v = -scale sum_r ((1-ls)[t_r = v] + ls/V) E_r
    G = np.full((16, 128), -scale * ls / 128)
    G[np.arange(16), t] -= scale * (1 - ls)
    np.testing.assert_allclose(b_all.dC, G.T @ E, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(b_all.dE, G @ C, rtol=1e-12, atol=1e-15)


def test_vocab_tile_evaluation_agrees_with_full(monkeypatch):
    """dC and dbias rows of whole vocabulary tiles from the LSE vector equal the full evaluation's,
    with skipped tiles among the chosen ones, a ragged last tile, a bias, smoothing and z-loss."""
    monkeypatch.setattr(O, "ROW_GROUP", 16)
    rng = np.random.default_rng(34)
    N, D, V, tn = 56, 128, 1000, 64  # 16 vocabulary tiles, the last one 40 columns wide
    C = rng.standard_normal((V, D)) / np.sqrt(D)
    t = rng.integers(0, V, N)
    t[[4, 33]] = -100
    t[:8] = rng.integers(0, 64, 8)  # some targets inside tile 0
    E = 18.0 * C[np.where(t >= 0, t, 0)] + rng.standard_normal((N, D))
    bias = rng.standard_normal(V) * 0.3
    kw = dict(filter_eps=2.0 ** -12, tile_m=8, tile_n=tn, bias=bias, label_smoothing=0.1, z_loss=1e-3)
    tiles = [15, 0, 7, 3]
    for red in ("mean", "none"):
        g = rng.standard_normal(N) if red == "none" else 0.7
        f = O.forward(E, C, t, reduction=red, bias=bias, label_smoothing=0.1, z_loss=1e-3)
        full = O.backward(E, C, t, grad_out=g, reduction=red, **kw)
        r = O.vocab_tiles(E, C, t, f.lse, tiles, grad_out=g, reduction=red, **kw)
        assert list(r.tiles) == sorted(tiles) and r.cols[-1] == V - 1 and len(r.cols) == 3 * tn + 40
        np.testing.assert_allclose(r.dC, full.dC[r.cols], rtol=1e-11, atol=1e-14)
        np.testing.assert_allclose(r.dbias, full.dbias[r.cols], rtol=1e-11, atol=1e-14)
        margin = O.tile_log_margin(O.logits(E, C, bias) - f.lse[:, None], t != -100, 8, tn)[:, sorted(tiles)]
        np.testing.assert_allclose(r.margin, margin, rtol=1e-13)
        skipped = int(O.filtered_tiles(margin, 2.0 ** -12).sum())
        assert r.filtered == skipped and 0 < skipped < margin.size
    # a wrong LSE (one row shifted) must change the result: the function really reads it
    lse_bad = f.lse.copy()
    lse_bad[10] += 0.5
    r_bad = O.vocab_tiles(E, C, t, lse_bad, tiles, grad_out=g, reduction="none", **kw)
    assert np.abs(r_bad.dC - r.dC).max() > 1e-6
