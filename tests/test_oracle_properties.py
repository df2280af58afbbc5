"""Randomised pins of the fp64 oracle (CPU only), over shapes the fixed-seed pins do not reach.

hypothesis draws the sizes (down to N = 1, D = 1, V = 1), the ignored rows, the reduction, the
loss variants, a bias or none, and the skip rule's tile and threshold. Every example is checked
against something other than the oracle:
  - torch float64 autograd on the materialised logits (the plain definition of the loss and of its
    gradients, with label smoothing over all V classes and the z-loss as the Loss functions
    explainer defines them), with skipping off;
  - the skip count by pure-Python enumeration of the softmax (mlx-cross-entropy README, How it
    works item 2), with skipping on.
The runs are derandomised, so the CPU suite sees the same examples every time.
"""
import math

import numpy as np
import pytest
import torch

from oracle import cce_oracle as O

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402

SETTINGS = settings(max_examples=60, deadline=None, derandomize=True, database=None)


@st.composite
def problems(draw):
    N = draw(st.integers(1, 12))
    D = draw(st.integers(1, 8))
    V = draw(st.integers(1, 40))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    rng = np.random.default_rng(seed)
    E = rng.standard_normal((N, D)) * draw(st.sampled_from([0.5, 1.0, 3.0]))
    C = rng.standard_normal((V, D))
    t = rng.integers(0, V, N)
    ignored = draw(st.lists(st.integers(0, N - 1), max_size=N, unique=True))
    t[ignored] = -100
    bias = rng.standard_normal(V) if draw(st.booleans()) else None
    return E, C, t, bias, rng


def _torch_reference(E, C, t, bias, reduction, ls, zl, g):
    Et = torch.tensor(E, requires_grad=True)
    Ct = torch.tensor(C, requires_grad=True)
    bt = torch.tensor(bias if bias is not None else np.zeros(len(C)), requires_grad=True)
    tt = torch.tensor(t)
    z = Et @ Ct.T + bt
    valid = tt != -100
    lse = torch.logsumexp(z, dim=1)
    safe_t = torch.where(valid, tt, torch.zeros_like(tt))
    z_t = z.gather(1, safe_t[:, None])[:, 0]
    # smoothed target (1 - ls) onehot + ls / V, and the z-loss zl * LSE^2, per non-ignored token
    per_tok = (lse - (1 - ls) * z_t - (ls / z.shape[1]) * z.sum(dim=1) + zl * lse ** 2) * valid.double()
    count = int(valid.sum())
    out = {"mean": per_tok.sum() / max(count, 1), "sum": per_tok.sum(), "none": per_tok}[reduction]
    (out * torch.tensor(g)).sum().backward()
    return out.detach().numpy(), Et.grad.numpy(), Ct.grad.numpy(), bt.grad.numpy()


@SETTINGS
@given(problems(), st.sampled_from(["mean", "sum", "none"]), st.sampled_from([0.0, 0.1, 1.0]),
       st.sampled_from([0.0, 1e-4, 0.05]))
def test_oracle_matches_torch_autograd_on_random_shapes(prob, reduction, ls, zl):
    E, C, t, bias, rng = prob
    g = rng.standard_normal(len(t)) if reduction == "none" else 1.5
    ref_loss, ref_dE, ref_dC, ref_db = _torch_reference(E, C, t, bias, reduction, ls, zl, g)
    f = O.forward(E, C, t, reduction=reduction, bias=bias, label_smoothing=ls, z_loss=zl)
    b = O.backward(E, C, t, grad_out=g, reduction=reduction, filter_eps=0.0, bias=bias, label_smoothing=ls,
                   z_loss=zl)
    np.testing.assert_allclose(np.asarray(f.loss), ref_loss, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(b.dE, ref_dE, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(b.dC, ref_dC, rtol=1e-10, atol=1e-12)
    if bias is not None:
        np.testing.assert_allclose(b.dbias, ref_db, rtol=1e-10, atol=1e-12)
    assert b.filtered == 0
    # rows of ignored tokens: exactly zero gradient
    assert not b.dE[t == -100].any()


def _brute_force_skipped(E, C, t, eps, tm, tn):
    N, V = len(t), len(C)
    probs = []
    for r in range(N):
        z = [sum(E[r][d] * C[v][d] for d in range(len(E[r]))) for v in range(V)]
        m = max(z)
        s = sum(math.exp(x - m) for x in z)
        probs.append([math.exp(x - m) / s for x in z])
    skipped = borderline = 0
    for b0 in range(0, N, tm):
        for v0 in range(0, V, tn):
            ps = [probs[r][v] for r in range(b0, min(b0 + tm, N)) if t[r] != -100 for v in range(v0, min(v0 + tn, V))]
            skipped += not any(p >= eps for p in ps)
            borderline += any(abs(math.log(p) - math.log(eps)) < 1e-9 for p in ps if p > 0)
    return skipped, borderline


@SETTINGS
@given(problems(), st.integers(1, 5), st.integers(1, 9), st.sampled_from([2.0 ** -12, 2.0 ** -6, 0.02, 0.2]))
def test_skip_count_matches_enumeration_on_random_shapes(prob, tm, tn, eps):
    E, C, t, _, _ = prob
    b = O.backward(E, C, t, filter_eps=eps, tile_m=tm, tile_n=tn)
    want, borderline = _brute_force_skipped(E.tolist(), C.tolist(), t.tolist(), eps, tm, tn)
    assert borderline == 0 or abs(b.filtered - want) <= borderline
    if borderline == 0:
        assert b.filtered == want
    assert b.n_tiles == -(-len(t) // tm) * -(-len(C) // tn)
