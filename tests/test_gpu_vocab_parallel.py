"""GPU parity of the vocabulary-shard calls against the fp64 oracle of the whole problem.

The classifier is split by rows into shards (linear_cross_entropy_06_b200.vocab_parallel.shard_range),
and the shards run one after another on one GPU, as the ranks of a vocabulary-parallel group would
(their only exchange, the all-gather of the partial results and the sum of dE, is done here by
stacking and adding). cce_forward_partial on every shard and cce_forward_merge give the loss and
LSE; cce_backward on every shard with the merged LSE and count gives the shards' dC and dbias rows
and their parts of dE. The results must match the oracle evaluated on the whole vocabulary, with
the tolerances of the other parity tests, and the tile skip decisions of the shards, put side by
side, must be the oracle's tile by tile.
"""
import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, assume, given, settings
from hypothesis import strategies as st

from linear_cross_entropy_06_b200 import ops
from linear_cross_entropy_06_b200.inputs import make_inputs
from linear_cross_entropy_06_b200.vocab_parallel import shard_range
from oracle import cce_oracle as O

from test_gpu_bias import make_bias
from test_gpu_parity import (EPS, LOSS_TOL, assert_close_elementwise, assert_skip_decisions, fp32_floor, frob_ok,
                             oracle_decisions, rel_frob)

pytestmark = pytest.mark.gpu


def run_shards(inp, bias, device, shards, reduction, eps, g, ls, zl):
    E, C, t = inp.E.to(device), inp.C.to(device), inp.targets.to(device)
    N, D = E.shape
    V = C.shape[0]
    b = None if bias is None else bias.to(device)
    ranges = [shard_range(V, shards, r) for r in range(shards)]
    parts, tmaxes = [], []
    for vs, n in ranges:
        partial, tmax = ops.cce_forward_partial(E, C[vs:vs + n], t, vs, V, -100,
                                                bias=None if b is None else b[vs:vs + n], label_smoothing=ls,
                                                check=True)
        parts.append(partial)
        tmaxes.append(tmax)
    # the merge takes the shards in any order: here the last one first
    loss, lse, count = ops.cce_forward_merge(torch.stack(parts[::-1]), t, V, D, -100, reduction, ls, zl)
    gd = g.to(device)
    dE = torch.zeros(N, D, device=device)
    dC, db, maps, filtered = [], [], [], 0
    for (vs, n), tmax in zip(ranges, tmaxes):
        out = ops.cce_backward(E, C[vs:vs + n], t, lse, tmax, count, gd, eps, -100, reduction,
                               out_fp32=ops.OUT_DE_FP32, check=True, bias=None if b is None else b[vs:vs + n],
                               dbias=True, label_smoothing=ls, z_loss=zl, skip_map=True, vocab_start=vs,
                               vocab_total=V)
        assert out[0].dtype == torch.float32 and out[1].dtype == torch.bfloat16
        dE += out[0]
        dC.append(out[1])
        db.append(out[3])
        maps.append(out[4])
        filtered += int(out[2].item())
    torch.cuda.synchronize()
    return dict(loss=loss.double().cpu().numpy(), lse=lse.double().cpu().numpy(), count=int(count.item()),
                dE=dE.double().cpu().numpy(), dC=torch.cat(dC).double().cpu().numpy(),
                dbias=torch.cat(db).double().cpu().numpy(), skipped=torch.cat(maps, dim=1).cpu().numpy().astype(bool),
                filtered=filtered)


def check_shards(inp, bias, device, shards, reduction, g, ls, zl):
    """The shards' merged loss, LSE and count, their gradients put together, and their skip
    decisions side by side, against the oracle of the whole problem (skipping off and on)."""
    N, V = inp.E.shape[0], inp.C.shape[0]
    g_or = g.numpy() if reduction == "none" else float(g.reshape(-1)[0])
    tm, tn = ops.backward_tile_shape()
    f = O.forward(inp.E, inp.C, inp.targets, -100, reduction, bias=bias, label_smoothing=ls, z_loss=zl)
    sc = O.row_scale(inp.targets, -100, reduction, g_or, f.count) * (1.0 + 2.0 * zl * np.abs(f.lse).max())
    for eps in (0.0, EPS):
        o = O.backward(inp.E, inp.C, inp.targets, g_or, -100, reduction, eps, tm, tn,
                       bias=np.zeros(V) if bias is None else bias, label_smoothing=ls, z_loss=zl)
        r = run_shards(inp, bias, device, shards, reduction, eps, g, ls, zl)
        assert np.abs(r["loss"].reshape(np.shape(f.loss)) - f.loss).max() <= LOSS_TOL * (
            max(f.count, 1) if reduction == "sum" else 1)
        assert np.abs(r["lse"] - f.lse).max() <= LOSS_TOL
        assert r["count"] == f.count
        for name, got, want, operand in (("dE", r["dE"], o.dE, inp.C), ("dC", r["dC"], o.dC, inp.E),
                                         ("dbias", r["dbias"][:, None], o.dbias[:, None], 1.0)):
            floor = fp32_floor(f.lse, sc, operand)
            assert frob_ok(got, want, 1e-2, floor), (name, eps, rel_frob(got, want))
            assert_close_elementwise(got, want, f"{name} eps={eps}", floor)
        assert_skip_decisions(r["skipped"], r["filtered"], *oracle_decisions(o.margin, eps), f"{shards} shards")
        ign = (inp.targets == -100).numpy()
        assert not r["dE"][ign].any()


@pytest.mark.parametrize("shards", [2, 3])
@pytest.mark.parametrize("variant", ["plain", "bias+smoothing+z-loss"])
@pytest.mark.parametrize("reduction", ["mean", "none"])
def test_vocabulary_shards_match_the_whole_problem(device, shards, variant, reduction):
    # peaked targets (tiles skipped), a vocabulary that is no multiple of the tile (a ragged last shard)
    inp = make_inputs("llama3.1-8b-head", N=384, D=256, V=5000, alpha=12.0, seed=71)
    N, V = inp.E.shape[0], inp.C.shape[0]
    bias, ls, zl = (make_bias(V, 72, scale=0.5), 0.1, 1e-4) if variant != "plain" else (None, 0.0, 0.0)
    g = torch.from_numpy(np.random.default_rng(73).standard_normal(N).astype(np.float32)) if reduction == "none" \
        else torch.tensor([1.0])
    check_shards(inp, bias, device, shards, reduction, g, ls, zl)


@settings(max_examples=20, derandomize=True, deadline=None,
          suppress_health_check=[HealthCheck.function_scoped_fixture, HealthCheck.too_slow])
@given(shards=st.integers(2, 5), N=st.integers(1, 400), D8=st.integers(1, 40), V=st.integers(129, 3000),
       reduction=st.sampled_from(["mean", "sum", "none"]), with_bias=st.booleans(),
       ls=st.sampled_from([0.0, 0.1]), zl=st.sampled_from([0.0, 1e-4]), peaked=st.booleans(),
       seed=st.integers(0, 10_000))
def test_random_shards_match_the_whole_problem(device, shards, N, D8, V, reduction, with_bias, ls, zl, peaked,
                                               seed):
    """Random problems and shard counts (every shard at least one 128-row tile of the classifier)."""
    assume(V > 128 * (shards - 1))
    D = 8 * D8
    if peaked:
        inp = make_inputs("llama3.2-1b-head", N=N, D=D, V=V, seed=seed, alpha=16.0, ignore_frac=0.1)
    else:
        inp = make_inputs("tiny", N=N, D=D, V=V, seed=seed, ignore_frac=0.1)
    g = torch.from_numpy(np.random.default_rng(seed + 1).standard_normal(N).astype(np.float32)) \
        if reduction == "none" else torch.tensor([0.75])
    bias = make_bias(V, seed + 2, scale=0.5) if with_bias else None
    check_shards(inp, bias, device, shards, reduction, g, ls, zl)


def test_shards_agree_with_the_unsharded_path(device):
    """Two shards against cce_forward / cce_backward on the whole classifier: the same loss and LSE up
    to the merge's rounding, and the same gradients up to the fp32 summation order of dE (the
    shards' parts are added last)."""
    inp = make_inputs("llama3.1-8b-head", N=512, D=512, V=8192, alpha=12.0, seed=74)
    E, C, t = inp.E.to(device), inp.C.to(device), inp.targets.to(device)
    loss, lse, tmax, count = ops.cce_forward(E, C, t, check=True)
    dE, dC, filt = ops.cce_backward(E, C, t, lse, tmax, count, torch.ones(1, device=device), EPS, out_fp32=True)
    r = run_shards(inp, None, device, 2, "mean", EPS, torch.tensor([1.0]), 0.0, 0.0)
    assert abs(float(r["loss"][0]) - float(loss)) <= 1e-5
    assert np.abs(r["lse"] - lse.double().cpu().numpy()).max() <= 1e-5
    assert r["filtered"] == int(filt.item())
    assert rel_frob(r["dE"], dE.double().cpu().numpy()) <= 1e-4  # fp32 sums of the shards' parts
    assert rel_frob(r["dC"], dC.double().cpu().numpy()) <= 5e-3  # bf16 rounding of the shards' dC


def test_shard_arguments_are_checked(device):
    inp = make_inputs("tiny", N=64, D=64, V=1000, seed=75)
    E, C, t = inp.E.to(device), inp.C.to(device), inp.targets.to(device)
    with pytest.raises(ops.CCEError):  # the shard must lie inside the vocabulary
        ops.cce_forward_partial(E, C[:600], t, 500, 1000)
    with pytest.raises(ops.CCEError):  # a shard's loss needs the merge
        lib = ops.load_library()
        import ctypes
        p = ops.Problem(64, 64, 600, -100, 1, 0, 0.0, 0.0, 0, 1000)
        ws = torch.empty(lib.cce_forward_workspace_size(ctypes.byref(p)), dtype=torch.uint8, device=device)
        out = torch.empty(64 * 64, device=device)
        ops._check(lib.cce_forward(ctypes.byref(p), E.data_ptr(), C.data_ptr(), None, t.data_ptr(), out.data_ptr(),
                                   out.data_ptr(), out.data_ptr(), out.data_ptr(), ws.data_ptr(), ws.numel(),
                                   torch.cuda.current_stream().cuda_stream))
    bad = t.clone()
    bad[3] = 1000  # outside the whole vocabulary: reported by the shard's forward
    with pytest.raises(ops.CCEError) as ei:
        ops.cce_forward_partial(E, C[:512], bad, 0, 1000, check=True)
    assert ei.value.status == 4
