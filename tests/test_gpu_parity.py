"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same seeded inputs.

Tolerances: the loss and per-row LSE within 2e-3 absolute; dE and dC within a relative
Frobenius error of 1e-2 when nothing is skipped. With skipping, dE and dC are within 2e-2 of
the unskipped oracle and within 1e-2 of the oracle that applies the same tile rule.
Elementwise: |gpu - oracle| <= 3e-2 * rms(that row of the oracle) + 3e-2 * |oracle| + floor, where
floor = 8 * 2^-23 * max|LSE| * max(scale_r) * max|operand| is the absolute error fp32 leaves in one
term of G = scale_r * (exp(z - LSE) - y) when p is close to 1 (p - 1 is then far below the fp32
resolution of z and LSE), carried through one product with E (dC) or C (dE). It matters only for
rows of dC or dE made of such terms alone; when every row is (one very peaked row, say), the
relative Frobenius bound gives way to the same floor on the whole matrix, floor * sqrt(elements).
Rows of ignored tokens in dE are exactly +0 and skipped-tile counts equal the oracle's (unless the
oracle reports a tile whose margin lies within 2e-3 of ln eps, in which case the difference is
bounded by that number).
"""
import math
import os
import sys

import numpy as np
import pytest
import torch

from linear_cross_entropy_06_b200 import ops
from linear_cross_entropy_06_b200.inputs import make_inputs
from oracle import cce_oracle as O

pytestmark = pytest.mark.gpu

EPS = 2.0 ** -12
LOSS_TOL = 2e-3


WINDOW = 2e-3  # the oracle's borderline window around ln eps (its default)


def run(inp, device, filter_eps=EPS, reduction=None, out_fp32=False, grad_out=None):
    reduction = reduction or inp.workload.reduction
    E, C, t = inp.E.to(device), inp.C.to(device), inp.targets.to(device)
    g = (inp.grad_out if grad_out is None else grad_out).to(device)
    if reduction != "none":
        g = g[:1]
    loss, lse, tmax, count = ops.cce_forward(E, C, t, -100, reduction, check=True)
    dE, dC, filt, smap = ops.cce_backward(E, C, t, lse, tmax, count, g, filter_eps, -100, reduction, out_fp32,
                                          check=True, skip_map=True)
    torch.cuda.synchronize()
    return dict(loss=loss.double().cpu().numpy(), lse=lse.double().cpu().numpy(), count=int(count.item()),
                dE=dE.double().cpu().numpy(), dC=dC.double().cpu().numpy(), filtered=int(filt.item()),
                dE_raw=dE.cpu(), tmax=tmax, skipped=smap.cpu().numpy().astype(bool))


def assert_skip_decisions(gpu_skipped, gpu_count, oracle_skipped, near, what):
    """Tile by tile: the GPU's skip decision equals the oracle's for every tile whose margin
    max(z - LSE) lies farther than WINDOW from ln eps. Inside the window the GPU decides from fp32
    values (the MMA's accumulation order, an fp32 LSE) and either decision is a correct rounding;
    the count of such disagreements bounds the difference of the skipped counts."""
    assert gpu_skipped.shape == oracle_skipped.shape, (gpu_skipped.shape, oracle_skipped.shape)
    assert int(gpu_skipped.sum()) == gpu_count, f"{what}: skip map and filtered count disagree"
    differ = gpu_skipped != oracle_skipped
    outside = differ & ~near
    assert not outside.any(), (f"{what}: {int(outside.sum())} tiles outside the borderline window decided "
                               f"differently, first at {np.argwhere(outside)[:4].tolist()}")
    assert abs(gpu_count - int(oracle_skipped.sum())) <= int(differ.sum())
    print(f"{what}: skipped gpu {gpu_count}, oracle {int(oracle_skipped.sum())} of {oracle_skipped.size}; "
          f"{int(near.sum())} borderline tiles, {int(differ.sum())} decided differently")


def oracle_decisions(margin, eps):
    """The oracle's skipped tiles and its borderline tiles, from its fp64 margins."""
    if eps <= 0:
        return np.zeros(margin.shape, dtype=bool), np.zeros(margin.shape, dtype=bool)
    return O.filtered_tiles(margin, eps), np.abs(margin - math.log(eps)) < WINDOW


def rel_frob(a, b):
    n = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (n if n > 0 else 1.0)


def _absmax(x):
    if isinstance(x, torch.Tensor):
        return float(x.detach().abs().max().double()) if x.numel() else 0.0
    x = np.asarray(x, dtype=np.float64)
    return float(np.abs(x).max()) if x.size else 0.0


def fp32_floor(lse, scale, operand):
    """Absolute error fp32 leaves in one term scale_r * (p - 1) * operand when p is close to 1."""
    return 8 * 2.0 ** -23 * max(_absmax(lse), 1.0) * _absmax(scale) * _absmax(operand)


def frob_ok(got, want, tol, floor=0.0):
    """Relative Frobenius error within tol, or an absolute error within the fp32 floor per element
    (for gradients made only of terms p - 1 with p rounded to 1 in fp32)."""
    return rel_frob(got, want) <= tol or np.linalg.norm(got - want) <= floor * np.sqrt(got.size)


def assert_close_elementwise(a, b, what, floor=0.0):
    # Row-wise scale: a row of dE or dC is one column of G times E or C, so its rounding error
    # grows with that row's own magnitude (rows of popular targets are far larger than the rest).
    rms = np.sqrt(np.mean(b * b, axis=1, keepdims=True)) if b.size else 0.0
    bad = np.abs(a - b) > 3e-2 * rms + 3e-2 * np.abs(b) + floor + 1e-30
    assert not bad.any(), f"{what}: {int(bad.sum())} elements outside tolerance, worst {np.abs(a - b).max():.3e}"


def assert_grads(g_dE, g_dC, o_dE, o_dC, tol, what="", floor_dE=0.0, floor_dC=0.0):
    assert frob_ok(g_dE, o_dE, tol, floor_dE), f"{what} dE rel-Frobenius {rel_frob(g_dE, o_dE):.3e}"
    assert frob_ok(g_dC, o_dC, tol, floor_dC), f"{what} dC rel-Frobenius {rel_frob(g_dC, o_dC):.3e}"
    assert_close_elementwise(g_dE, o_dE, what + " dE", floor_dE)
    assert_close_elementwise(g_dC, o_dC, what + " dC", floor_dC)


def assert_ignored_rows_zero(res, targets):
    ign = (targets == -100).numpy()
    if ign.any():
        raw = res["dE_raw"][torch.from_numpy(ign)]
        bits = raw.view(torch.int16) if raw.dtype == torch.bfloat16 else raw.view(torch.int32)
        assert (bits == 0).all(), "dE rows of ignored tokens must be exactly +0"


def assert_count(gpu_count, oracle_count, borderline):
    assert abs(gpu_count - oracle_count) <= borderline, (gpu_count, oracle_count, borderline)
    if borderline == 0:
        assert gpu_count == oracle_count


def tile_shape():
    return ops.backward_tile_shape()


def check_full(inp, device, reduction=None, grad_out=None):
    """Whole-problem comparison for sizes the oracle finishes in seconds."""
    reduction = reduction or inp.workload.reduction
    tm, tn = tile_shape()
    g = inp.grad_out if grad_out is None else grad_out
    g_or = g.numpy() if reduction == "none" else float(g.reshape(-1)[0])
    f = O.forward(inp.E, inp.C, inp.targets, -100, reduction)
    b0 = O.backward(inp.E, inp.C, inp.targets, g_or, -100, reduction, 0.0, tm, tn)
    b1 = O.backward(inp.E, inp.C, inp.targets, g_or, -100, reduction, EPS, tm, tn)
    r0 = run(inp, device, 0.0, reduction, grad_out=grad_out)
    r1 = run(inp, device, EPS, reduction, grad_out=grad_out)
    for r in (r0, r1):
        if reduction == "sum":
            assert abs(r["loss"][0] - float(f.loss)) <= LOSS_TOL * max(f.count, 1)
        else:
            assert np.abs(r["loss"].reshape(np.asarray(f.loss).shape) - f.loss).max() <= LOSS_TOL
        assert np.abs(r["lse"] - f.lse).max() <= LOSS_TOL
        assert r["count"] == f.count
        assert_ignored_rows_zero(r, inp.targets)
    assert r0["filtered"] == 0
    sc = O.row_scale(inp.targets, -100, reduction, g_or, f.count)
    fl_dE, fl_dC = fp32_floor(f.lse, sc, inp.C), fp32_floor(f.lse, sc, inp.E)
    assert_grads(r0["dE"], r0["dC"], b0.dE, b0.dC, 1e-2, "filter off", fl_dE, fl_dC)
    assert_grads(r1["dE"], r1["dC"], b1.dE, b1.dC, 1e-2, "filter on", fl_dE, fl_dC)
    assert rel_frob(r1["dE"], b0.dE) <= 2e-2 and rel_frob(r1["dC"], b0.dC) <= 2e-2
    assert_count(r1["filtered"], b1.filtered, b1.borderline)
    assert_skip_decisions(r1["skipped"], r1["filtered"], *oracle_decisions(b1.margin, EPS), "filter on")
    assert not r0["skipped"].any()
    return r0, r1, b1


def test_tiny(device):
    inp = make_inputs("tiny")
    check_full(inp, device)


def test_tiny_fp32_originals_gap_is_small(device):
    """Information only: the bf16 rounding of the inputs moves the loss by far less than 1e-2."""
    inp = make_inputs("tiny")
    f16 = O.forward(inp.E, inp.C, inp.targets)
    f32 = O.forward(inp.E32, inp.C32, inp.targets)
    assert abs(float(f16.loss) - float(f32.loss)) < 1e-2


@pytest.mark.parametrize("shape", [(300, 136, 1000), (129, 72, 257), (1, 8, 17), (5, 64, 130), (200, 320, 640)])
@pytest.mark.parametrize("reduction", ["mean", "sum", "none"])
def test_ragged_shapes(device, shape, reduction):
    N, D, V = shape
    inp = make_inputs("tiny", N=N, D=D, V=V, seed=7 + N + D + V, ignore_frac=0.1)
    g = torch.from_numpy(np.random.default_rng(N).standard_normal(N).astype(np.float32))
    check_full(inp, device, reduction, grad_out=g if reduction == "none" else torch.tensor([0.75]))


def test_skipping_on_a_peaked_problem(device):
    # a seed with no unit of the skip rule (128 x 64) whose oracle margin lies within the borderline
    # window, so that the skipped counts must agree exactly
    inp = make_inputs("llama3.1-8b-head", N=512, D=256, V=16384, alpha=14.0, seed=27)
    _, r1, b1 = check_full(inp, device)
    tm, tn = tile_shape()
    assert 0 < r1["filtered"] < (512 // tm) * (16384 // tn)
    assert b1.borderline == 0


def test_every_row_ignored(device):
    inp = make_inputs("tiny", N=64, ignore_frac=1.0)
    r = run(inp, device, EPS, "mean")
    assert r["loss"][0] == 0.0 and r["count"] == 0
    assert not r["dE"].any() and not r["dC"].any()
    tm, tn = tile_shape()  # every tile holds only ignored rows: all skipped
    assert r["filtered"] == math.ceil(64 / tm) * math.ceil(4096 / tn)


def test_no_rows(device):
    inp = make_inputs("tiny", N=0)
    for red in ("mean", "sum"):
        r = run(inp, device, EPS, red)
        assert r["loss"][0] == 0.0 and r["count"] == 0
        assert r["dE"].shape == (0, 128) and not r["dC"].any()


def test_target_out_of_range_is_reported(device):
    inp = make_inputs("tiny", N=64)
    t = inp.targets.clone()
    t[5] = 4096
    E, C = inp.E.to(device), inp.C.to(device)
    with pytest.raises(ops.CCEError) as ei:
        ops.cce_forward(E, C, t.to(device), -100, "mean", check=True)
    assert ei.value.status == 4


def test_fp32_and_bf16_outputs_agree(device):
    inp = make_inputs("tiny", N=200, D=64, V=1000, seed=3)
    a = run(inp, device, EPS, "mean", out_fp32=False)
    b = run(inp, device, EPS, "mean", out_fp32=True)
    assert a["filtered"] == b["filtered"]
    assert rel_frob(a["dE"], b["dE"]) < 5e-3 and rel_frob(a["dC"], b["dC"]) < 5e-3


def test_forward_is_deterministic(device):
    inp = make_inputs("llama3.1-8b-head", N=1024, D=1024, V=32768, seed=5)
    E, C, t = inp.E.to(device), inp.C.to(device), inp.targets.to(device)
    outs = [ops.cce_forward(E, C, t, -100, "mean") for _ in range(3)]
    for o in outs[1:]:
        assert torch.equal(o[0], outs[0][0]) and torch.equal(o[1], outs[0][1]) and torch.equal(o[2], outs[0][2])


def test_autograd_wrapper(device):
    inp = make_inputs("tiny", N=96, D=128, V=2000, seed=9)
    e = inp.E.reshape(4, 24, 128).to(device).requires_grad_(True)
    c = inp.C.to(device).requires_grad_(True)
    t = inp.targets.reshape(4, 24).to(device)
    loss = ops.linear_cross_entropy(e, c, t)
    loss.backward()
    f = O.forward(inp.E, inp.C, inp.targets)
    tm, tn = tile_shape()
    b = O.backward(inp.E, inp.C, inp.targets, 1.0, -100, "mean", EPS, tm, tn)
    assert abs(float(loss.detach()) - float(f.loss)) <= LOSS_TOL
    assert rel_frob(e.grad.reshape(96, 128).double().cpu().numpy(), b.dE) <= 1e-2
    assert rel_frob(c.grad.double().cpu().numpy(), b.dC) <= 1e-2
    nll = ops.linear_cross_entropy(e, c, t, reduction="none")
    assert nll.shape == (4, 24)


# ------------------------------------------------------------------------------------------------
# Full-size workloads: every row's LSE, the loss and the skip count from a full fp64 pass; dE on
# seeded rows and dC on seeded vocabulary rows (popular target ids included).
# ------------------------------------------------------------------------------------------------

def _sample(n, k, seed, extra=()):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([rng.choice(n, size=min(k, n), replace=False), np.asarray(extra, int)]))


def _check_vs_oracle(g_dE, o_dE, g_dC, o_dC, lse_o, sc, E, C, tol, what):
    """GPU dE rows and dC rows against the oracle's: relative Frobenius error within tol and the
    elementwise bound (with the fp32 floor of one p - 1 term)."""
    fl_dE, fl_dC = fp32_floor(lse_o, sc, C), fp32_floor(lse_o, sc, E)
    assert rel_frob(g_dE, o_dE) <= tol, f"{what} dE rel-Frobenius {rel_frob(g_dE, o_dE):.3e}"
    assert rel_frob(g_dC, o_dC) <= tol, f"{what} dC rel-Frobenius {rel_frob(g_dC, o_dC):.3e}"
    assert_close_elementwise(g_dE, o_dE, what + " dE rows", fl_dE)
    assert_close_elementwise(g_dC, o_dC, what + " dC rows", fl_dC)


@pytest.mark.parametrize("name", ["llama3.2-1b-head", "gemma2-2b-head", "gemma2-2b-head-peaked", "llama3.1-8b-head"])
def test_full_size_workload(device, name):
    """Skipping on and off at full size. One fp64 pass gives every row's LSE, the loss and every
    tile's decision, dE on seeded rows and dC on seeded vocabulary rows (popular targets included);
    whole row blocks and whole vocabulary tiles are then evaluated exactly with and without skipping
    (the skip rule reads only a tile's own rows and columns)."""
    inp = make_inputs(name)
    w = inp.workload
    tm, tn = tile_shape()
    nb, nt = -(-w.N // tm), -(-w.V // tn)
    rows = _sample(w.N, 192, 1)
    cols = _sample(w.V, 192, 2, extra=np.unique(inp.targets[inp.targets >= 0].numpy())[:64])
    s = O.sampled(inp.E, inp.C, inp.targets, rows, cols, 1.0, -100, w.reduction, EPS, tm, tn)
    blocks, tiles = [0, nb // 2, nb - 1], [0, 1, nt // 2, nt - 1]
    rb = {e: O.row_blocks(inp.E, inp.C, inp.targets, blocks, 1.0, -100, w.reduction, e, tm, tn) for e in (0.0, EPS)}
    vt = {e: O.vocab_tiles(inp.E, inp.C, inp.targets, s.lse, tiles, 1.0, -100, w.reduction, e, tm, tn)
          for e in (0.0, EPS)}
    sc = O.row_scale(inp.targets, -100, w.reduction, 1.0, s.count)
    r1 = run(inp, device, EPS, w.reduction)
    r0 = run(inp, device, 0.0, w.reduction)
    for r in (r0, r1):
        assert abs(r["loss"][0] - float(s.loss)) <= LOSS_TOL
        assert np.abs(r["lse"] - s.lse).max() <= LOSS_TOL
        assert r["count"] == s.count
        assert_ignored_rows_zero(r, inp.targets)
    # skipping on: the oracle with the same tile rule, tile by tile
    assert_skip_decisions(r1["skipped"], r1["filtered"], *oracle_decisions(s.margin, EPS), name)
    assert rel_frob(r1["dE"][rows], s.dE_rows) <= 1e-2
    assert rel_frob(r1["dC"][cols], s.dC_cols) <= 1e-2
    assert_close_elementwise(r1["dE"][rows], s.dE_rows, "dE rows")
    assert_close_elementwise(r1["dC"][cols], s.dC_cols, "dC rows")
    _check_vs_oracle(r1["dE"][rb[EPS].rows], rb[EPS].dE, r1["dC"][vt[EPS].cols], vt[EPS].dC, s.lse, sc, inp.E, inp.C,
                     1e-2, "filter on")
    # skipping off: every tile kept, the plain definition
    assert r0["filtered"] == 0
    _check_vs_oracle(r0["dE"][rb[0.0].rows], rb[0.0].dE, r0["dC"][vt[0.0].cols], vt[0.0].dC, s.lse, sc, inp.E, inp.C,
                     1e-2, "filter off")
    # skipping on against the unskipped oracle: within 2e-2 wherever the skip rule itself (the oracle
    # against the oracle) stays within it; where the rule alone moves the gradient further (the Gemma
    # head's 256000-entry vocabulary), within the rule's own effect plus 2e-3
    for what, got, o1, o0 in (("dE", r1["dE"][rb[0.0].rows], rb[EPS].dE, rb[0.0].dE),
                              ("dC", r1["dC"][vt[0.0].cols], vt[EPS].dC, vt[0.0].dC)):
        rule = rel_frob(o1, o0)
        err = rel_frob(got, o0)
        print(f"{name} {what}: skipped against unskipped: gpu {err:.4f}, the rule alone (oracle) {rule:.4f}")
        assert err <= max(2e-2, rule + 2e-3), (what, err, rule)


LONG_BATCH_GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "long_batch_oracle.npz")


def test_long_batch(device):
    """N = 32768 tokens, D = 4096, V = 128256, reduction 'none' with grad_out ~ N(0, 1), bf16 outputs
    (the bench's launch configuration for this workload), skipping at 2^-12 and off.

    Every row's LSE and per-token loss and the skipped-tile count come from one full fp64 pass of the
    oracle, stored by tests/golden/make_long_batch.py (minutes of CPU time). dE of whole row blocks
    and dC of whole vocabulary tiles (tile 0 holds the most popular Zipf targets) are evaluated here
    by the oracle, with the stored LSE for dC."""
    inp = make_inputs("long-batch")
    w = inp.workload
    gold = np.load(LONG_BATCH_GOLDEN)
    sys.path.insert(0, os.path.dirname(LONG_BATCH_GOLDEN))
    from make_long_batch import fingerprint
    assert str(gold["fingerprint"]) == fingerprint(inp), "the seeded inputs differ from those the file was made from"
    tm, tn = tile_shape()
    assert tuple(gold["tile"]) == (tm, tn) and float(gold["eps"]) == EPS
    g = inp.grad_out.numpy()
    E, C, t, gd = (x.to(device) for x in (inp.E, inp.C, inp.targets, inp.grad_out))
    loss, lse, tmax, count = ops.cce_forward(E, C, t, -100, "none", check=True)
    assert int(count.item()) == int(gold["count"])
    assert np.abs(lse.double().cpu().numpy() - gold["lse"]).max() <= LOSS_TOL
    assert np.abs(loss.double().cpu().numpy() - gold["nll"]).max() <= LOSS_TOL
    nb, nt = -(-w.N // tm), -(-w.V // tn)
    blocks, tiles = [3, 200, nb - 1], [0, 1, nt // 2, nt - 1]
    sc = O.row_scale(inp.targets, -100, "none", g, int(gold["count"]))
    got = {}
    for e in (EPS, 0.0):
        dE, dC, filt, smap = ops.cce_backward(E, C, t, lse, tmax, count, gd, e, -100, "none", out_fp32=False,
                                              check=True, skip_map=True)
        torch.cuda.synchronize()
        if e > 0:
            shape = tuple(gold["grid"])
            o_skip = np.unpackbits(gold["skipped_bits"])[:shape[0] * shape[1]].reshape(shape).astype(bool)
            o_near = np.unpackbits(gold["borderline_bits"])[:shape[0] * shape[1]].reshape(shape).astype(bool)
            assert int(o_skip.sum()) == int(gold["filtered"]) and float(gold["window"]) == WINDOW
            assert_skip_decisions(smap.cpu().numpy().astype(bool), int(filt.item()), o_skip, o_near, "long-batch")
        else:
            assert not smap.any()
        rb = O.row_blocks(inp.E, inp.C, inp.targets, blocks, g, -100, "none", e, tm, tn)
        vt = O.vocab_tiles(inp.E, inp.C, inp.targets, gold["lse"], tiles, g, -100, "none", e, tm, tn)
        np.testing.assert_allclose(rb.lse, gold["lse"][rb.rows], rtol=1e-12)
        assert_ignored_rows_zero(dict(dE_raw=dE.cpu()), inp.targets)
        g_dE = dE[torch.from_numpy(rb.rows).to(device)].double().cpu().numpy()
        g_dC = dC[torch.from_numpy(vt.cols).to(device)].double().cpu().numpy()
        _check_vs_oracle(g_dE, rb.dE, g_dC, vt.dC, gold["lse"], sc, inp.E, inp.C, 1e-2, f"eps={e}")
        got[e] = (int(filt.item()), g_dE, g_dC, rb, vt)
        del dE, dC
    assert got[0.0][0] == 0
    assert got[EPS][4].filtered > 0  # skipped tiles among the checked vocabulary tiles
    rb0, vt0 = got[0.0][3], got[0.0][4]
    for what, g_, o1, o0 in (("dE", got[EPS][1], got[EPS][3].dE, rb0.dE), ("dC", got[EPS][2], got[EPS][4].dC, vt0.dC)):
        rule, err = rel_frob(o1, o0), rel_frob(g_, o0)
        print(f"long-batch {what}: skipped against unskipped: gpu {err:.4f}, the rule alone (oracle) {rule:.4f}")
        assert err <= max(2e-2, rule + 2e-3), (what, err, rule)


def _extra_loss_memory(device, N, D, V):
    """Peak device memory of one forward + backward beyond the inputs and the fp32 gradients."""
    inp = make_inputs("llama3.1-8b-head", N=N, D=D, V=V, seed=11)
    E, C, t = inp.E.to(device), inp.C.to(device), inp.targets.to(device)
    g = torch.ones(1, device=device)
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    loss, lse, tmax, count = ops.cce_forward(E, C, t)
    dE, dC, filt = ops.cce_backward(E, C, t, lse, tmax, count, g, out_fp32=True)
    torch.cuda.synchronize()
    extra = torch.cuda.max_memory_allocated() - base
    del loss, lse, tmax, count, dE, dC, filt
    return extra - (N + V) * D * 4


def _memory_bound(N, V):
    """Tile statistics (8 N bytes per 64 columns), the tile plan (at most 48 bytes per 128x128
    tile), the gradient-tile scratch (4 MiB per 128-row block, at least 128 MiB) and 8 MiB of
    small buffers and allocator rounding."""
    nb, nt = math.ceil(N / 128), math.ceil(V / 128)
    return 8 * N * math.ceil(V / 64) + 48 * nb * nt + max(128 << 20, nb * (4 << 20)) + (8 << 20)


def test_no_logit_sized_allocation(device):
    """Extra device memory of forward + backward is O(N + N*V/64), never O(N*V).

    Beyond the gradients themselves ((N+V)*D*4 with fp32 outputs) the path holds the forward's
    per-sub-tile maxima and exp sums (8*N*ceil(V/64) bytes), the backward's tile plan
    (flags, ranks, the two tile lists, the map between them and the kept-half prefix: 29 bytes per
    128x128 tile; the pair lists: about 12 more) and the gradient tiles of two vocabulary chunks
    (4 MiB per 128-row block, at least 128 MiB). Doubling V must grow that by the tile statistics
    only.
    """
    N, D = 4096, 1024
    m1, m2 = _extra_loss_memory(device, N, D, 64128), _extra_loss_memory(device, N, D, 128256)
    for V, m in ((64128, m1), (128256, m2)):
        assert m <= _memory_bound(N, V), (V, m, _memory_bound(N, V))
    assert m2 < N * 128256 * 2 / 4, m2  # at the Llama-3 vocabulary, far below even bf16 logits
    # growth with V: the tile statistics (8 N bytes per 64 columns), not N*V*2
    assert m2 - m1 <= 8 * N * math.ceil(64128 / 64) * 1.25 + (4 << 20), (m1, m2)


def test_no_logit_sized_allocation_long_batch(device):
    """At the long-batch token count (N = 32768) the scratch grows with N (4 MiB per 128 rows)
    and the extra memory stays a small fraction of the bf16 logits (N*V*2 = 8.4 GB)."""
    N, D, V = 32768, 1024, 128256
    m = _extra_loss_memory(device, N, D, V)
    assert m <= _memory_bound(N, V), (m, _memory_bound(N, V))
    assert m < N * V * 2 / 4, m


@pytest.mark.parametrize("D", [8192, 12296])
def test_large_hidden_sizes(device, D):
    """Hidden sizes beyond the pages' heads: many 256-column slices per dE/dC item, and (12296 =
    48 * 256 + 8) a last slice of 8 columns."""
    inp = make_inputs("tiny", N=200, D=D, V=1500, seed=D, ignore_frac=0.1)
    check_full(inp, device, "mean")
