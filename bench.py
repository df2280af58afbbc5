"""Benchmark of the Cut Cross-Entropy hot path: forward + backward tokens/s on one B200 per rank.

A step is one forward (loss and LSE) and one backward (dE and dC, tile skipping at 2^-12) over
one batch of the workload, through the library's C ABI. With no flags: 1 GPU, the Llama-3.1-8B
head shape (N = 4096 tokens, D = 4096, V = 128256, peaked Zipf(1.1) targets, 5% ignored,
reduction mean), synthetic seeded data.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

Under torchrun (N > 1) every rank runs its own batch (independent replicas: the method shards by
tokens with no exchange in the loss), the step time is the max over ranks, and rank 0 prints one
JSON line. ``--impl reference`` times the fp64 CPU oracle on a bounded row sample of the same
workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
EPS = 2.0 ** -12
# The headline metric: tokens/s of one forward + backward at the Llama-3.1-8B head shape, with the
# fraction of the B200 bf16 tensor peak reported beside it (tensor_peak_frac).
METRIC = "fwd+bwd tokens/s at Llama-3-8B head shape; % of B200 BF16 tensor peak"
L2_FLUSH_BYTES = 512 << 20
# The skip rule's tile (rows x vocabulary columns) given to the oracle when it is timed: the
# backward's tile shape, stated here so that timing the oracle never loads the CUDA library.
ORACLE_SKIP_TILE = (128, 64)
# DRAM bytes (read + write) of one launch of each tensor-core kernel, from a one-kernel, one-launch,
# one-pass ncu capture (dram__bytes_read.sum + dram__bytes_write.sum), reported as the roofline's
# "traffic". Each entry is keyed by the workload's (N, D, V) and holds the SHA-256 of the kernel's
# sources at the time of the capture: when those sources change, the figure no longer describes the
# kernel and the bench reports null instead. The ncu summaries under profiles/ give the commands.
KERNEL_SOURCES = {  # the kernel and what sets up its work (maps, plan, chunking)
    "fwd_lse_kernel": ("cce_fwd.cu", "cce_device.cuh", "cce_internal.h", "cce_api.cu"),
    "bwd_kernel": ("cce_bwd.cu", "cce_device.cuh", "cce_internal.h", "cce_api.cu", "cce_bwd_plan.cu"),
}
TRAFFIC_BYTES = {
    "fwd_lse_kernel": {
        (4096, 4096, 128256): ("2ed61cfe1a1a6ec72e48cd6d2754b958037681af0ba13cc5ce0ada1deecb2e2f",
                               1085621248 + 67207680),
    },
    "bwd_kernel": {
        (4096, 4096, 128256): ("d17440dea28d61347ec4d2753c760768a083030d6a3fd051d876eebdf64ec76e",
                               4559904512 + 1673345536),
    },
}


def kernel_source_hash(kernel: str) -> str:
    """SHA-256 over the kernel's source files, in a fixed order."""
    import hashlib

    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "linear_cross_entropy_06_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(kernel: str, shape: tuple):
    """DRAM bytes per launch from the capture of this kernel at this shape, or None when there is
    none or the kernel's sources changed since it was taken."""
    entry = TRAFFIC_BYTES.get(kernel, {}).get(tuple(shape))
    if entry is None:
        return None
    sha, nbytes = entry
    return nbytes if sha == kernel_source_hash(kernel) else None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(PEAKS_FALLBACK), "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,power.limit")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None
        self.out = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        self.out = os.fdopen(fd, "w")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            self.proc.wait(timeout=10)
        self.out.close()
        if self.proc is None:
            os.unlink(self.path)
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower().startswith("active")})
        busy = [s for s in sm if s > 0.5 * (max(sm) if sm else 0)]
        power = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        limit = [float(r[9]) for r in rows if len(r) > 9 and r[9].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(busy) if busy else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "power_w_max": max(power) if power else None,
                "power_limit_w": max(limit) if limit else None}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's value: step times are reported as the max over ranks."""
    if world == 1:
        return x
    import torch.distributed as dist

    if dist.get_backend() == "gloo":
        device = torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world: int, tokens_per_rank: int, steps: int, max_seconds: float) -> float:
    """Whole-job tokens/s: every rank processes its own batch; time is the slowest rank's."""
    return world * tokens_per_rank * steps / max_seconds


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def algorithmic_flops(N: int, D: int, V: int, kept_tiles: int, tile: tuple) -> tuple:
    """2NVD forward; 6 * rows * cols * D per kept unit of the skip rule (recompute, dE, dC).

    Kept units are counted at their full size: at every bench workload N and V are multiples of
    the unit, so none is partial (for ragged shapes this slightly overcounts the backward)."""
    tm, tn = tile
    return 2.0 * N * V * D, 6.0 * tm * tn * D * kept_tiles


def listed_tile_count(skip_map) -> int:
    """Backward tiles (128 x 128) with a kept 128 x 64 unit: the tiles whose dC MMAs run (over both
    halves)."""
    kept = (skip_map == 0)
    if kept.shape[1] % 2:
        kept = torch.nn.functional.pad(kept, (0, 1))
    return int((kept[:, 0::2] | kept[:, 1::2]).sum().item())


def issued_mma_flops(D: int, kept_units: int, listed_tiles: int, tile: tuple) -> float:
    """The backward's tensor-core work as issued: the recompute and the dE MMAs run over the kept
    units only, the dC MMAs over every listed tile's two units (a skipped unit reads as zeros)."""
    tm, tn = tile
    return 4.0 * tm * tn * D * kept_units + 2.0 * tm * (2 * tn) * D * listed_tiles


def oracle_sample_seconds(inp, rows: int):
    """fp64 oracle forward + backward on the first `rows` tokens of the workload (full vocabulary)."""
    from oracle import cce_oracle as O

    tm, tn = ORACLE_SKIP_TILE
    w = inp.workload
    E, t = inp.E[:rows], inp.targets[:rows]
    g = inp.grad_out[:rows] if w.reduction == "none" else inp.grad_out
    gv = g.numpy() if w.reduction == "none" else float(g.reshape(-1)[0])
    t0 = time.perf_counter()
    O.forward(E, inp.C, t, -100, w.reduction)
    O.backward(E, inp.C, t, gv, -100, w.reduction, EPS, tm, tn)
    return time.perf_counter() - t0


def oracle_threads() -> int:
    """Threads the oracle's arithmetic runs on: its one library step is numpy's matmul, so the size
    of the BLAS thread pool numpy loaded (threadpoolctl), not torch's intra-op pool."""
    import numpy  # noqa: F401  (loads the BLAS whose pool is inspected)
    from threadpoolctl import threadpool_info

    blas = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
    return max(blas) if blas else 1


def run_reference(args, world, rank):
    """--impl reference: the fp64 CPU oracle, as it stands, on a bounded row sample per step."""
    if rank != 0:
        return
    from linear_cross_entropy_06_b200.inputs import make_inputs

    inp = make_inputs(args.workload)
    w = inp.workload
    rows = args.ref_rows
    for _ in range(args.warmup):
        oracle_sample_seconds(inp, rows)
    secs = [oracle_sample_seconds(inp, rows) for _ in range(args.steps)]
    total = sum(secs)
    value = rows * args.steps / total
    cores = oracle_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"first {rows} of {w.N} tokens per step, full V={w.V} and D={w.D}, fp64"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w, gpus, shape=None):
    N, D, V = shape or (w.N, w.D, w.V)
    return {"workload": w.name, "tokens_per_gpu": N, "hidden": D, "vocab": V, "targets": w.targets,
            "ignore_frac": w.ignore_frac, "reduction": w.reduction, "filter_eps": EPS,
            "parallelism": f"replicas x{gpus} (tokens sharded, no collective)",
            "l2": "512 MiB written between timed steps; C (up to 2 GB) is larger than L2"}


def run_ours(args, world, rank, local):
    from linear_cross_entropy_06_b200 import ops
    from linear_cross_entropy_06_b200.inputs import make_inputs

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    lib = ops.load_library()
    over = dict(zip("NDV", map(int, args.shape.split(",")))) if args.shape else {}
    inp = make_inputs(args.workload, seed=None if world == 1 else 1238 + 1000 * rank, **over)
    w = inp.workload
    N, D, V = inp.E.shape[0], inp.E.shape[1], inp.C.shape[0]
    E, C, t = inp.E.to(dev), inp.C.to(dev), inp.targets.to(dev)
    g = inp.grad_out.to(dev)
    if w.reduction != "none":
        g = g[:1]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    tile = ops.backward_tile_shape()

    def step():
        loss, lse, tmax, count = ops.cce_forward(E, C, t, -100, w.reduction)
        dE, dC, filt = ops.cce_backward(E, C, t, lse, tmax, count, g, EPS, -100, w.reduction, out_fp32=False)
        return loss, filt

    # check once that nothing was reported on the device; the skip map of that call gives the
    # tensor-core work the backward issues (below)
    loss0, lse0, tmax0, count0 = ops.cce_forward(E, C, t, -100, w.reduction, check=True)
    skip_map = ops.cce_backward(E, C, t, lse0, tmax0, count0, g, EPS, -100, w.reduction, check=True,
                                skip_map=True)[-1]
    listed_tiles = listed_tile_count(skip_map)
    del loss0, lse0, tmax0, count0, skip_map

    # peak device memory of one forward + backward beyond the resident inputs (untimed): the bf16
    # gradients themselves, plus everything the loss needs, which must stay far below N*V*2
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats(dev)
    base = torch.cuda.memory_allocated(dev)
    step()
    torch.cuda.synchronize()
    peak = torch.cuda.max_memory_allocated(dev) - base
    grads = (N + V) * D * 2
    memory = {"peak_extra_bytes": peak, "gradients_bytes": grads, "beyond_gradients_bytes": peak - grads,
              "logits_bf16_bytes": N * V * 2, "beyond_gradients_over_logits": (peak - grads) / (N * V * 2)}

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    for e6 in ev:  # materialise the raw handles
        for e in e6:
            e.record()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    launches0 = lib.cce_kernel_launch_count()
    filt_last = None
    for k in range(args.steps):
        flush.fill_(k & 0xFF)
        s0, s1, f0, f1, b0, b1 = ev[k]
        lib.cce_set_kernel_events(f0.cuda_event, f1.cuda_event, b0.cuda_event, b1.cuda_event)
        s0.record()
        loss, filt_last = step()
        s1.record()
    lib.cce_set_kernel_events(None, None, None, None)
    torch.cuda.synchronize()
    launches = lib.cce_kernel_launch_count() - launches0
    barrier(world)
    torch.cuda.synchronize()
    clocks = sampler.stop()

    step_ms = [e[0].elapsed_time(e[1]) for e in ev]
    fwd_ms = [e[2].elapsed_time(e[3]) for e in ev]
    bwd_ms = [e[4].elapsed_time(e[5]) for e in ev]
    total_s = max_over_ranks(sum(step_ms) / 1e3, world, dev)
    value = weak_scaling_value(world, N, args.steps, total_s)
    filtered = int(filt_last.item())
    nb, nt = -(-N // tile[0]), -(-V // tile[1])
    kept = nb * nt - filtered
    fwd_flop, bwd_flop = algorithmic_flops(N, D, V, kept, tile)
    peaks, peak_kind = load_peaks()
    peak_tf = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    peak_sus = peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"])

    def kernel_line(flop, ms_list, what):
        avg = statistics.mean(ms_list)
        return {"ms": avg, "ms_median": statistics.median(ms_list), "ms_min": min(ms_list), "launches_per_step": 1,
                "tflops": flop / avg / 1e9, "frac": flop / avg / 1e9 / peak_tf,
                "frac_sustained": flop / avg / 1e9 / peak_sus, "what": what}

    kernels = {
        "fwd_lse_kernel": kernel_line(fwd_flop, fwd_ms, "persistent logit tiles with per-row max and sum-exp"),
        "bwd_kernel": kernel_line(bwd_flop, bwd_ms,
                                  "one persistent launch per step: recompute, gradient tiles, dC and dE MMAs"),
    }
    issued = issued_mma_flops(D, kept, listed_tiles, tile)
    kernels["bwd_kernel"].update(listed_tiles=listed_tiles, issued_mma_flops=issued,
                                 issued_mma_tflops=issued / kernels["bwd_kernel"]["ms"] / 1e9,
                                 issued_mma_frac=issued / kernels["bwd_kernel"]["ms"] / 1e9 / peak_tf)
    # The dominant kernel: the forward and the backward are one launch each per step; the roofline
    # line reports the longer one (by average launch duration over the timed steps).
    dom = "bwd_kernel" if kernels["bwd_kernel"]["ms"] > kernels["fwd_lse_kernel"]["ms"] else "fwd_lse_kernel"
    dom_flop = bwd_flop if dom == "bwd_kernel" else fwd_flop
    dom_ms = kernels[dom]["ms"]
    dom_traffic = measured_traffic(dom, (N, D, V))
    ms_step = 1e3 * total_s / args.steps
    path_tflops = (fwd_flop + bwd_flop) / (ms_step / 1e3) / 1e12

    # end to end through the public API: every step copies its inputs from pinned host memory and
    # reads its loss back to the host. Two device input slots let the copy of step k + 1 (on a copy
    # stream) run while step k computes, as a training loop with a prefetching loader would.
    # copy_c=False keeps the classifier C on the device across steps (a model parameter, as in
    # training) and copies only the hidden states E and the targets.
    def measure_e2e(copy_c: bool):
        hE, ht = inp.E.pin_memory(), inp.targets.pin_memory()
        hC = inp.C.pin_memory() if copy_c else None
        slots = [(torch.empty_like(E), torch.empty_like(C) if copy_c else C, torch.empty_like(t)) for _ in range(2)]
        h2d = hE.numel() * 2 + ht.numel() * 8 + (hC.numel() * 2 if copy_c else 0)
        d2h = 4
        compute = torch.cuda.current_stream(dev)
        copier = torch.cuda.Stream(dev)
        copied = [torch.cuda.Event() for _ in range(2)]
        used = [torch.cuda.Event() for _ in range(2)]

        def issue_copy(k):
            dst = slots[k % 2]
            with torch.cuda.stream(copier):
                if k >= 2:
                    copier.wait_event(used[k % 2])  # step k - 2 is done with this slot
                dst[0].copy_(hE, non_blocking=True)
                if copy_c:
                    dst[1].copy_(hC, non_blocking=True)
                dst[2].copy_(ht, non_blocking=True)
                copied[k % 2].record(copier)

        def run_steps(n):
            start = torch.cuda.Event()
            start.record(compute)
            copier.wait_event(start)
            issue_copy(0)
            for k in range(n):
                if k + 1 < n:
                    issue_copy(k + 1)
                compute.wait_event(copied[k % 2])
                dE_in, dC_in, dt = slots[k % 2]
                e_ = dE_in.detach().requires_grad_(True)
                c_ = dC_in.detach().requires_grad_(True)
                out = ops.linear_cross_entropy(e_, c_, dt, reduction=w.reduction)
                out.backward(torch.ones_like(out) if w.reduction == "none" else None)
                used[k % 2].record(compute)
                _ = out.sum().item()  # device -> host read of the step's result

        run_steps(2)
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(compute)
        run_steps(args.e2e_steps)
        e1.record(compute)
        torch.cuda.synchronize()
        e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1e3, world, dev)
        copied_what = "E, C and targets" if copy_c else "E and targets (C stays on the device)"
        return {"value": weak_scaling_value(world, N, args.e2e_steps, e2e_s), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
                "path": f"linear_cross_entropy(e, c, targets) + backward; each step's {copied_what} copied from "
                        "pinned host memory on a copy stream while the previous step computes; loss read back "
                        "every step"}

    e2e = e2e_resident = None
    if not args.no_e2e:
        e2e = measure_e2e(copy_c=True)
        e2e_resident = measure_e2e(copy_c=False)

    # Context, not the product (the pages' own comparison): the logits materialised in bf16 by a
    # cuBLAS matmul and torch's cross_entropy, forward and backward through autograd, on the same
    # inputs, timed like the steps above (L2 flushed between steps).
    def measure_torch_ce(steps=5, warmup=2):
        e_, c_ = E.detach().requires_grad_(True), C.detach().requires_grad_(True)

        def run():
            logits = e_ @ c_.t()
            loss = torch.nn.functional.cross_entropy(logits, t, ignore_index=-100, reduction=w.reduction)
            loss.backward(g if w.reduction == "none" else None)
            e_.grad = c_.grad = None

        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats(dev)
        base = torch.cuda.memory_allocated(dev)
        try:
            for _ in range(warmup):
                run()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
            for k in range(steps):
                flush.fill_(k & 0xFF)
                evs[k][0].record()
                run()
                evs[k][1].record()
            torch.cuda.synchronize()
        except torch.cuda.OutOfMemoryError:
            return {"skipped": "out of memory"}
        ms = [a.elapsed_time(b) for a, b in evs]
        return {"value": N * steps / (sum(ms) / 1e3), "unit": "tokens/s", "ms_per_step": statistics.mean(ms),
                "ms_per_step_median": statistics.median(ms), "steps": steps,
                "peak_extra_bytes": torch.cuda.max_memory_allocated(dev) - base,
                "what": "bf16 logits E @ C.T (cuBLAS) + torch.nn.functional.cross_entropy, forward + backward "
                        "through autograd; context, not a target"}

    comparators = None
    if world == 1 and not args.no_compare:
        comparators = {"torch_standard_ce": measure_torch_ce()}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        rows = args.cpu_rows
        secs = oracle_sample_seconds(inp, rows)
        cpu = {"value": rows / secs, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
               "sample": f"first {rows} of {N} tokens, full V={V} and D={D}, fp64 forward + backward, {secs:.1f} s"}

    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_config(w, world, (N, D, V)),
        "ms_per_step_median": statistics.median(step_ms), "ms_per_step_min": min(step_ms),
        "ms_per_step_each": [round(x, 4) for x in step_ms],
        "tensor_peak_frac": {"achieved_tflops": path_tflops, "peak": peak_tf, "frac": path_tflops / peak_tf,
                             "frac_sustained": path_tflops / peak_sus, "peak_sustained": peak_sus,
                             "peak_kind": f"bf16_tflops ({peak_kind})",
                             "flops_per_step": fwd_flop + bwd_flop, "kept_tiles": kept, "filtered_tiles": filtered},
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": dom_flop / dom_ms / 1e9, "peak": peak_tf,
                     "unit": "TFLOP/s", "frac": dom_flop / dom_ms / 1e9 / peak_tf,
                     "frac_sustained": dom_flop / dom_ms / 1e9 / peak_sus,
                     "traffic": dom_traffic,
                     "traffic_source": None if dom_traffic is None else f"ncu capture of {dom} at this shape, "
                                                                       f"sources sha256 {kernel_source_hash(dom)[:12]}",
                     "peak_kind": f"bf16_tflops ({peak_kind}, burst; the kernel is timed alone)",
                     "algorithmic_flops_per_launch": dom_flop},
        "kernels": kernels,
        "memory": memory,
        "clocks": clocks,
        "gpu_launches": launches,
        "e2e": e2e,
        "e2e_classifier_resident": e2e_resident,
        "cpu_baseline": cpu,
        "comparators": comparators,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=int(os.environ.get("WORLD_SIZE", "1")))
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama3.1-8b-head")
    ap.add_argument("--shape", default=None,
                    help="N,D,V override of the workload's sizes (profiling captures on a smaller case)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-rows", type=int, default=1536)
    ap.add_argument("--ref-rows", type=int, default=128)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-compare", action="store_true", help="skip the torch standard cross-entropy comparator")
    ap.add_argument("--no-cpu", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
        return
    world, rank, local = dist_setup()
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
