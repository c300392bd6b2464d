#!/usr/bin/env python
"""Throughput of the Q-GaLore optimizer step on B200: INT8 weights updated per second.

Workload: a LLaMA-7B-shaped stack, 32 decoder layers x {q, k, v, o: 4096 x 4096;
gate, up: 4096 x 11008; down: 11008 x 4096}, rank r = 1024: 224 weight matrices,
6.48 G INT8 weights.  One step = the optimizer step a1..a5 on every matrix
(dequantize INT4 P, R = P^T G, Adam on the INT8 moments, U = P N, stochastic
rounding into INT8 W), issued as one batched call for the whole stack (inside
it, batches of 8 matrices, three launches each: the INT4 dequantization and two
tcgen05 GEMMs, alternating between two streams).  Inputs are
seeded synthetic bf16 gradients (rank-256 signal, s_i = 1e-2 * 0.97^i, noise
sigma = 1e-4) resident in HBM (13 GB, far larger than L2).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank updates its own full stack (weak scaling, no
collective on the data path); rank 0 prints one JSON line.

Variants of the stack workload, by environment (the workload name says which ran):
    QG_BENCH_SIDE=right-tall   project matrices with m > n on the right (P n x r)
    QG_BENCH_W_RESCALE=1       weight groups leaving the INT8 grid grow their scale
    QG_BENCH_PER_LAYER=1       one qg_step_batch call per decoder layer, one stream
A run still going after QG_BENCH_WATCHDOG_S seconds (default 1800) ends itself.
Other workloads: --workload llama1b-stack | llama60m-stack | refresh-stress |
linear-grad-stress | linear-7b | linear-7b-decode.
"""
from __future__ import annotations

import argparse
import csv
import datetime
import io
import json
import math
import os
import statistics
import subprocess
import sys
import time
from ctypes import byref, c_int64, c_void_p

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Q-GaLore step: INT8 weights updated/s at 7B shapes; % of step roofline"
UNIT = "weights/s"
WORKLOAD = "llama7b-stack-r1024"
R_RANK = 1024
L2_BYTES = 126 << 20


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=None, help="decoder layers (default: the stack's own count)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=16, help="linear-7b-decode: tokens of the headline line (1..64)")
    ap.add_argument("--workload", choices=sorted(STACKS) + ["refresh-stress", "linear-grad-stress", "linear-7b",
                                                            "linear-7b-decode"],
                    default="llama7b-stack",
                    help="a decoder stack (llama7b-stack is the default and the headline); refresh-stress: "
                         "one 4096 x 11008 layer, r = 1024, a drifting gradient subspace, subspace refreshes on "
                         "the layer-adaptive schedule (--steps defaults to 2000); linear-grad-stress: the same "
                         "layer and schedule with G = D^T X of a linear layer over 8192 tokens whose output-"
                         "gradient subspace turns for 600 steps and then settles; linear-7b: the INT8-weight "
                         "forward and backward products of the LLaMA-7B stack's 224 linear layers at 8192 tokens; "
                         "linear-7b-decode: Y = X W~^T of the same 224 INT8 weights for a few tokens, W read once")
    return ap.parse_args()


# Decoder stacks: hidden size, MLP size, layers, projection rank r, and the
# synthetic gradient's signal (rank, s0, decay of s_i = s0 decay^i, noise sigma).
STACKS = {
    "llama7b-stack": dict(hidden=4096, inter=11008, layers=32, rank=1024, sig=(256, 1e-2, 0.97, 1e-4)),
    "llama1b-stack": dict(hidden=2048, inter=5461, layers=24, rank=512, sig=(256, 1e-2, 0.97, 1e-4)),
    "llama60m-stack": dict(hidden=512, inter=1376, layers=8, rank=128, sig=(64, 1e-2, 0.8, 1e-4)),
}


def stack_shapes(layers, hidden=4096, inter=11008):
    per = [(hidden, hidden)] * 4 + [(hidden, inter)] * 2 + [(inter, hidden)]
    return [per for _ in range(layers)]


KERNEL_SOURCES = ["qg_step.cu", "qg_gemm.cuh", "qg_device.cuh", "qg_philox.cuh", "qg_exact.cuh"]
PROFILE = os.path.join(ROOT, "profiles", "step_kernels_llama7b_layer_ncu.md")
FUSED_SOURCES = ["qg_linear.cu", "qg_device.cuh"]
FUSED_PROFILE = os.path.join(ROOT, "profiles", "linear_forward_int8_llama7b_decode_ncu.md")


def kernel_digest(sources=KERNEL_SOURCES):
    import hashlib
    h = hashlib.sha256()
    for f in sources:
        with open(os.path.join(ROOT, "quantized_rank_gradient_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, alg_bytes_per_launch, profile=PROFILE, sources=KERNEL_SOURCES):
    """DRAM bytes per launch of `kernel`: the ratio of measured DRAM traffic to
    algorithmic bytes in the committed ncu capture, times this run's
    algorithmic bytes per launch.  For the step kernels the ratio is taken
    from one launch of the same kernel, the 7-matrix batch of one decoder
    layer; for the fused INT8 forward, from the four launches of one decoder
    layer.  Traffic grows in proportion to the bytes a launch reads.  None when
    the kernel sources changed since that capture."""
    try:
        text = open(profile).read()
    except OSError:
        return None
    digest = ratio = None
    for line in text.splitlines():
        if line.startswith("kernel sources digest:"):
            digest = line.split(":", 1)[1].strip()
        if line.startswith("traffic_over_algorithmic:"):
            ratio = dict(kv.split("=") for kv in line.split(":", 1)[1].split())
    if digest != kernel_digest(sources) or not ratio or kernel not in ratio:
        return None
    return float(ratio[kernel]) * alg_bytes_per_launch


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained", d["bf16_tflops"]), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id):
        self.bus_id = bus_id
        self.proc = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.bus_id:
            cmd += ["-i", self.bus_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def bus_id_of(dev):
    import torch
    try:
        p = torch.cuda.get_device_properties(dev)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        return None


# ---------------------------------------------------------------- CPU oracle sample

def oracle_sample_seconds(cols, seed=1):
    """One oracle step on a 4096 x `cols` column slice of a 4096 x 4096 (r = 1024)
    matrix.  Columns are independent in every stage of the step, so the weights
    per second of a slice equal those of the full matrix."""
    import numpy as np

    import oracle as O
    import synth
    m, r = 4096, R_RANK
    oc = O.Config(m=m, n=cols, r=r, seed=seed)
    st = O.LayerState.create(oc, synth.weight_codes(m, cols, seed), synth.weight_scales(m, cols, seed=seed))
    O.set_projection(st, synth.orthonormal(m, r, seed))
    G = O.bf16_round((np.random.default_rng(seed).standard_normal((m, cols)) * 1e-4).astype(np.float32))
    t0 = time.perf_counter()
    O.step(st, G)
    return time.perf_counter() - t0


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(cols=2048):
    t = oracle_sample_seconds(cols)
    return {"value": 4096 * cols / t, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
            "sample": f"one oracle step on a 4096x{cols} column slice of a 4096x4096 r=1024 matrix "
                      f"({t:.1f} s); columns are independent, so weights/s carry over",
            "host_cpus": os.cpu_count()}


def cpu_baseline_forward(T, m=4096, n=4096, reps=3, seed=1):
    """The oracle's forward for a few tokens, W~ = bf16(q s) then Y = X W~^T in
    float64, on one 4096 x 4096 matrix, `reps` times (INT8 weights per second)."""
    import numpy as np

    import oracle as O
    import synth
    Wq = synth.weight_codes(m, n, seed)
    sW = synth.weight_scales(m, n, seed=seed)
    X = O.bf16_round(np.random.default_rng(seed).standard_normal((T, n)).astype(np.float32))
    t0 = time.perf_counter()
    for _ in range(reps):
        O.linear_forward(X, O.dequant_weight_bf16(Wq, sW))
    t = time.perf_counter() - t0
    return {"value": reps * m * n / t, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
            "sample": f"{reps} oracle forwards (dequantize, then a float64 product) of one {m}x{n} INT8 matrix "
                      f"at T = {T} ({t:.1f} s)", "host_cpus": os.cpu_count()}


# ---------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    if rank != 0:
        return 0
    cols = 512
    for _ in range(args.warmup):
        oracle_sample_seconds(cols)
    ts = [oracle_sample_seconds(cols, seed=3 + k) for k in range(args.steps)]
    ms = 1000.0 * sum(ts) / len(ts)
    value = 4096 * cols / (ms / 1000.0)
    cores = oracle_threads()
    sample = f"each step: one oracle step on a 4096x{cols} column slice of a 4096x4096 r=1024 matrix"
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64/f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": sample}, "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our arm

class Stack:
    """The 7B stack on one GPU: per matrix W, W scales, state, gradient."""

    def __init__(self, layers, rank, device, spec=None):
        import torch

        import quantized_rank_gradient_b200 as qg
        import synth
        self.qg = qg
        self.device = device
        self.layers = []
        self.keep = []
        stream = c_void_p(torch.cuda.current_stream().cuda_stream)
        spec = spec or STACKS["llama7b-stack"]
        R = spec["rank"]
        self.rank_r = R
        lid = 0
        # QG_BENCH_SIDE=right-tall projects matrices with m > n on the right
        # (P n x r), as GaLore does; the default projects every matrix on the left
        right_tall = os.environ.get("QG_BENCH_SIDE") == "right-tall"
        # QG_BENCH_W_RESCALE=1 lets a weight group that the update would carry off
        # the INT8 grid grow its scale instead of saturating
        w_rescale = 1 if os.environ.get("QG_BENCH_W_RESCALE") == "1" else 0
        self.variant = ("-right-tall" if right_tall else "") + ("-wrescale" if w_rescale else "")
        for li, shapes in enumerate(stack_shapes(layers, spec["hidden"], spec["inter"])):
            group = []
            for (m, n) in shapes:
                seed = matrix_seed(rank, lid)
                side = 1 if (right_tall and m > n) else 0
                c = qg.config(m, n, R, seed=seed, layer_id=lid, proj_side=side, w_rescale=w_rescale)
                ldw = -(-n // 16) * 16
                W = synth.device_weight_codes(m, n, ldw, seed, device)
                sW = synth.device_weight_scales(m, n, seed, device)
                G = synth.device_lowrank_gradient(m, n, *spec["sig"], seed, device)
                state = torch.empty(qg.qg_state_bytes(byref(c)), dtype=torch.uint8, device=device)
                h = c_void_p()
                qg.check(qg.qg_layer_init(byref(h), byref(c), state.data_ptr(), state.numel(), W.data_ptr(), ldw,
                                          sW.data_ptr(), stream), "qg_layer_init")
                # starting projection: an orthonormal basis quantized to INT4 on the device
                g = torch.Generator(device=device)
                g.manual_seed(seed + 17)
                pr = n if side else m
                P = torch.linalg.qr(torch.randn(pr, R, generator=g, device=device))[0].contiguous()
                Pq = torch.empty((pr * R + 1) // 2, dtype=torch.uint8, device=device)
                sP = torch.empty(-(-pr * R // 64), dtype=torch.float32, device=device)
                qg.check(qg.qg_quantize_projection(P.data_ptr(), R, pr, R, Pq.data_ptr(), sP.data_ptr(),
                                                   stream))
                qg.check(qg.qg_layer_set_projection(h, Pq.data_ptr(), sP.data_ptr(), 0, stream))
                torch.cuda.synchronize()
                del P, Pq, sP
                group.append(dict(cfg=c, h=h, W=W, sW=sW, G=G, ldg=G.shape[1], state=state, m=m, n=n, side=side))
                lid += 1
            self.layers.append(group)
        # the step: one batched call for all matrices (batches of 8 on three lanes
        # inside the library), or with QG_BENCH_PER_LAYER=1 one call per decoder
        # layer.  The per-layer calls (the 7 matrices of a layer in one batch, one
        # stream, kernels one after another) also serve the kernel-timing pass.
        whole = [[e for group in self.layers for e in group]]
        self.per_layer_only = os.environ.get("QG_BENCH_PER_LAYER") == "1"
        if self.per_layer_only:
            self.variant += "-per-layer"
        need = 0
        for group in whole + self.layers:
            arr = (qg.POINTER(qg.qg_config) * len(group))(*[qg.ctypes.pointer(e["cfg"]) for e in group])
            need = max(need, qg.qg_step_batch_workspace_bytes(arr, len(group)))
        self.ws = torch.empty(need, dtype=torch.uint8, device=device)

        def calls_of(groups):
            out = []
            for group in groups:
                k = len(group)
                out.append(((c_void_p * k)(*[e["h"].value for e in group]),
                            (c_void_p * k)(*[e["G"].data_ptr() for e in group]),
                            (c_int64 * k)(*[e["ldg"] for e in group]), k))
            return out
        self.calls_layer = calls_of(self.layers)
        self.calls = self.calls_layer if self.per_layer_only else calls_of(whole)
        self.weights = sum(e["m"] * e["n"] for group in self.layers for e in group)
        self.flops = sum(4.0 * e["m"] * e["n"] * R for group in self.layers for e in group)
        self.alg_bytes = sum(alg_bytes(e["m"], e["n"], R, e["side"]) for group in self.layers for e in group)
        self.grad_bytes = sum(e["G"].numel() * 2 for group in self.layers for e in group)

    def step(self, stream, per_layer=False):
        qg = self.qg
        for hs, gs, lds, k in (self.calls_layer if per_layer else self.calls):
            st = qg.qg_step_batch(hs, gs, lds, k, self.ws.data_ptr(), self.ws.numel(), stream)
            if st != qg.QG_OK:
                raise qg.QGError(st, "qg_step_batch")

    def statuses(self):
        return [e["state"] for group in self.layers for e in group]


def matrix_seed(rank, lid):
    """Seed of matrix `lid` of rank `rank`'s stack: every rank updates its own
    independent stack (weak scaling)."""
    return 1_000_003 * (rank + 1) + lid


def reduce_max(value, world):
    """The largest `value` over all ranks (the slowest rank sets the job's time):
    an all-reduce on the process group's device (CUDA for NCCL, host for gloo)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, ms):
    """Units processed by all ranks per second, over the max-over-ranks time."""
    return world * units_per_rank / (ms / 1000.0)


def alg_bytes(m, n, r, side=0):
    """Algorithmic HBM bytes of one matrix step: G, W read and written, W scales,
    INT4 P and scales, moments read and written, their scales.  P is m x r and
    the moments r x n (left projection), or n x r and m x r (right)."""
    p_rows, rows, cols = (n, m, r) if side else (m, r, n)
    nb = -(-cols // 256)
    return (2 * m * n + 2 * m * n + 4 * math.ceil(m * n / 256) + p_rows * r / 2 + 4 * p_rows * r / 64
            + 4 * rows * cols + 16 * rows * nb)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import quantized_rank_gradient_b200 as qg
    qg.lib()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    spec = STACKS[args.workload]
    layers = args.layers or spec["layers"]
    stack = Stack(layers, rank, device, spec)
    stream = c_void_p(torch.cuda.current_stream().cuda_stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        stack.step(stream)
    torch.cuda.synchronize()

    # ---- device-timed region: inputs resident in HBM
    clocks = ClockSampler(bus_id_of(device))
    clocks.start()
    time.sleep(0.3)
    qg.check(qg.qg_profile_enable(1))
    barrier()
    torch.cuda.synchronize()
    flush = None
    if stack.grad_bytes < 2 * L2_BYTES:
        # inputs that fit in L2: each step timed alone, L2 flushed between steps
        # (a 256 MB write outside the timed events)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    if flush is None:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record()
        for _ in range(args.steps):
            stack.step(stream)
        t_end.record()
        torch.cuda.synchronize()
        ms = t_start.elapsed_time(t_end) / args.steps
    else:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for e0, e1 in evs:
            flush.fill_(1)
            e0.record()
            stack.step(stream)
            e1.record()
        torch.cuda.synchronize()
        ms = sum(e0.elapsed_time(e1) for e0, e1 in evs) / args.steps
    barrier()
    kt_run = (qg.qg_kernel_times * qg.QG_KERNEL_KINDS)()
    qg.check(qg.qg_profile_collect(kt_run, qg.QG_KERNEL_KINDS))
    qg.check(qg.qg_profile_enable(0))
    clk = clocks.stop()
    ms = reduce_max(ms, world)

    # ---- kernel durations: in the timed region the lanes' kernels overlap,
    # so a launch's events would also span the other lane's work.  The same
    # kernels on the same data are timed again one after another: one call per
    # decoder layer on one stream (a step counts once more for every matrix's t).
    qg.check(qg.qg_profile_enable(1))
    for _ in range(args.steps):
        stack.step(stream, per_layer=True)
    torch.cuda.synchronize()
    kt = (qg.qg_kernel_times * qg.QG_KERNEL_KINDS)()
    qg.check(qg.qg_profile_collect(kt, qg.QG_KERNEL_KINDS))
    qg.check(qg.qg_profile_enable(0))

    # ---- end to end: gradients copied from pinned host memory every step,
    # the per-matrix status words read back
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(stack, args, stream, world, device, barrier)

    if rank != 0:
        return 0
    peaks = load_peaks()
    value = whole_job_rate(stack.weights, world, ms)
    names = {qg.QG_KERNEL_DEQUANT: "dequant_projection", qg.QG_KERNEL_PROJECT_ADAM: "project_adam_tcgen05",
             qg.QG_KERNEL_BACKPROJECT_SR: "backproject_sround_tcgen05"}
    kernels = {}
    for k, nm in names.items():
        e = kt[k]
        if e.launches:
            kernels[nm] = {"launches_per_step": e.launches / args.steps, "ms_per_step": e.device_ms / args.steps,
                           "avg_launch_ms": e.device_ms / e.launches,
                           "tflops": e.flops / (e.device_ms / 1000.0) / 1e12 if e.flops else None,
                           "gbs": e.bytes / (e.device_ms / 1000.0) / 1e9}
    dom_k = max([qg.QG_KERNEL_PROJECT_ADAM, qg.QG_KERNEL_BACKPROJECT_SR], key=lambda k: kt[k].device_ms)
    dom = kt[dom_k]
    achieved = (dom.flops / dom.launches) / (dom.device_ms / dom.launches / 1000.0) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    launches = sum(kt_run[k].launches for k in range(qg.QG_KERNEL_KINDS)) / args.steps
    t_roof_ms = max(stack.flops / (peaks["bf16_tflops"] * 1e12), stack.alg_bytes / (peaks["hbm_gbs"] * 1e9)) * 1e3
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16/f32/int8",
        "data": "synthetic (seeded low-rank-plus-noise bf16 gradients)",
        "config": {"workload": f"{args.workload}-r{spec['rank']}" + ("" if layers == spec["layers"] else f"-{layers}l")
                   + stack.variant,
                   "matrices": 7 * layers, "weights_per_gpu": stack.weights,
                   "rank": spec["rank"], "l2": "inputs larger than L2 (%.1f GB of gradients per step)"
                   % (stack.grad_bytes / 1e9) if flush is None else "L2 flushed between steps (each step timed alone)",
                   "parallelism": f"independent stacks x{world}"},
        "step_roofline": {"t_roof_ms": t_roof_ms, "frac": t_roof_ms / ms,
                          "bound": "tensor" if stack.flops / (peaks["bf16_tflops"] * 1e12) >
                          stack.alg_bytes / (peaks["hbm_gbs"] * 1e9) else "hbm",
                          "peaks": "burst bf16 %.1f TF/s, HBM %.1f GB/s (%s)" % (peaks["bf16_tflops"], peaks["hbm_gbs"],
                                                                              peaks["source"])},
        "roofline": {"bound": "tensor", "kernel": names[dom_k], "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "traffic": profiled_traffic(names[dom_k], dom.bytes / dom.launches)
                     if args.workload == "llama7b-stack" else None,
                     "traffic_unit": "DRAM bytes per launch (ncu traffic/algorithmic ratio x this launch)",
                     "algorithmic_bytes_per_launch": dom.bytes / dom.launches,
                     "peak_kind": "sustained bf16 (%s)" % peaks["source"]},
        "kernels": kernels,
        "kernels_timing": "a pass after the timed region, one call per decoder layer on one stream, so that "
                          "each launch's events span that kernel alone",
        "gpu_launches": launches * args.steps,
        "clocks": clk,
    }
    if e2e:
        line["e2e"] = e2e
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline()
    print(json.dumps(line), flush=True)
    return 0


def run_refresh_stress(args, rank, world, local_rank):
    """One 4096 x 11008 layer at r = 1024 over `steps` steps (2000 by default):
    the gradient's rank-256 signal subspace (s_i = 1e-2 * 0.97^i, noise 1e-4)
    turns by 0.02 rad per step until step 800, then stays.  Every step runs
    qg_refresh (a randomized top-r SVD and CosSim when the layer is due; the
    interval starts at 200 and doubles when CosSim > 0.4) and then qg_step, both
    timed with CUDA events; the gradient is drawn outside the timed region.

    With --workload linear-grad-stress the gradient is that of a linear layer,
    G = D^T X over B = 8192 tokens (the weight-gradient model of Theorem 3.1):
    X and D draw from principal subspaces of width r; the output-gradient one
    turns by 0.0075 rad per step (1.5 rad between refreshes 200 steps apart)
    until step 600 and then stays.  G is formed by qg_linear_backward_weight,
    outside the timed region."""
    import torch
    import quantized_rank_gradient_b200 as qg
    import synth
    qg.lib()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    steps = args.steps if args.steps != 20 else 2000
    m, n, r = 4096, 11008, R_RANK
    seed = 4_000_037 * (rank + 1)
    c = qg.config(m, n, r, seed=seed, layer_id=0)
    c.delta0, c.gamma = 200, 0.4
    ldw = -(-n // 16) * 16
    W = synth.device_weight_codes(m, n, ldw, seed, device)
    sW = synth.device_weight_scales(m, n, seed, device)
    linear = args.workload == "linear-grad-stress"
    if linear:
        lin = synth.DeviceLinearLayerBatch(m, n, LINEAR_TOKENS, r, 0.999, 1e-3, 0.0075, 600, seed, device)
        ldg_lin = -(-n // 8) * 8
        G_lin = torch.zeros(m, ldg_lin, dtype=torch.bfloat16, device=device)

        class _LinearSource:
            @staticmethod
            def draw(t):
                X, D = lin.draw(t)
                qg.check(qg.qg_linear_backward_weight(D.data_ptr(), lin.ldd, X.data_ptr(), lin.ldx, LINEAR_TOKENS, m,
                                                      n, G_lin.data_ptr(), ldg_lin,
                                                      c_void_p(torch.cuda.current_stream().cuda_stream)),
                         "qg_linear_backward_weight")
                return G_lin
        gen = _LinearSource()
    else:
        gen = synth.DeviceDriftingGradient(m, n, 256, 1e-2, 0.97, 1e-4, 0.02, 800, seed, device)
    cs = torch.cuda.current_stream()
    stream = c_void_p(cs.cuda_stream)
    state = torch.empty(qg.qg_state_bytes(byref(c)), dtype=torch.uint8, device=device)
    h = c_void_p()
    qg.check(qg.qg_layer_init(byref(h), byref(c), state.data_ptr(), state.numel(), W.data_ptr(), ldw,
                              sW.data_ptr(), stream), "qg_layer_init")
    ws = torch.empty(qg.qg_step_workspace_bytes(byref(c)), dtype=torch.uint8, device=device)
    rws = torch.empty(qg.qg_refresh_workspace_bytes(byref(c)), dtype=torch.uint8, device=device)
    info = qg.qg_refresh_info()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    refresh_ms, trace = [], []
    clocks = ClockSampler(bus_id_of(device))
    clocks.start()
    for t in range(steps):
        G = gen.draw(t)
        e0, e1 = ev[t]
        e0.record(cs)
        qg.check(qg.qg_refresh(h, G.data_ptr(), G.shape[1], 1 if t == 0 else 0, rws.data_ptr(), rws.numel(),
                               byref(info), stream), "qg_refresh")
        qg.check(qg.qg_step(h, G.data_ptr(), G.shape[1], ws.data_ptr(), ws.numel(), stream), "qg_step")
        e1.record(cs)
        if info.refreshed:
            trace.append({"t": t, "cossim": round(float(info.cossim), 4) if info.has_cossim else None,
                          "delta": int(info.delta), "t_next": int(info.t_next)})
    torch.cuda.synchronize()
    clk = clocks.stop()
    st = qg.qg_layer_status(h, stream)
    ms = [a.elapsed_time(b) for a, b in ev]
    for item in trace:
        refresh_ms.append(ms[item["t"]])
    total_ms = reduce_max(sum(ms), world)
    plain = sorted(ms[t] for t in range(steps) if t not in {i["t"] for i in trace})
    if rank != 0:
        return 0
    value = whole_job_rate(steps * m * n, world, total_ms)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps, "warmup": 0,
            "ms_per_step": total_ms / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16/f32/int8",
            "data": "synthetic (linear-layer gradients G = D^T X over 8192 tokens)" if linear
            else "synthetic (drifting low-rank-plus-noise bf16 gradients)",
            "config": {"workload": ("linear-grad-stress-4096x11008-r1024-B8192" if linear
                                    else "refresh-stress-4096x11008-r1024"),
                       "steps": steps, "delta0": 200, "gamma": 0.4,
                       "drift": ("output-gradient subspace turns 0.0075 rad/step, frozen after step 600" if linear
                                 else "0.02 rad/step, frozen after step 800"),
                       "l2": "gradient redrawn every step outside the timed region"},
            "refreshes": len(trace), "svd_fraction_vs_fixed_interval": len(trace) / max(1, -(-steps // 200)),
            "refresh_ms": {"mean": sum(refresh_ms) / max(1, len(refresh_ms)), "max": max(refresh_ms or [0.0])},
            "step_ms_median_without_refresh": plain[len(plain) // 2] if plain else None,
            "cossim_trace": trace, "status": int(st), "clocks": clk}
    print(json.dumps(line), flush=True)
    qg.qg_layer_destroy(h)
    return 0


LINEAR_TOKENS = 8192


def run_linear(args, rank, world, local_rank):
    """The INT8-weight linear layers around the optimizer (simulated weight-only
    quantization), LLaMA-7B stack at 8192 tokens.  One step runs, for each of the
    224 weight matrices, W~ = bf16(q s), Y = X W~^T, dX = D_y W~ and G = D_y^T X
    through the C ABI on one stream.  Each matrix has its own INT8 weight and
    scales.  Activations and output gradients are seeded synthetic bf16 matrices,
    one set per layer shape, all larger than L2 together with a matrix's weight.
    Every rank runs its own stack (weak scaling)."""
    import torch
    import torch.distributed as dist

    import quantized_rank_gradient_b200 as qg
    import synth
    qg.lib()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    spec = STACKS["llama7b-stack"]
    layers = args.layers or spec["layers"]
    T = LINEAR_TOKENS
    stream = c_void_p(torch.cuda.current_stream().cuda_stream)
    shapes = [s for group in stack_shapes(layers, spec["hidden"], spec["inter"]) for s in group]
    mats = []
    for lid, (m, n) in enumerate(shapes):
        seed = matrix_seed(rank, lid)
        ldw = -(-n // 16) * 16
        mats.append((m, n, synth.device_weight_codes(m, n, ldw, seed, device), ldw,
                     synth.device_weight_scales(m, n, seed, device)))
    gen = torch.Generator(device=device)
    gen.manual_seed(4_000_117 * (rank + 1))
    bufs = {}
    for (m, n) in sorted(set(shapes)):
        bf = torch.bfloat16
        bufs[(m, n)] = dict(X=torch.randn(T, n, generator=gen, device=device).to(bf),
                            D=(torch.randn(T, m, generator=gen, device=device) * 1e-2).to(bf),
                            Y=torch.empty(T, m, dtype=bf, device=device), dX=torch.empty(T, n, dtype=bf, device=device),
                            G=torch.empty(m, n, dtype=bf, device=device),
                            Wt=torch.empty(m, -(-n // 8) * 8, dtype=bf, device=device))

    def step():
        for (m, n, W, ldw, sW) in mats:
            b = bufs[(m, n)]
            ldt = b["Wt"].shape[1]
            qg.check(qg.qg_linear_dequant_weight(W.data_ptr(), ldw, sW.data_ptr(), m, n, b["Wt"].data_ptr(), ldt,
                                                 stream), "qg_linear_dequant_weight")
            qg.check(qg.qg_linear_forward(b["X"].data_ptr(), n, b["Wt"].data_ptr(), ldt, T, m, n, b["Y"].data_ptr(),
                                          m, stream), "qg_linear_forward")
            qg.check(qg.qg_linear_backward_data(b["D"].data_ptr(), m, b["Wt"].data_ptr(), ldt, T, m, n,
                                                b["dX"].data_ptr(), n, stream), "qg_linear_backward_data")
            qg.check(qg.qg_linear_backward_weight(b["D"].data_ptr(), m, b["X"].data_ptr(), n, T, m, n,
                                                  b["G"].data_ptr(), n, stream), "qg_linear_backward_weight")

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(bus_id_of(device))
    clocks.start()
    time.sleep(0.3)
    qg.check(qg.qg_profile_enable(1))
    barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / args.steps
    barrier()
    kt = (qg.qg_kernel_times * qg.QG_KERNEL_KINDS)()
    qg.check(qg.qg_profile_collect(kt, qg.QG_KERNEL_KINDS))
    qg.check(qg.qg_profile_enable(0))
    clk = clocks.stop()
    ms = reduce_max(ms, world)
    if rank != 0:
        return 0
    peaks = load_peaks()
    flops = sum(6.0 * T * m * n for (m, n, *_rest) in mats)
    gemm, deq = kt[qg.QG_KERNEL_LINEAR_GEMM], kt[qg.QG_KERNEL_LINEAR_DEQUANT]
    achieved = (gemm.flops / gemm.launches) / (gemm.device_ms / gemm.launches / 1000.0) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    line = {
        "metric": "INT8-weight linear layers, forward + backward (Y = X W~^T, dX = D_y W~, G = D_y^T X): TFLOP/s",
        "value": flops / (ms / 1000.0) / 1e12 * world, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 operands (W~ from INT8), f32 accumulate", "data": "synthetic (seeded bf16 activations and "
        "output gradients; seeded INT8 weights and scales)",
        "config": {"workload": f"linear-llama7b-stack-{T}tok" + ("" if layers == spec["layers"] else f"-{layers}l"),
                   "matrices": len(mats), "tokens": T, "weights_per_gpu": sum(m * n for (m, n, *_r) in mats),
                   "l2": "inputs larger than L2 (a matrix's weight and activations exceed 126 MB)",
                   "parallelism": f"independent stacks x{world}"},
        "tokens_per_s": T / (ms / 1000.0) * world,
        "roofline": {"bound": "tensor", "kernel": "linear_gemm_tcgen05", "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None,
                     "peak_kind": "sustained bf16 (%s)" % peaks["source"]},
        "kernels": {"linear_dequant_weight": {"launches_per_step": deq.launches / args.steps,
                                              "ms_per_step": deq.device_ms / args.steps,
                                              "gbs": deq.bytes / (deq.device_ms / 1000.0) / 1e9},
                    "linear_gemm_tcgen05": {"launches_per_step": gemm.launches / args.steps,
                                            "ms_per_step": gemm.device_ms / args.steps, "tflops": achieved}},
        "gpu_launches": (gemm.launches + deq.launches),
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


DECODE_TOKENS = (1, 4, 8, 16, 32, 64)


def run_linear_decode(args, rank, world, local_rank):
    """The forward product Y = X W~^T of the LLaMA-7B stack's INT8 weights for a
    few tokens (--tokens, default 16; the line also sweeps T = 1 to 64).

    The weights are laid out as decoders run them for inference: per layer the
    q, k and v weights stacked in one 12288 x 4096 buffer and gate and up in one
    22016 x 4096 buffer (the matrices of a stack read the same input), o and down
    alone, each buffer's group scales the concatenation of its matrices' (the
    groups never straddle two matrices, n % 256 == 0).  The optimizer still sees
    each matrix as a row slice of its buffer.  One step runs
    qg_linear_forward_int8 once per buffer (4 per layer, 128 launches), each
    INT8 weight read once and dequantized in registers.  Beside it, on the same
    buffers: the two-step path (qg_linear_dequant_weight into a bf16 scratch,
    then the tcgen05 qg_linear_forward), and the fused kernel once per matrix
    (224 launches).  The weights (6.5 GB) are larger than L2, so every step reads
    them from HBM.  Every rank runs its own stack (weak scaling)."""
    import torch
    import torch.distributed as dist

    import quantized_rank_gradient_b200 as qg
    import synth
    qg.lib()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    spec = STACKS["llama7b-stack"]
    layers = args.layers or spec["layers"]
    if not 1 <= args.tokens <= 64:
        raise SystemExit("--tokens must be in 1..64")
    stream = c_void_p(torch.cuda.current_stream().cuda_stream)
    h, f = spec["hidden"], spec["inter"]
    # per layer: (rows of each stacked matrix, n)
    layout = [((h, h, h), h), ((h,), h), ((f, f), h), ((h,), f)]
    bufs, mats = [], []
    for layer in range(layers):
        for bi, (rows, n) in enumerate(layout):
            m = sum(rows)
            ldw = -(-n // 16) * 16
            seed = matrix_seed(rank, layer * len(layout) + bi)
            W = synth.device_weight_codes(m, n, ldw, seed, device)
            sW = synth.device_weight_scales(m, n, seed, device)
            bufs.append((m, n, W, ldw, sW))
            r0 = 0
            for r in rows:  # the matrices as row slices of the buffer
                mats.append((r, n, W[r0:], ldw, sW[(r0 * n) // 256:]))
                r0 += r
    gen = torch.Generator(device=device)
    gen.manual_seed(5_000_011 * (rank + 1))
    bf = torch.bfloat16
    shapes = sorted({(m, n) for (m, n, *_r) in bufs} | {(m, n) for (m, n, *_r) in mats})
    io = {(m, n): dict(X=torch.randn(64, n, generator=gen, device=device).to(bf),
                       Y=torch.empty(64, m, dtype=bf, device=device),
                       Wt=torch.empty(m, -(-n // 8) * 8, dtype=bf, device=device))
          for (m, n) in shapes}

    def fused(T, items=bufs):
        for (m, n, W, ldw, sW) in items:
            b = io[(m, n)]
            qg.check(qg.qg_linear_forward_int8(b["X"].data_ptr(), n, W.data_ptr(), ldw, sW.data_ptr(), T, m, n,
                                               b["Y"].data_ptr(), m, stream), "qg_linear_forward_int8")

    def per_matrix(T):
        fused(T, mats)

    def two_step(T):
        for (m, n, W, ldw, sW) in bufs:
            b = io[(m, n)]
            ldt = b["Wt"].shape[1]
            qg.check(qg.qg_linear_dequant_weight(W.data_ptr(), ldw, sW.data_ptr(), m, n, b["Wt"].data_ptr(), ldt,
                                                 stream), "qg_linear_dequant_weight")
            qg.check(qg.qg_linear_forward(b["X"].data_ptr(), n, b["Wt"].data_ptr(), ldt, T, m, n, b["Y"].data_ptr(),
                                          m, stream), "qg_linear_forward")

    def barrier():
        if world > 1:
            dist.barrier()

    def timed(fn, T, steps, warmup, profile=False):
        for _ in range(warmup):
            fn(T)
        barrier()
        torch.cuda.synchronize()
        if profile:
            qg.check(qg.qg_profile_enable(1))
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(steps):
            fn(T)
        t1.record()
        torch.cuda.synchronize()
        kt = None
        if profile:
            kt = (qg.qg_kernel_times * qg.QG_KERNEL_KINDS)()
            qg.check(qg.qg_profile_collect(kt, qg.QG_KERNEL_KINDS))
            qg.check(qg.qg_profile_enable(0))
        barrier()
        return reduce_max(t0.elapsed_time(t1) / steps, world), kt

    weights = sum(m * n for (m, n, *_r) in bufs)
    T = args.tokens
    clocks = ClockSampler(bus_id_of(device))
    clocks.start()
    time.sleep(0.3)
    ms, _ = timed(fused, T, args.steps, args.warmup)
    clk = clocks.stop()
    # per-launch device times (events around each launch) from a separate pass,
    # so that the headline time carries no profiling events
    _, kt = timed(fused, T, max(3, args.steps // 4), 1, profile=True)
    sweep = {}
    for Ts in DECODE_TOKENS:
        n_steps = max(3, args.steps // 4)
        f_ms, _ = timed(fused, Ts, n_steps, args.warmup)
        p_ms, _ = timed(per_matrix, Ts, n_steps, args.warmup)
        t_ms, _ = timed(two_step, Ts, n_steps, args.warmup)
        sweep[str(Ts)] = {"fused_ms": f_ms, "fused_per_matrix_ms": p_ms, "two_step_ms": t_ms,
                          "speedup_vs_two_step": t_ms / f_ms, "fused_tbs": weights / (f_ms / 1000.0) / 1e12}
    if rank != 0:
        return 0
    peaks = load_peaks()
    k = kt[qg.QG_KERNEL_LINEAR_FUSED]
    achieved = (k.bytes / k.launches) / (k.device_ms / k.launches / 1000.0) / 1e9
    line = {
        "metric": "INT8-weight forward for a few tokens (Y = X W~^T, W read once): INT8 weights/s",
        "value": weights / (ms / 1000.0) * world, "unit": "weights/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "INT8 weights, bf16 activations, f32 accumulate, bf16 out",
        "data": "synthetic (seeded bf16 activations; seeded INT8 weights and scales)",
        "config": {"workload": f"linear-llama7b-stack-decode-{T}tok" + ("" if layers == spec["layers"]
                                                                       else f"-{layers}l"),
                   "buffers": len(bufs), "matrices": len(mats), "tokens": T, "weights_per_gpu": weights,
                   "layout": "per layer: qkv 12288x4096, o 4096x4096, gate_up 22016x4096, down 4096x11008",
                   "l2": "inputs larger than L2 (6.5 GB of INT8 weights per step)",
                   "parallelism": f"independent stacks x{world}"},
        "roofline": {"bound": "hbm", "kernel": "linear_forward_int8", "achieved": achieved,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": profiled_traffic("linear_forward_int8", k.bytes / k.launches, FUSED_PROFILE,
                                                 FUSED_SOURCES),
                     "traffic_unit": "DRAM bytes per launch (ncu traffic/algorithmic ratio x this launch)",
                     "algorithmic_bytes_per_launch": k.bytes / k.launches,
                     "peak_kind": "HBM copy (%s)" % peaks["source"]},
        "kernels": {"linear_forward_int8": {"launches_per_step": len(bufs),
                                            "device_ms_per_launch": k.device_ms / k.launches, "gbs": achieved}},
        "tokens_sweep": sweep,
        "gpu_launches": len(bufs) * args.steps,
        "clocks": clk,
    }
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline_forward(T)
    print(json.dumps(line), flush=True)
    return 0


def run_e2e(stack, args, stream, world, device, barrier):
    import torch
    import torch.distributed as dist
    qg = stack.qg
    # one pinned host gradient per distinct shape; every matrix's gradient is
    # copied from host memory each step
    host = {}
    for group in stack.layers:
        for e in group:
            key = tuple(e["G"].shape)
            if key not in host:
                host[key] = e["G"].cpu().pin_memory()
    status_host = torch.zeros(sum(len(g) for g in stack.layers), dtype=torch.int32).pin_memory()
    views = []
    for group in stack.layers:
        for e in group:
            v = qg.qg_layer_views()
            qg.check(qg.qg_layer_views_get(e["h"], byref(v)))
            off = v.status - e["state"].data_ptr()
            views.append(e["state"][off: off + 4].view(torch.int32))
    h2d = sum(e["G"].numel() * 2 for group in stack.layers for e in group)
    d2h = 4 * len(views)
    # The copies run on their own stream, one decoder layer at a time; the
    # layer's qg_step_batch call waits for its own copy only, so the host link
    # and the step overlap (the step of layer i runs while layer i + 1 is
    # copied).  A layer's gradient buffers are rewritten only after the
    # previous step's call on that layer has consumed them.
    comp = torch.cuda.current_stream()
    copy_stream = torch.cuda.Stream(device=device)
    nl = len(stack.layers)
    copied = [torch.cuda.Event() for _ in range(nl)]
    consumed = [torch.cuda.Event() for _ in range(nl)]
    start = torch.cuda.Event()

    def one():
        start.record(comp)
        copy_stream.wait_event(start)
        with torch.cuda.stream(copy_stream):
            for li, group in enumerate(stack.layers):
                copy_stream.wait_event(consumed[li])
                for e in group:
                    e["G"].copy_(host[tuple(e["G"].shape)], non_blocking=True)
                copied[li].record(copy_stream)
        for li, (hs, gs, lds, k) in enumerate(stack.calls_layer):
            comp.wait_event(copied[li])
            st = qg.qg_step_batch(hs, gs, lds, k, stack.ws.data_ptr(), stack.ws.numel(), stream)
            if st != qg.QG_OK:
                raise qg.QGError(st, "qg_step_batch")
            consumed[li].record(comp)
        for j, v in enumerate(views):
            status_host[j: j + 1].copy_(v, non_blocking=True)
        comp.synchronize()
        if int(status_host.max()) != 0:
            raise RuntimeError("device status word set during the e2e run")

    one()
    steps = max(2, min(args.steps, 5))
    barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        one()
    t1.record()
    torch.cuda.synchronize()
    barrier()
    ms = reduce_max(t0.elapsed_time(t1) / steps, world)
    return {"value": whole_job_rate(stack.weights, world, ms), "unit": UNIT, "ms_per_step": ms, "steps": steps,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "note": "bf16 gradients copied from pinned host memory each step, layer by layer on a copy stream "
                    "overlapping the per-layer qg_step_batch calls; status words read back"}


def start_watchdog():
    """A run that has not ended after QG_BENCH_WATCHDOG_S seconds (default 1800;
    the default run takes one to two minutes) is stuck, most likely in a CUDA
    call that waits for a kernel: a daemon thread then ends the process, which
    also releases its GPU context."""
    import threading
    limit = float(os.environ.get("QG_BENCH_WATCHDOG_S", "1800"))
    if limit <= 0:
        return

    def fire():
        sys.stderr.write(f"bench.py: no result after {limit:.0f} s; exiting\n")
        sys.stderr.flush()
        os._exit(3)

    t = threading.Timer(limit, fire)
    t.daemon = True
    t.start()


def main():
    args = parse_args()
    start_watchdog()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.workload in ("refresh-stress", "linear-grad-stress"):
            return run_refresh_stress(args, rank, world, local_rank)
        if args.workload == "linear-7b":
            return run_linear(args, rank, world, local_rank)
        if args.workload == "linear-7b-decode":
            return run_linear_decode(args, rank, world, local_rank)
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
