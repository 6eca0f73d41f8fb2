#!/usr/bin/env python3
"""Benchmark of the packed INT-b decode path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mine|reference]

Workload (the decode GEMV sweep): W 4096x4096 fp32 ~ N(0, 0.02^2) with 0.1%
outliers x20, quantized per row to b = 6 bits (the headline width; the whole
sweep b in {4,5,6,7,8,10,12} x M in {1,4,16} is reported beside it), x bf16
M = 1.  One step is one decode pass over a pool of distinct packed copies of
the matrix (more than 4x the L2 size, so no step reads from L2), one fused
dequantize-GEMV launch per copy, captured in a CUDA graph.

value = packed-weight bytes (codes + scales) streamed per second, whole job.
Everything else on the JSON line (sweep, quantizer, 27B-class MLP matrices,
tensor-core prefill, mixed-bit recipe pass, e2e through host buffers, the
oracle's CPU time, SM clocks) is measured in the same run.

Multi-GPU: the decode pass does not shard; each rank runs an independent
replica and value is the sum over ranks of the work, divided by the slowest
rank's time ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

HEADLINE_BITS = 6
DECODE_BITS = [4, 5, 6, 7, 8, 10, 12]
DECODE_MS = [1, 4, 16]
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
METRIC = "packed b-bit dequant-GEMV GB/s and % HBM peak at M=1; prefill TFLOP/s"


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# Sources whose change invalidates a committed DRAM-traffic figure for the
# decode kernel that the headline times.
TMA_GEMV_SOURCES = ["gemv_tma.cuh", "gemv_tma_dispatch.cuh", "gemv_tma.cu", "gemv_tma_canon.cu",
                    "expand.cuh", "tc_ptx.cuh"]


def kernel_source_hash(names):
    h = hashlib.sha256()
    for n in names:
        h.update(open(os.path.join(ROOT, "mixed_precision_weight_row_b200", "csrc", n), "rb").read())
    return h.hexdigest()[:16]


def profile_traffic(profile_name, source_files, launches_bytes_scale=1.0):
    """DRAM bytes per launch from a committed ncu summary, if still current."""
    p = os.path.join(ROOT, "profiles", profile_name)
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
    except Exception:
        return None
    if d.get("source_hash") != kernel_source_hash(source_files):
        return None
    return float(d["dram_bytes_per_launch"]) * launches_bytes_scale


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", self.uuid],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.15)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    rows.append((float(parts[0]), float(parts[1]), parts[2], parts[3], parts[4:8]))
                except ValueError:
                    continue
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = sorted(r[0] for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[4]) if v.lower() == "active"})
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl != "reference":
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(v, world, device="cuda"):
    """The largest v over the ranks (every rank gets it)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, units_per_rank_step, max_ms_per_step):
    """Units per second of the whole job: every rank processes the same units
    per step (weak scaling) and the slowest rank sets the time."""
    return world * units_per_rank_step / (max_ms_per_step * 1e-3)


# ----------------------------------------------------------------------------
# GPU measurements
# ----------------------------------------------------------------------------

class Pool:
    """P distinct device copies of one packed matrix (P * bytes > 4 x L2)."""

    def __init__(self, packed, scales, min_bytes):
        import torch

        per = packed.numel() + scales.numel() * 4
        self.P = max(2, -(-min_bytes // per))
        self.packed = [packed.clone() for _ in range(self.P)]
        self.scales = [scales.clone() for _ in range(self.P)]
        self.bytes_each = per
        torch.cuda.synchronize()


# Where a code in the device error word comes from: 100 * kernel + place.
WAIT_KERNELS = {1: "gemv_tma_kernel", 2: "gemv_tc_kernel", 3: "gemm_kernel", 4: "gemv_sk_kernel",
                5: "gemm_fp8_kernel"}
WAIT_PLACES = {1: "x producer: free x stage", 2: "x producer: last copies", 3: "producer: free stage",
               4: "producer: last copies", 5: "consumer / MMA issuer: loaded stage",
               6: "MMA issuer: converted weights", 7: "converter: loaded weight stage",
               8: "converter: free tensor-memory stage", 9: "epilogue: accumulator",
               10: "sums of squares: loaded x stage"}


def describe_wait_code(code):
    k, p = divmod(int(code), 100)
    return f"{WAIT_KERNELS.get(k, f'kernel {k}')}, {WAIT_PLACES.get(p, f'place {p}')}"


class Sections:
    """Runs the bench's measurements one by one.  After each one the device
    error word is read (and cleared), so that a wait that gave up is charged
    to the section that ran it; a section that raises or sets the word is
    recorded in `errors` and the remaining sections still run."""

    def __init__(self, mpw):
        self.mpw = mpw
        self.errors = []
        self.names = []

    def run(self, name, fn, *args, **kw):
        self.names.append(name)
        result = None
        try:
            result = fn(*args, **kw)
        except Exception as e:  # recorded on the JSON line instead of ending the run
            self.errors.append({"section": name, "error": f"{type(e).__name__}: {e}"[:400]})
        try:
            code = self.mpw.device_error()
        except Exception as e:
            self.errors.append({"section": name, "error": f"device error word unreadable: {e}"[:400]})
            return result
        if code:
            self.errors.append({"section": name, "device_error": code, "where": describe_wait_code(code)})
        return result

    def failed(self, name):
        return any(e["section"] == name for e in self.errors)


def graph_of(fn):
    import torch

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm the launch path before capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def time_graph(g, steps, warmup, world=1):
    """Device time (ms) of `steps` replays of g, max over ranks."""
    import torch

    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    ms = e0.elapsed_time(e1)
    return max_over_ranks(ms, world)


def decode_setup(mpw, W_gpu, b, l2_bytes, layout="canonical"):
    packed, scales = mpw.quantize_pack(W_gpu, b)
    if layout != "canonical":
        packed = mpw.repack(packed, W_gpu.shape[1], b, "canonical", layout)
    return Pool(packed, scales, 4 * l2_bytes)


def measure_decode(mpw, pool, b, M, K, N, steps, warmup, world=1, x=None, layout="canonical", x_ready=True):
    """Back-to-back launches over the pool's distinct matrices with one x,
    each writing its own output.  No launch writes x or another launch's y,
    which each call states (x_ready, y_unshared) unless asked not to, so that
    a launch overlaps its predecessors; x_ready=False times the same launches
    as a dependent chain."""
    import torch

    import workloads as wl

    if x is None:
        x = wl.gen_x(M, K, wl.DECODE["x_seed"]).cuda()
    ys = torch.empty((pool.P, M, N), dtype=torch.bfloat16, device="cuda")

    def step():
        for i in range(pool.P):
            mpw.qlinear(x, pool.packed[i], pool.scales[i], b, y=ys[i], layout=layout, x_ready=x_ready,
                        y_unshared=x_ready)

    g = graph_of(step)
    ms = time_graph(g, steps, warmup, world)
    launches = steps * pool.P
    us_per_launch = ms * 1e3 / launches
    alg_bytes = pool.bytes_each + M * K * 2 + M * N * 2
    out = {
        "b": b, "M": M, "pool": pool.P, "us_per_launch": us_per_launch,
        "weight_GBps": pool.bytes_each / (us_per_launch * 1e3),
        "alg_GBps": alg_bytes / (us_per_launch * 1e3),
        "ms_total": ms, "launches": launches, "alg_bytes_per_launch": alg_bytes,
    }
    del g
    return out


def measure_cold_launch(mpw, pool, x, b, N, layout, l2_bytes, reps=7):
    """One decode launch alone, after a write larger than L2 has flushed it:
    CUDA events around the single launch, median of `reps`."""
    import torch

    flush = torch.empty(int(2 * l2_bytes), dtype=torch.uint8, device="cuda")
    y = torch.empty((x.shape[0], N), dtype=torch.bfloat16, device="cuda")
    times = []
    for r in range(reps):
        i = r % pool.P
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        mpw.qlinear(x, pool.packed[i], pool.scales[i], b, y=y, layout=layout)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3)
    us = sorted(times)[len(times) // 2]
    del flush
    return {"us": round(us, 3), "weight_GBps": round(pool.bytes_each / (us * 1e3), 1),
            "note": "median of single launches after an L2 flush, events around the launch"}


def measure_quantize(mpw, W_gpu, b, steps, warmup, l2_bytes):
    import torch

    N, K = W_gpu.shape
    copies = max(2, -(-4 * l2_bytes // (N * K * 4)))
    Ws = [W_gpu.clone() for _ in range(copies)]
    rb = mpw.packed_row_bytes(K, b)
    packed = torch.empty((N, rb), dtype=torch.uint8, device="cuda")
    scales = torch.empty((N,), dtype=torch.float32, device="cuda")

    def step():
        for Wc in Ws:
            mpw.quantize_pack(Wc, b, packed=packed, scales=scales)

    g = graph_of(step)
    ms = time_graph(g, steps, warmup)
    per = ms * 1e3 / (steps * copies)
    alg = N * K * 4 + N * rb + N * 4
    return {"b": b, "N": N, "K": K, "us_per_launch": per, "alg_GBps": alg / (per * 1e3),
            "weights_per_s": N * K / (per * 1e-6), "copies": copies}


def measure_groups(mpw, W_gpu, b, g, l2_bytes, layout, steps, warmup=3):
    """Group-wise scales (one per g weights of a row): the quantizer, and the
    decode GEMV at M = 1 over a pool of distinct copies, flagged like the
    headline (x_ready + y_unshared).  GB/s count the packed codes and the
    group scales."""
    import torch

    import workloads as wl

    N, K = W_gpu.shape
    packed, scales = mpw.quantize_pack_groups(W_gpu, b, g)
    torch.cuda.synchronize()
    # quantizer: distinct W copies > 4x L2
    copies = max(2, -(-4 * l2_bytes // (N * K * 4)))
    Ws = [W_gpu.clone() for _ in range(copies)]

    def qstep():
        for Wc in Ws:
            mpw.quantize_pack_groups(Wc, b, g, packed=packed, scales=scales)

    gq = graph_of(qstep)
    qms = time_graph(gq, 20, warmup)
    del gq, Ws
    q_us = qms * 1e3 / (20 * copies)
    q_bytes = N * K * 4 + packed.numel() + scales.numel() * 4
    if layout != "canonical":
        packed = mpw.repack(packed, K, b, "canonical", layout)
    per = packed.numel() + scales.numel() * 4
    P = max(2, -(-4 * l2_bytes // per))
    pk = [packed.clone() for _ in range(P)]
    sc = [scales.clone() for _ in range(P)]
    x = wl.gen_x(1, K, wl.DECODE["x_seed"]).cuda()
    ys = torch.empty((P, 1, N), dtype=torch.bfloat16, device="cuda")

    def step():
        for i in range(P):
            mpw.qlinear_groups(x, pk[i], sc[i], b, g, y=ys[i], layout=layout, x_ready=True, y_unshared=True)

    gd = graph_of(step)
    ms = time_graph(gd, steps, warmup)
    del gd
    us = ms * 1e3 / (steps * P)
    return {"b": b, "group": g, "layout": layout, "scale_bytes": scales.numel() * 4,
            "us_per_launch": round(us, 4), "weight_GBps": round(per / (us * 1e3), 1),
            "alg_GBps": round((per + 2 * K + 2 * N) / (us * 1e3), 1),
            "quantize_us": round(q_us, 3), "quantize_GBps": round(q_bytes / (q_us * 1e3), 1)}


def measure_sharded(mpw, world, rank, steps=20, warmup=3, layout="paired"):
    """Output-row sharding across the ranks (every rank calls this; one NCCL
    all-gather per call): the 27B-class gate matrix 17408x5120, b = 6, split
    into row blocks, M = 1 and M = 8.  GB/s count the whole matrix's packed
    bytes over the slowest rank's time per call; the gathered y is checked
    against the unsharded linear on this rank."""
    import torch
    import torch.distributed as dist

    import workloads as wl
    from mixed_precision_weight_row_b200 import shard

    name, N, K = [s for s in wl.MLP27B["shapes"] if s[0] == "gate"][0]
    b = 6
    W = wl.gen_weight_torch(N, K, wl.MLP27B["sigma"], 17 + N)
    packed, scales = mpw.quantize_pack(W, b)
    del W
    if layout != "canonical":
        packed = mpw.repack(packed, K, b, "canonical", layout)
    lin = shard.ShardedLinear.from_full(packed, scales, N, K, b, world, rank, layout=layout)
    out = {"shape": f"{name} {N}x{K}", "b": b, "ranks": world, "rows_per_rank": lin.Nl}
    for M in (1, 8):
        x = wl.gen_x(M, K, 1).cuda()
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        for _ in range(warmup):
            shard.qlinear_sharded(x, lin, y=y)
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            shard.qlinear_sharded(x, lin, y=y)
        e1.record()
        torch.cuda.synchronize()
        barrier(world)
        ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
        full = mpw.qlinear(x, packed, scales, b, layout=layout)
        torch.cuda.synchronize()
        diff = float((full.float() - y.float()).abs().max())
        scale = float(full.float().abs().max())
        out[f"M{M}"] = {"us_per_call": round(ms * 1e3, 3),
                        "matrix_GBps": round((packed.numel() + scales.numel() * 4) / (ms * 1e-3) / 1e9, 1),
                        "max_abs_diff_vs_unsharded": diff, "max_abs_y": scale}
    del packed, scales, lin
    torch.cuda.empty_cache()
    return out


def measure_e2e(mpw, packed_host, scales_host, x_host, b, M, N, K, steps, warmup, pool_n, layout="canonical",
                world=1):
    """Same metric through the public call with host buffers: each step copies
    pool_n packed matrices and x host->device, runs the GEMV on each and reads
    y back to the host.  Whole-job GB/s over `world` ranks (slowest rank)."""
    import torch

    dp = [torch.empty_like(packed_host, device="cuda") for _ in range(2)]
    ds = [torch.empty_like(scales_host, device="cuda") for _ in range(2)]
    dx = torch.empty_like(x_host, device="cuda")
    dy = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    y_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()

    def step():
        dx.copy_(x_host, non_blocking=True)
        for i in range(pool_n):
            j = i & 1
            dp[j].copy_(packed_host, non_blocking=True)
            ds[j].copy_(scales_host, non_blocking=True)
            mpw.qlinear(dx, dp[j], ds[j], b, y=dy, layout=layout)
        y_host.copy_(dy, non_blocking=True)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    wbytes = pool_n * (packed_host.numel() + scales_host.numel() * 4)
    return {"value": whole_job_rate(world, wbytes, ms / steps) / 1e9, "unit": "GB/s",
            "h2d_bytes_per_step": wbytes + x_host.numel() * 2,
            "d2h_bytes_per_step": M * N * 2, "ms_per_step": ms / steps}


def measure_prefill(mpw, pk, reps=10, layout="canonical"):
    """Tensor-core prefill GEMM, x 2048x5120 bf16 against the two weight shapes."""
    import torch

    import workloads as wl

    c = wl.PREFILL
    x = wl.gen_x(c["M"], 5120, c["x_seed"]).cuda()
    out = []
    for name, N, K in c["shapes"]:
        W = wl.gen_weight_torch(N, K, c["sigma"], 11 + N)
        for b in c["bits"]:
            packed, scales = mpw.quantize_pack(W, b)
            if layout != "canonical":
                packed = mpw.repack(packed, K, b, "canonical", layout)
            y = torch.empty((c["M"], N), dtype=torch.bfloat16, device="cuda")
            for _ in range(3):
                mpw.qlinear(x, packed, scales, b, y=y, layout=layout)
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                mpw.qlinear(x, packed, scales, b, y=y, layout=layout)
            e1.record()
            torch.cuda.synchronize()
            us = e0.elapsed_time(e1) * 1e3 / reps
            flops = 2.0 * c["M"] * N * K
            tf = flops / (us * 1e-6) / 1e12
            executed = tf * (2 if b > 9 else 1)
            out.append({"shape": f"{name} {N}x{K}", "b": b, "us": round(us, 2), "TFLOPs": round(tf, 1),
                        "pct_bf16_peak": round(100 * tf / pk["bf16_tflops"], 2),
                        "executed_mma_TFLOPs": round(executed, 1)})
            del packed, scales, y
        del W
        torch.cuda.empty_cache()
    return out


def measure_prefill_fp8(mpw, pk, reps=10, layout="canonical"):
    """FP8 (E4M3) prefill GEMM for 4- and 5-bit codes on the prefill shapes:
    x 2048x5120 quantized per token once (timed apart), then the GEMM.
    The FP8 tensor-core peak is taken as twice the measured bf16 one (the
    nominal ratio of the two dense rates)."""
    import torch

    import workloads as wl

    c = wl.PREFILL
    x = wl.gen_x(c["M"], 5120, c["x_seed"]).cuda()
    xq, sx = mpw.quantize_x_fp8(x)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        mpw.quantize_x_fp8(x, xq=xq, sx=sx)
    e1.record()
    torch.cuda.synchronize()
    xq_us = e0.elapsed_time(e1) * 1e3 / reps
    fp8_peak = 2.0 * pk["bf16_tflops"]
    out = []
    for name, N, K in c["shapes"]:
        W = wl.gen_weight_torch(N, K, c["sigma"], 11 + N)
        for b in (4, 5):
            packed, scales = mpw.quantize_pack(W, b)
            if layout != "canonical":
                packed = mpw.repack(packed, K, b, "canonical", layout)
            y = torch.empty((c["M"], N), dtype=torch.bfloat16, device="cuda")
            for _ in range(3):
                mpw.qlinear_fp8(x, packed, scales, b, y=y, layout=layout, xq=xq, sx=sx)
            torch.cuda.synchronize()
            e0.record()
            for _ in range(reps):
                mpw.qlinear_fp8(x, packed, scales, b, y=y, layout=layout, xq=xq, sx=sx)
            e1.record()
            torch.cuda.synchronize()
            us = e0.elapsed_time(e1) * 1e3 / reps
            tf = 2.0 * c["M"] * N * K / (us * 1e-6) / 1e12
            out.append({"shape": f"{name} {N}x{K}", "b": b, "us": round(us, 2), "TFLOPs": round(tf, 1),
                        "pct_fp8_peak": round(100 * tf / fp8_peak, 2),
                        "pct_bf16_peak": round(100 * tf / pk["bf16_tflops"], 2),
                        "x_quantize_us": round(xq_us, 2)})
            del packed, scales, y
        del W
        torch.cuda.empty_cache()
    return out


def measure_allocator(mpw, reps=20):
    """Host time of the water-filling bit allocator over the recipe stack's 448
    matrix shapes (synthetic log-normal sensitivities), at the byte budget of a
    5.7-bit mean, in both modes."""
    import numpy as np

    import workloads as wl

    shapes = [(N, K) for _, _, N, K in wl.recipe_shapes()]
    sens = np.exp(np.random.default_rng(2).normal(0.0, 1.5, size=len(shapes)))
    params = sum(N * K for N, K in shapes)
    budget = int(params * 5.7 / 8)
    out = []
    for mode in ("native", "full"):
        mpw.allocate_bits(sens, shapes, budget, mode)
        t0 = time.perf_counter()
        for _ in range(reps):
            bits, total = mpw.allocate_bits(sens, shapes, budget, mode)
        us = (time.perf_counter() - t0) / reps * 1e6
        t0 = time.perf_counter()
        fb, fl = mpw.allocation_frontier(sens, shapes, mode)
        us_front = (time.perf_counter() - t0) * 1e6
        out.append({"mode": mode, "matrices": len(shapes), "budget_bytes": budget, "us": round(us, 1),
                    "mean_bits": round(sum(b * N * K for b, (N, K) in zip(bits, shapes)) / params, 3),
                    "bytes": total, "frontier_points": len(fb), "frontier_us": round(us_front, 1)})
    return out


def measure_recipe(mpw, pk, steps=10, warmup=3, layout="canonical"):
    """448-matrix mixed-bit decode pass (M = 1) captured in one CUDA graph."""
    import torch

    import workloads as wl

    shapes, bits, links = wl.recipe_shapes(), wl.recipe_bits(), wl.recipe_links()
    layers = []
    wbytes = 0
    for i, ((layer, name, N, K), b, (si, so, nrm)) in enumerate(zip(shapes, bits, links)):
        W = wl.gen_weight_torch(N, K, wl.RECIPE["sigma"], wl.recipe_weight_seed(i))
        packed, scales = mpw.quantize_pack(W, b)
        del W
        if layout != "canonical":
            mpw.repack(packed, K, b, "canonical", layout, out=packed)
        layers.append(mpw.Linear(packed, scales, N, K, b, si, so, nrm, layout=layout))
        wbytes += packed.numel() + scales.numel() * 4
    slots = [torch.zeros((1, wl.SLOT_WIDTH[s]), dtype=torch.bfloat16, device="cuda") for s in range(8)]
    slots[wl.SLOT_H].copy_(wl.gen_x(1, 5120, wl.RECIPE["x_seed"]).cuda())
    g = graph_of(lambda: mpw.recipe_run(layers, slots, 1))
    ms = time_graph(g, steps, warmup)
    per = ms / steps
    del g
    res = {"matrices": len(layers), "weight_bytes": wbytes, "ms_per_token": round(per, 4),
           "tokens_per_s": round(1e3 / per, 2), "weight_GBps": round(wbytes / (per * 1e-3) / 1e9, 1),
           "pct_hbm": round(100 * wbytes / (per * 1e-3) / 1e9 / pk["hbm_gbs"], 2),
           "launches_per_token": len(layers)}
    if layout == "paired":
        # the same pass planned as one persistent kernel (mpw_pass_*)
        p = mpw.Pass(layers, slots, 1)
        g = graph_of(p.run)
        ms = time_graph(g, steps, warmup) / steps
        del g
        p.close()
        res["persistent_pass"] = {"ms_per_token": round(ms, 4), "tokens_per_s": round(1e3 / ms, 2),
                                  "pct_hbm": round(100 * wbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"], 2),
                                  "launches_per_token": 1, "note": "opt-in; slower than the per-linear launches"}
    del layers
    torch.cuda.empty_cache()
    return res


# ----------------------------------------------------------------------------
# CPU baseline: the oracle, as it stands
# ----------------------------------------------------------------------------

def cpu_baseline(seconds=10.0, b=HEADLINE_BITS):
    """The oracle's decode GEMV (unpack + fp64 dequantize-matmul) on a sample
    of rows of the same workload, repeated for about `seconds`."""
    import numpy as np

    import oracle
    import workloads as wl

    c = wl.DECODE
    rows = 256
    W = wl.gen_weight(c["N"], c["K"], c["sigma"], c["w_seed"], c["outlier_frac"], c["outlier_scale"])[:rows]
    x = wl.gen_x(1, c["K"], c["x_seed"]).float().numpy()
    packed, s = oracle.quantize_pack(W, b)
    t0 = time.perf_counter()
    n = 0
    while True:
        q = oracle.unpack(packed, c["K"], b)
        oracle.qlinear_ref(x, q, s)
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    wbytes = n * (packed.size + s.size * 4)
    try:
        from threadpoolctl import threadpool_info

        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        threads = 1
    return {"value": wbytes / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{rows} of 4096 rows (b={b}, M=1) x {n} repetitions in {dt:.1f} s; "
                      f"host has {os.cpu_count()} cores, numpy BLAS threads {threads}"}


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    steps, warmup = args.steps, args.warmup
    for _ in range(warmup):
        cpu_baseline(seconds=0.0)
    t0 = time.perf_counter()
    samples = []
    for _ in range(steps):
        samples.append(cpu_baseline(seconds=min(5.0, max(0.5, 30.0 / max(steps, 1)))))
    dt = time.perf_counter() - t0
    v = sum(s["value"] for s in samples) / len(samples)
    cb = dict(samples[-1])
    cb["value"] = v
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": warmup, "ms_per_step": dt * 1e3 / max(steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": decode_config(args, pool=None),
            "cpu_baseline": cb, "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def run_case(args):
    """A few launches of one kernel on one workload (for ncu captures)."""
    import torch

    import mixed_precision_weight_row_b200 as mpw
    import workloads as wl

    b, M = args.bits, args.M
    if args.case in ("decode", "quantize", "groups"):
        c = wl.DECODE
        W = torch.from_numpy(wl.gen_weight(c["N"], c["K"], c["sigma"], c["w_seed"], c["outlier_frac"],
                                           c["outlier_scale"])).cuda()
    elif args.case in ("gate", "down"):
        _, N, K = dict((n, (n, a, k)) for n, a, k in wl.MLP27B["shapes"])[args.case]
        W = wl.gen_weight_torch(N, K, wl.MLP27B["sigma"], 17 + N)
    elif args.case in ("prefill", "prefill_fp8"):
        _, N, K = wl.PREFILL["shapes"][0]
        W = wl.gen_weight_torch(N, K, wl.PREFILL["sigma"], 11 + N)
        M = wl.PREFILL["M"]
    if args.case in ("recipe", "pass"):
        shapes, bits, links = wl.recipe_shapes(1), wl.recipe_bits()[:7], wl.recipe_links(1)
        layers = []
        for i, ((_, _, N, K), bb, (si, so, nrm)) in enumerate(zip(shapes, bits, links)):
            packed, scales = mpw.quantize_pack(wl.gen_weight_torch(N, K, 0.02, wl.recipe_weight_seed(i)), bb)
            if args.layout != "canonical":
                mpw.repack(packed, K, bb, "canonical", args.layout, out=packed)
            layers.append(mpw.Linear(packed, scales, N, K, bb, si, so, nrm, layout=args.layout))
        slots = [torch.zeros((1, wl.SLOT_WIDTH[s]), dtype=torch.bfloat16, device="cuda") for s in range(8)]
        if args.case == "pass":
            # one layer of the recipe stack as one persistent kernel
            p = mpw.Pass(layers, slots, 1)
            for _ in range(args.launches):
                p.run()
            torch.cuda.synchronize()
            p.close()
        else:
            for _ in range(args.launches):
                mpw.recipe_run(layers, slots, 1)
    elif args.case == "quantize":
        for _ in range(args.launches):
            mpw.quantize_pack(W, b)
    elif args.case == "groups":
        packed, scales = mpw.quantize_pack_groups(W, b, args.group)
        if args.layout != "canonical":
            packed = mpw.repack(packed, W.shape[1], b, "canonical", args.layout)
        x = wl.gen_x(M, W.shape[1], 1).cuda()
        for _ in range(args.launches):
            mpw.qlinear_groups(x, packed, scales, b, args.group, layout=args.layout)
    elif args.case == "prefill_fp8":
        packed, scales = mpw.quantize_pack(W, b)
        if args.layout != "canonical":
            packed = mpw.repack(packed, W.shape[1], b, "canonical", args.layout)
        x = wl.gen_x(M, W.shape[1], 1).cuda()
        xq, sx = mpw.quantize_x_fp8(x)
        for _ in range(args.launches):
            mpw.qlinear_fp8(x, packed, scales, b, layout=args.layout, xq=xq, sx=sx)
    else:
        packed, scales = mpw.quantize_pack(W, b)
        if args.layout != "canonical":
            packed = mpw.repack(packed, W.shape[1], b, "canonical", args.layout)
        x = wl.gen_x(M, W.shape[1], 1).cuda()
        for _ in range(args.launches):
            mpw.qlinear(x, packed, scales, b, layout=args.layout)
    torch.cuda.synchronize()
    return 0


def decode_config(args, pool):
    return {"workload": "decode GEMV sweep: W 4096x4096 ~N(0,0.02^2) + 0.1% outliers x20, "
                        f"b={HEADLINE_BITS}, x bf16 M=1",
            "N": 4096, "K": 4096, "bits": HEADLINE_BITS, "M": 1,
            "pool_matrices": pool, "l2": "inputs larger than L2: rotating pool of distinct packed "
                                         "matrices totalling > 4x L2 per step",
            "parallelism": f"replicas x{args.gpus}",
            "launches": "one qlinear call per matrix, back to back on one stream in a CUDA graph, each "
                        "into its own output and flagged x_ready + y_unshared (no launch writes x or "
                        "another's y); dependent_chain times them unflagged",
            "layout": (f"{args.layout}" + (": paired-halves re-ordering of the canonical bits, same bytes, "
                                           "repacked once outside the timed region"
                                           if args.layout == "paired" else ""))}


# ----------------------------------------------------------------------------

def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["mine", "reference"], default="mine")
    ap.add_argument("--case", choices=["decode", "gate", "down", "prefill", "recipe", "pass", "quantize", "groups",
                                       "prefill_fp8"],
                    default=None, help="profiling target: run a few launches of one kernel, print nothing")
    ap.add_argument("--bits", type=int, default=HEADLINE_BITS, help="bit width for --case")
    ap.add_argument("--M", type=int, default=1, help="tokens for --case")
    ap.add_argument("--layout", choices=["canonical", "paired"], default="paired",
                    help="packed layout the decode and prefill kernels read (repacked outside the timed region)")
    ap.add_argument("--launches", type=int, default=5, help="launches for --case")
    ap.add_argument("--group", type=int, default=128, help="group size for --case groups")
    ap.add_argument("--quick", action="store_true",
                    help="headline and e2e only (no sweep, extras or CPU baseline)")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        return run_reference(args, world, rank)
    if args.case is not None:
        return run_case(args)

    import numpy as np
    import torch

    import mixed_precision_weight_row_b200 as mpw
    import workloads as wl

    torch.cuda.set_device(local)
    dev = torch.cuda.current_device()
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))
    uuid = str(getattr(props, "uuid", ""))
    uuid = ("GPU-" + uuid) if uuid and not uuid.startswith("GPU-") else uuid
    pk = peaks()
    c = wl.DECODE
    N, K = c["N"], c["K"]
    W_np = wl.gen_weight(N, K, c["sigma"], c["w_seed"], c["outlier_frac"], c["outlier_scale"])
    W = torch.from_numpy(W_np).cuda()

    sec = Sections(mpw)

    # ---- headline: b = 6, M = 1 (every rank; collectives inside) ----
    lay = args.layout
    pool = decode_setup(mpw, W, HEADLINE_BITS, l2, lay)
    x1 = wl.gen_x(1, K, c["x_seed"]).cuda()
    y1 = torch.empty((pool.P, 1, N), dtype=torch.bfloat16, device="cuda")

    def step():
        # distinct matrices applied to one x, each into its own output: no
        # launch writes x or another launch's y (x_ready, y_unshared)
        for i in range(pool.P):
            mpw.qlinear(x1, pool.packed[i], pool.scales[i], HEADLINE_BITS, y=y1[i], layout=lay, x_ready=True,
                        y_unshared=True)

    def headline():
        g = graph_of(step)
        with ClockSampler(uuid) as cs:
            ms = time_graph(g, args.steps, args.warmup, world)
        del g
        return ms, cs.summary()

    ms, clocks = sec.run("headline", headline) or (None, None)
    launches = args.steps * pool.P
    weight_bytes_per_step = pool.P * pool.bytes_each
    alg_bytes = pool.bytes_each + K * 2 + N * 2
    if ms is not None:
        ms_per_step = ms / args.steps
        value = whole_job_rate(world, weight_bytes_per_step, ms_per_step) / 1e9
        us_launch = ms * 1e3 / launches
        achieved = alg_bytes / (us_launch * 1e-6) / 1e9
    else:
        ms_per_step = value = us_launch = achieved = None

    # ---- e2e: the public call with host buffers (every rank; collectives) ----
    packed_h = pool.packed[0].cpu().pin_memory()
    scales_h = pool.scales[0].cpu().pin_memory()
    x_h = x1.cpu().pin_memory()
    e2e = sec.run("e2e", measure_e2e, mpw, packed_h, scales_h, x_h, HEADLINE_BITS, 1, N, K,
                  max(3, min(args.steps, 10)), 3, pool.P, layout=lay, world=world)

    # output-row sharding over the ranks (every rank; collectives)
    extras = {}
    if world > 1:
        extras["sharded"] = sec.run("sharded", measure_sharded, mpw, world, rank, layout=lay)

    # rank 0 alone from here on: no collective until the end
    if rank == 0:
        # the same launches, each one waiting for its predecessor before it
        # reads x (what a chain of dependent linears sees)
        r = sec.run("dependent_chain", measure_decode, mpw, pool, HEADLINE_BITS, 1, K, N,
                    max(20, args.steps // 4), 3, layout=lay, x=x1, x_ready=False)
        if r is not None:
            extras["dependent_chain"] = {"us_per_launch": round(r["us_per_launch"], 4),
                                         "weight_GBps": round(r["weight_GBps"], 1),
                                         "pct_hbm": round(100.0 * r["alg_GBps"] / pk["hbm_gbs"], 2)}
        extras["cold_single_launch"] = sec.run("cold_single_launch", measure_cold_launch, mpw, pool, x1,
                                               HEADLINE_BITS, N, lay, l2)
    if rank == 0 and not args.quick:
        def row(r, layout):
            r["pct_hbm"] = 100.0 * r["alg_GBps"] / pk["hbm_gbs"]
            r["layout"] = layout
            return {k: (round(v, 4) if isinstance(v, float) else v) for k, v in r.items()
                    if k in ("b", "M", "layout", "us_per_launch", "weight_GBps", "alg_GBps", "pct_hbm")}

        sweep = []
        for b in DECODE_BITS:
            p = pool if b == HEADLINE_BITS else sec.run(f"decode_setup b={b}", decode_setup, mpw, W, b, l2, lay)
            if p is None:
                continue
            for M in DECODE_MS:
                r = sec.run(f"decode_sweep b={b} M={M}", measure_decode, mpw, p, b, M, K, N,
                            max(20, args.steps // 4), 3, layout=lay)
                if r is not None:
                    sweep.append(row(r, lay))
            if lay != "canonical":
                # the canonical rows, read directly (no re-ordering), at M = 1
                pc = sec.run(f"decode_setup canonical b={b}", decode_setup, mpw, W, b, l2)
                if pc is not None:
                    r = sec.run(f"decode_sweep canonical b={b} M=1", measure_decode, mpw, pc, b, 1, K, N,
                                max(20, args.steps // 4), 3)
                    if r is not None:
                        sweep.append(row(r, "canonical"))
                del pc
            if p is not pool:
                del p
                torch.cuda.empty_cache()
        extras["decode_sweep"] = sweep
        extras["quantize_pack"] = []
        for b in (4, 6, 8, 12):
            r = sec.run(f"quantize_pack b={b}", measure_quantize, mpw, W, b, 20, 3, l2)
            if r is not None:
                r["pct_hbm"] = 100.0 * r["alg_GBps"] / pk["hbm_gbs"]
                extras["quantize_pack"].append({k: (round(v, 4) if isinstance(v, float) else v)
                                                for k, v in r.items()})
        groups = []
        for b in (4, 6):
            for gsize in (128, 256):
                r = sec.run(f"groups b={b} g={gsize}", measure_groups, mpw, W, b, gsize, l2, lay,
                            max(20, args.steps // 4))
                if r is not None:
                    r["pct_hbm"] = round(100.0 * r["alg_GBps"] / pk["hbm_gbs"], 2)
                    groups.append(r)
        extras["group_scales"] = groups
        mlp = []
        for name, n_, k_ in wl.MLP27B["shapes"][1:]:
            Wm = wl.gen_weight_torch(n_, k_, wl.MLP27B["sigma"], 17 + n_)
            for b in wl.MLP27B["bits"]:
                pm = sec.run(f"mlp27b setup {name} b={b}", decode_setup, mpw, Wm, b, l2, lay)
                if pm is None:
                    continue
                for M in wl.MLP27B["Ms"]:
                    r = sec.run(f"mlp27b {name} b={b} M={M}", measure_decode, mpw, pm, b, M, k_, n_, 20, 3,
                                x=wl.gen_x(M, k_, 1).cuda(), layout=lay)
                    if r is not None:
                        mlp.append({"shape": f"{name} {n_}x{k_}", "b": b, "M": M,
                                    "us_per_launch": round(r["us_per_launch"], 3),
                                    "weight_GBps": round(r["weight_GBps"], 1),
                                    "pct_hbm": round(100 * r["alg_GBps"] / pk["hbm_gbs"], 2)})
                del pm
                torch.cuda.empty_cache()
            del Wm
            torch.cuda.empty_cache()
        extras["mlp27b"] = mlp
        extras["prefill"] = sec.run("prefill", measure_prefill, mpw, pk, layout=lay)
        extras["prefill_fp8"] = sec.run("prefill_fp8", measure_prefill_fp8, mpw, pk, layout=lay)
        extras["allocator"] = sec.run("allocator", measure_allocator, mpw)
        extras["recipe"] = sec.run("recipe", measure_recipe, mpw, pk, layout=lay)
        summary = {}
        for p in extras.get("prefill") or []:
            summary[f"prefill {p['shape']} b={p['b']} TFLOPs"] = p["TFLOPs"]
        for p in extras.get("prefill_fp8") or []:
            summary[f"prefill fp8 {p['shape']} b={p['b']} TFLOPs"] = p["TFLOPs"]
        if extras.get("recipe"):
            summary["recipe tokens_per_s"] = extras["recipe"]["tokens_per_s"]
            summary["recipe pct_hbm"] = extras["recipe"]["pct_hbm"]
        extras["summary"] = summary

    traffic = profile_traffic(f"gemv_tma_decode_b6_m1_{lay}.json", TMA_GEMV_SOURCES)
    roof = {"bound": "hbm",
            "kernel": f"gemv_tma_kernel<{HEADLINE_BITS},1,0,{str(lay == 'paired').lower()},false,1,1,8>",
            "achieved": round(achieved, 1) if achieved is not None else None,
            "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / pk["hbm_gbs"], 4) if achieved is not None else None,
            "traffic": traffic, "alg_bytes_per_launch": alg_bytes,
            "us_per_launch": round(us_launch, 4) if us_launch is not None else None,
            "peak_source": pk["source"] + " (copy bandwidth; burst figure, kernel timed alone)"}

    line = {"metric": METRIC, "value": round(value, 2) if value is not None else None, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 5) if ms_per_step is not None else None,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": decode_config(args, pool.P),
            "roofline": roof, "e2e": e2e, "gpu_launches": launches, "clocks": clocks,
            "pct_hbm_peak": round(100 * value / world / pk["hbm_gbs"], 2) if value is not None else None}
    line.update(extras)
    if rank == 0 and world == 1 and not args.quick:
        line["cpu_baseline"] = cpu_baseline(seconds=10.0)
    line["sections"] = len(sec.names)
    line["errors"] = sec.errors
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0 if value is not None else 1


if __name__ == "__main__":
    sys.exit(main())
