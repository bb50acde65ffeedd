#!/usr/bin/env python
"""Benchmark of exact blockwise (ring) attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--sched auto|persistent|fused|unfused] [--order ring|tokenring]
                    [--impl ours|reference]

One step = one ra_ring_attention call over the workload (partition of Q, K, V
into block order, block attention over every (query block, KV block) pair in
schedule order with the merge rule, output in original order).  The default
workload is the 1M-token one (the largest that fits one GPU); the 4k and 24k
workloads are timed the same way beside it, each in its own sub-object.  The
metric is causal-adjusted attention throughput, 4 * B * Hq * D * P FLOPs per
step with P the number of visible (query, key) pairs.  Inputs are resident in
HBM when the timed region starts; L2 is flushed between timed steps (a
256 MiB write, then read back), outside the timed events.  Each step is timed
on the device with CUDA events on the launching stream.  With N GPUs each rank
runs the same workload on its own GPU (replicas, weak scaling; the method needs
no exchange on one node here) and the slowest rank's time counts.

--impl reference times the CPU fp64 oracle on the host cores instead (a
bounded sample of the same workload).  --backward, --decode, --merge-sweep
and --shards time the gradient, decode over a KV cache, the merge kernels,
and the sequence-parallel rank programs (one block per rank, all ranks on
this GPU) instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from seeded_inputs import WORKLOADS, workload_inputs  # noqa: E402

DEFAULT_WORKLOAD = "long1m"
DEFAULT_STEPS = {"tiny": 2000, "zigzag4k": 2000, "gqa24k": 400, "long1m": 5}
# Workloads timed beside the headline one on the default line, with the
# steps each runs there (enough for the clock sampler to see the region).
SIDE_WORKLOADS = {"zigzag4k": 2000, "gqa24k": 200}
METRIC = "causal-adj attention TFLOP/s (% of dense bf16 peak)"
L2_FLUSH_BYTES = 256 << 20
L2_FLUSH_DESC = (f"flushed between steps: a {L2_FLUSH_BYTES >> 20} MiB write, then that buffer read back, "
                 f"so no input is L2-resident and L2 holds no dirty lines")


class L2Flush:
    """Evicts the inputs of the last step from L2 (126 MB) between timed
    steps, outside their events.  A write of a buffer twice the size of L2
    alone would leave up to 126 MB of dirty lines whose write-back the next
    timed kernel would pay; reading the buffer back leaves only clean lines."""

    def __init__(self, dev):
        import torch
        self.buf = torch.empty(L2_FLUSH_BYTES // 8, dtype=torch.int64, device=dev)

    def __call__(self):
        self.buf.zero_()
        self.buf.sum()


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=None)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    p.add_argument("--sched", default="auto", choices=["auto", "persistent", "fused", "unfused"])
    p.add_argument("--order", default="ring", choices=["ring", "tokenring"])
    p.add_argument("--tiling", default="auto", choices=["auto", "row_pairs", "kv_split", "cluster2"])
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-merge", action="store_true")
    p.add_argument("--merge-sweep", action="store_true",
                   help="time the merge kernels over the whole token / partial sweep instead")
    p.add_argument("--merge-T", type=int, nargs="*", default=None, help="token counts of the merge sweep")
    p.add_argument("--merge-k", type=int, nargs="*", default=None, help="partial counts of the merge sweep")
    p.add_argument("--decode", action="store_true",
                   help="time decode-phase attention over a KV cache (both decode workloads) instead")
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--backward", action="store_true",
                   help="time the backward pass (ra_ring_attention_backward) on --workload instead")
    p.add_argument("--no-backward", action="store_true")
    p.add_argument("--backward-workload", default="gqa24k", choices=sorted(WORKLOADS),
                   help="workload of the backward object on the default line")
    p.add_argument("--no-side", action="store_true", help="time only --workload (no other attention workloads)")
    p.add_argument("--cta-timeline", action="store_true",
                   help="record where every CTA of the forward (and with --backward, of the two backward "
                        "kernels) ran, once, after warm-up; print a per-kernel summary instead")
    p.add_argument("--shards", action="store_true",
                   help="time the sequence-parallel rank programs (one block per rank), all ranks on one GPU")
    a = p.parse_args()
    if a.steps is None:
        a.steps = DEFAULT_STEPS[a.workload]
    if a.warmup < 3:
        p.error("--warmup must be >= 3")
    return a


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def workload_config(w, args, l2):
    return {"workload": w.name, "B": w.B, "S": w.S, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "n_blocks": w.n_blocks,
            "causal": w.causal, "partition": w.partition, "in_dtype": w.in_dtype, "out_dtype": w.out_dtype,
            "sched": args.sched, "order": args.order, "tiling": args.tiling, "l2": l2,
            "parallelism": f"replicas{args.gpus}"}


# ------------------------------------------------------------- CPU oracle

def blas_threads(n=None):
    """Pins the oracle's BLAS (OpenBLAS under NumPy) to n threads (default:
    every core this process may run on) and returns (context, n).  The
    count is what the baseline reports as `cores`."""
    import numpy as np  # noqa: F401  (loads the BLAS library threadpoolctl controls)
    from threadpoolctl import threadpool_limits
    n = n or len(os.sched_getaffinity(0))
    return threadpool_limits(limits=n, user_api="blas"), n


def sample_rows(w, count, seed=0):
    """`count` seeded (batch, position, query head) rows of workload w, drawn
    uniformly over positions and heads (the first and the last position
    always included)."""
    import numpy as np
    rng = np.random.default_rng(seed)
    pos = rng.integers(0, w.S, size=count)
    pos[0], pos[-1] = 0, w.S - 1
    heads = rng.integers(0, w.Hq, size=count)
    return [(0, int(i), int(h)) for i, h in zip(pos, heads)]


def rows_flops(w, rows):
    """Causal-adjusted FLOPs of the given query rows: 4 * D per visible key."""
    return sum(4.0 * w.D * ((i + 1) if w.causal else w.S) for _, i, _ in rows)


def oracle_f_sample(w, inputs, budget_s=15.0, threads=None, count=None):
    """Times the oracle's plain path F (full softmax attention in fp64, the
    definition the method reproduces) on a bounded sample of workload w, with
    the BLAS pinned to `threads` threads.  Up to 24,000 tokens the sample is
    the first h query heads of batch 0 in full, h sized to the budget from a
    first one-head run; beyond that it is a seeded set of query rows, each
    computed against every key it sees (oracle.attention.attention_rows):
    `count` rows, or as many as the budget allows after an 8-row probe (at
    least 64).  Returns (TFLOP/s, threads, sample description, seconds,
    rows or heads sampled)."""
    from oracle import attention as F
    q, k, v = inputs
    ctx, n = blas_threads(threads)
    with ctx:
        if w.S <= 24000:
            g = w.gqa_groups
            per_head = w.flops / (w.B * w.Hq)
            t0 = time.perf_counter()
            F.full_attention(q[:1, :, :1], k[:1, :, :1], v[:1, :, :1], w.causal, 1)
            t1 = time.perf_counter() - t0
            heads = max(1, min(w.Hq, int(budget_s / max(t1, 1e-3))))
            nkv = (heads + g - 1) // g
            t0 = time.perf_counter()
            F.full_attention(q[:1, :, :heads], k[:1, :, :nkv], v[:1, :, :nkv], w.causal, g)
            dt = time.perf_counter() - t0
            return (per_head * heads / dt / 1e12, n,
                    f"oracle path F (plain fp64 attention, NumPy) on batch 0, query heads 0..{heads - 1} of {w.Hq}, "
                    f"all {w.S} rows", dt, heads)
        if count is None:
            probe = sample_rows(w, 8, seed=1)
            t0 = time.perf_counter()
            F.attention_rows(q, k, v, probe, w.causal, w.gqa_groups)
            t1 = time.perf_counter() - t0
            count = int(max(64, min(4096, 8 * budget_s / max(t1, 1e-3))))
        rows = sample_rows(w, count, seed=2)
        t0 = time.perf_counter()
        F.attention_rows(q, k, v, rows, w.causal, w.gqa_groups)
        dt = time.perf_counter() - t0
        return (rows_flops(w, rows) / dt / 1e12, n,
                f"oracle path F rows (plain fp64 attention per query row, NumPy): {count} seeded rows of batch 0 "
                f"over all positions and query heads, each against every key it sees", dt, count)


def cpu_baseline(w, inputs, budget_s=15.0):
    """The `cpu_baseline` object: path F on every core of this process, and
    a per-core figure (path F, one BLAS thread, one head of the 4k zigzag
    workload)."""
    v_, n, sample, dt, _ = oracle_f_sample(w, inputs, budget_s)
    w4 = WORKLOADS["zigzag4k"]
    one = workload_inputs(w4) if w.name != "zigzag4k" else inputs
    v1, _, s1, dt1, _ = oracle_f_sample(w4, one, budget_s=0.0, threads=1)
    return {"value": v_, "unit": "TFLOP/s", "cores": n, "kind": "oracle", "sample": sample, "seconds": dt,
            "blas_threads": n,
            "per_core": {"value": v1, "unit": "TFLOP/s", "cores": 1, "workload": "zigzag4k", "sample": s1,
                         "seconds": dt1}}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    inputs = workload_inputs(w)
    per_step = []
    budget = max(1.0, 120.0 / max(args.steps + args.warmup, 1))
    row_mode = w.S > 24000
    for _ in range(args.warmup):  # untimed
        oracle_f_sample(w, inputs, budget_s=0.0, count=8 if row_mode else None)
    cores, sample, count = None, None, None
    for _ in range(args.steps):
        # every step samples the same amount: the first step sizes it
        v, cores, sample, dt, got = oracle_f_sample(w, inputs, budget_s=budget, count=count)
        if row_mode:
            count = got
        per_step.append(v)
    value = statistics.median(per_step)
    line = {"impl": "reference", "metric": METRIC, "value": value,
            "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": None, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded randn, bf16-rounded)", "config": workload_config(w, args, "n/a (CPU)"),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample,
                             "blas_threads": cores},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ----------------------------------------------------------------- clocks

class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.proc = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(gpu_id), "-lms", "100"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def local_gpu_id(dev):
    """nvidia-smi id of this process's GPU (its UUID; the index as fallback)."""
    import torch
    props = torch.cuda.get_device_properties(dev)
    gpu_id = getattr(props, "uuid", None)
    if gpu_id is None:
        return dev.index
    return f"GPU-{gpu_id}" if not str(gpu_id).startswith("GPU-") else gpu_id


FWD_SOURCES = ["attn_fwd.cuh", "common.cuh", "tmem_ld.cuh", "merge_rule.cuh"]
BWD_SOURCES = FWD_SOURCES + ["attn_bwd.cuh"]


def kernel_sha(files=FWD_SOURCES):
    import hashlib
    h = hashlib.sha256()
    src = os.path.join(ROOT, "blockwise_exact_attention_block_b200", "csrc")
    for f in files:
        h.update(open(os.path.join(src, f), "rb").read())
    return h.hexdigest()[:16]


def attn_traffic(workload, record="attn_fwd_traffic.json", files=FWD_SOURCES):
    """The committed ncu record of this workload: DRAM bytes per launch (per
    call for the backward's two kernels) and a note on what they count; None
    when there is none for this workload or the kernel sources changed since."""
    path = os.path.join(ROOT, "profiles", record)
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(workload)
    if not rec or rec.get("kernel_sha") != kernel_sha(files):
        return None
    return rec


# ------------------------------------------------------------- multi-rank

def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` over all ranks (the slowest rank's time); the
    identity without an initialised process group.  Works with any backend:
    the tensor lives on `device` (a CUDA device for NCCL, the CPU for gloo)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(flops_per_step: float, world: int, steps: int, max_ms: float) -> float:
    """Whole-job TFLOP/s of `world` replicas that each ran `steps` steps, timed
    by the slowest rank (weak scaling: every rank does the same work)."""
    return flops_per_step * world * steps / (max_ms * 1e-3) / 1e12


# ------------------------------------------------------------ merge kernels

MERGE_HBM_BUDGET = 140 << 30  # device bytes the k-way sweep may hold in partials


def bench_merge(ra, dev, T, k, reps, flush, kway=False):
    """GB/s of merging k partials of [T, 32, 128] fp32 (+ lse [T, 32]).

    Pairwise: k-1 ra_merge_partial launches into one accumulator, 12*D+12
    bytes per row each; every launch is timed on its own, after an L2 flush,
    and the GB/s is that of the median launch (the bytes of one launch do not
    depend on k).  The partials cycle through at most 4 buffers: each launch
    reads one of them once, so nothing it reads was left in L2 by the launch
    before.
    k-way: one ra_merge_partials call over k distinct partial buffers (a
    repeated buffer inside one call would be read from L2, since the kernel
    reads every partial of a row together), (k+1)*(4*D+4) bytes per row.
    Returns (GB/s, ms), or (None, None) when k distinct partials of this size
    do not fit in the device memory set aside for them."""
    import torch
    H, D = 32, 128
    rows = T * H
    part_bytes = rows * (D + 1) * 4
    if kway and k * part_bytes > MERGE_HBM_BUDGET:
        return None, None
    nb = k if kway else min(max(k - 1, 1), 4)
    g = torch.Generator(device=dev).manual_seed(1)
    out = torch.randn((T, H, D), device=dev, generator=g)
    lse = torch.rand((T, H), device=dev, generator=g) * 20 - 5
    n_extra = k - 1 if kway else nb
    bos = [torch.randn((T, H, D), device=dev, generator=g) for _ in range(n_extra)]
    bls = [torch.rand((T, H), device=dev, generator=g) * 20 - 5 for _ in range(n_extra)]
    stream = torch.cuda.current_stream(dev)
    times = []
    for rep in range(reps + 2):
        launches = [None] if kway else list(range(k - 1))
        for j in launches:
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            if kway:
                ra.ra_merge_partials([out] + bos, [lse] + bls, out=out, lse=lse)
            else:
                ra.ra_merge_partial(out, lse, bos[j % nb], bls[j % nb])
            e1.record(stream)
            e1.synchronize()
            if rep >= 2:
                times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    nbytes = rows * ((k + 1) * (4 * D + 4) if kway else (12 * D + 12))
    del out, lse, bos, bls
    torch.cuda.empty_cache()
    return nbytes / (ms * 1e-3) / 1e9, ms


# ------------------------------------------------------------ decode phase

def bench_decode(ra, dev, w, reps, flush):
    """GB/s of one ra_decode_attention call on workload w: the bytes it must
    move (K and V cache and Q read, out and lse written) over the call's time,
    both kernels (chunk partials and their merge) included.  The cache is
    drawn on the device (its values do not change the time; the parity tests
    use the seeded host inputs)."""
    import torch
    g = torch.Generator(device=dev).manual_seed(2)
    q = torch.randn((w.B, w.Tq, w.Hq, w.D), device=dev, generator=g).to(torch.bfloat16)
    k = torch.randn((w.B, w.Skv, w.Hkv, w.D), device=dev, generator=g).to(torch.bfloat16)
    v = torch.randn((w.B, w.Skv, w.Hkv, w.D), device=dev, generator=g).to(torch.bfloat16)
    out = torch.empty((w.B, w.Tq, w.Hq, w.D), dtype=torch.float32 if w.out_dtype == "f32" else torch.bfloat16,
                      device=dev)
    lse = torch.empty((w.B, w.Tq, w.Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(max(ra.ra_decode_workspace(w.B, w.Tq, w.Skv, w.Hq, w.Hkv, w.D, 0), 1), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream(dev)
    times = []
    for rep in range(reps + 3):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        ra.ra_decode_attention(q, k, v, w.causal, 0, out=out, lse=lse, workspace=ws)
        e1.record(stream)
        e1.synchronize()
        if rep >= 3:
            times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    splits = ra.ra_decode_splits(w.B, w.Tq, w.Skv, w.Hq, w.Hkv, w.D, 0)
    del q, k, v, out, lse, ws
    torch.cuda.empty_cache()
    return w.bytes / (ms * 1e-3) / 1e9, ms, splits


def run_decode(args):
    import torch
    import blockwise_exact_attention_block_b200 as ra
    from seeded_inputs import DECODE_WORKLOADS
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    flush = L2Flush(dev)
    pk, pk_kind = peaks()
    lines = []
    clocks = Clocks(local_gpu_id(dev))
    time.sleep(0.3)
    for name, w in DECODE_WORKLOADS.items():
        gbs, ms, splits = bench_decode(ra, dev, w, min(max(args.steps, 10), 50), flush)
        lines.append((name, w, gbs, ms, splits))
    clk = clocks.stop()
    status = ra.ra_get_device_status()
    for name, w, gbs, ms, splits in lines:
        line = {"metric": "decode GB/s (% of HBM peak)", "value": gbs, "unit": "GB/s", "n_gpus": 1, "steps": None,
                "warmup": 3, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic (device randn, bf16-rounded)",
                "config": {"workload": name, "B": w.B, "Tq": w.Tq, "Skv": w.Skv, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
                           "causal": w.causal, "chunks": splits, "bytes_per_call": w.bytes,
                           "l2": L2_FLUSH_DESC},
                "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                             "frac": gbs / pk["hbm_gbs"], "traffic": None, "kernel": "decode_partial_kernel",
                             "peak_source": f"{pk_kind} copy bandwidth"},
                "clocks": clk, "gpu_launches": 2, "device_status": ra.ra_status_string(status)}
        print(json.dumps(line))
    return 0 if status == 0 else 1


# ---------------------------------------------------------------- our arm

# ------------------------------------------------------------ backward pass

def bench_backward(ra, dev, w, reps, flush, order="ring"):
    """One ra_ring_attention_backward call on workload w (inputs and the
    forward's out and lse resident in HBM, L2 flushed before each call).
    The algorithmic work is five products of the forward's size (S = Q K^T,
    dP = dO V^T, dV = P^T dO, dQ = dS K, dK = dS^T Q): 2.5x the forward's
    causal-adjusted FLOPs.  Returns (call TFLOP/s, kernels TFLOP/s, call ms,
    kernels ms): the kernels are the dK/dV and dQ launches alone (events the
    library records around them), the call adds the Delta / lse pass."""
    import torch
    from seeded_inputs import backward_inputs
    q, k, v, do = (x.to(dev) for x in backward_inputs(w.B, w.S, w.Hq, w.Hkv, w.D, w.in_dtype, seed=10))
    odt = torch.bfloat16 if w.out_dtype == "bf16" else torch.float32
    o, l = ra.ra_ring_attention(q, k, v, w.n_blocks, w.causal, w.partition, w.gqa_groups, out_dtype=odt)
    ws = torch.empty(ra.ra_ring_attention_backward_workspace(w.B, w.S, w.Hq, w.D, w.n_blocks, w.gqa_groups,
                                                             w.partition, q.dtype), dtype=torch.uint8, device=dev)
    dq = torch.empty(q.shape, dtype=torch.float32, device=dev)
    dk = torch.empty(k.shape, dtype=torch.float32, device=dev)
    dv = torch.empty(k.shape, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    call, kern = [], []

    def one(events=None):
        ra.ra_ring_attention_backward(q, k, v, o, l, do, w.n_blocks, w.causal, w.partition, w.gqa_groups, dq=dq,
                                      dk=dk, dv=dv, workspace=ws, order=order, attn_events=events)

    # whole calls (no events inside), then the two kernels alone (events the
    # library records around them) in a second pass
    for timed, out_list in ((False, call), (True, kern)):
        for rep in range(reps + 3):
            flush()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            if timed:
                one(tuple(ev))
            else:
                ev[0].record(stream)
                one()
                ev[1].record(stream)
            ev[1].synchronize()
            if rep >= 3:
                out_list.append(ev[0].elapsed_time(ev[1]))
    ms, kms = statistics.median(call), statistics.median(kern)
    del q, k, v, do, o, l, ws, dq, dk, dv
    torch.cuda.empty_cache()
    fl = 2.5 * w.flops
    return fl / (ms * 1e-3) / 1e12, fl / (kms * 1e-3) / 1e12, ms, kms


def run_backward(args):
    import torch
    import blockwise_exact_attention_block_b200 as ra
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    flush = L2Flush(dev)
    w = WORKLOADS[args.workload]
    pk, pk_kind = peaks()
    clocks = Clocks(local_gpu_id(dev))
    time.sleep(0.3)
    reps = min(max(args.steps, 5), 200)
    tf, ktf, ms, kms = bench_backward(ra, dev, w, reps, flush, args.order)
    clk = clocks.stop()
    status = ra.ra_get_device_status()
    sustained = kms > 100.0
    peak = pk["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    line = {"metric": "backward causal-adj TFLOP/s (2.5x forward FLOPs)", "value": tf, "unit": "TFLOP/s",
            "n_gpus": 1, "steps": reps, "warmup": 3, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded randn, bf16-rounded)",
            "config": dict(workload_config(w, args, L2_FLUSH_DESC),
                           flops_per_step=2.5 * w.flops),
            "roofline": {"bound": "tensor", "achieved": ktf, "peak": peak, "unit": "TFLOP/s", "frac": ktf / peak,
                         "traffic": (attn_traffic(w.name, "attn_bwd_traffic.json", BWD_SOURCES) or {}).get(
                             "dram_bytes_per_launch"),
                         "kernel": "bwd_dkv_kernel + bwd_dq_kernel",
                         "peak_source": f"{pk_kind} {'sustained' if sustained else 'burst'} bf16 dense"},
            "kernels_ms": kms, "clocks": clk, "gpu_launches": reps * (3 if w.in_dtype == "bf16" else 7),
            "device_status": ra.ra_status_string(status)}
    print(json.dumps(line))
    return 0 if status == 0 else 1


# ------------------------------------------------- sequence-parallel programs

def shard_pairs(n, order, s):
    """(query block, KV block) each rank computes at step s of the order:
    ring, s = 0..n-1, rank r meets KV block (r - s) mod n; TokenRing,
    s = 1..n, rank j computes query block (j - s + 1) mod n on its KV j."""
    if order == "ring":
        return [(r, (r - s) % n) for r in range(n)]
    return [((j - s + 1) % n, j) for j in range(n)]


def shard_step_estimate(pair_ms, n, order, merge_ms=0.0):
    """Per-step compute time with one rank per GPU: the slowest rank's pair
    (plus, under TokenRing, the merge of the partial it receives).  pair_ms
    maps (query block, KV block) to the pair's kernel time; a pair absent
    from it ran nothing (causal skip).  Transfers are assumed to overlap."""
    steps = range(n) if order == "ring" else range(1, n + 1)
    out = []
    for s in steps:
        worst = 0.0
        for qb, kb in shard_pairs(n, order, s):
            t = pair_ms.get((qb, kb), 0.0)
            if order == "tokenring" and s > 1 and (qb, kb) in pair_ms:
                t += merge_ms
            worst = max(worst, t)
        out.append(worst)
    return out


def shard_exchange_bytes(w, order):
    """Bytes one rank sends per step: the K/V block (ring), or the Q block
    plus one fp32 partial, block_out and block_lse (TokenRing)."""
    L = w.S // w.n_blocks
    if order == "ring":
        return 2 * w.B * L * w.Hkv * w.D * 2
    return w.B * L * w.Hq * w.D * 2 + w.B * L * w.Hq * (w.D + 1) * 4


def run_shards(args):
    """The sequence-parallel rank programs (one block per rank) with every
    rank on this GPU, messages as device copies.  Reports the whole pass, and
    an estimate for one rank per GPU from each pair's kernel time."""
    import torch
    import blockwise_exact_attention_block_b200 as ra
    from blockwise_exact_attention_block_b200 import ring
    if int(os.environ.get("WORLD_SIZE", "1")) != 1:
        raise SystemExit("--shards runs every rank on one GPU (no torchrun)")
    w = WORKLOADS[args.workload]
    if w.in_dtype != "bf16":
        raise SystemExit("--shards needs a bf16 workload")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = L2Flush(dev)
    pk, pk_kind = peaks()
    n = w.n_blocks
    q, k, v = (x.to(dev) for x in workload_inputs(w))

    def shard(x, r):
        return torch.cat([x[:, p:p + ln] for p, ln in ring.block_segments(w.S, n, w.partition, r)], dim=1).contiguous()

    qs, ks, vs = ([shard(x, r) for r in range(n)] for x in (q, k, v))
    del q, k, v
    stream = torch.cuda.current_stream(dev)

    class TimedOps(ring.BlockOps):
        record = None

        def _timed(self, key, fn, *a):
            if self.record is None:
                return fn(*a)
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            ev[0].record(stream)
            fn(*a)
            ev[1].record(stream)
            self.record.append((key, ev))

        def attn_merge(self, qq, kk, vv, qb, kb, out, lse):
            self._timed((qb, kb), super().attn_merge, qq, kk, vv, qb, kb, out, lse)

        def attn(self, qq, kk, vv, qb, kb, bo, bl):
            self._timed((qb, kb), super().attn, qq, kk, vv, qb, kb, bo, bl)

        def merge(self, out, lse, bo, bl):
            self._timed("merge", super().merge, out, lse, bo, bl)

    ops = TimedOps(w.S, n, w.causal, w.partition)
    clocks = Clocks(local_gpu_id(dev))
    time.sleep(0.3)
    passes = []
    for rep in range(args.warmup + args.steps):
        flush()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record(stream)
        ring.ring_attention_lockstep(qs, ks, vs, w.S, w.causal, w.partition, args.order, ops=ops)
        ev[1].record(stream)
        ev[1].synchronize()
        if rep >= args.warmup:
            passes.append(ev[0].elapsed_time(ev[1]))
    # one more pass with events around every kernel, for the per-pair times
    ops.record = []
    flush()
    ring.ring_attention_lockstep(qs, ks, vs, w.S, w.causal, w.partition, args.order, ops=ops)
    torch.cuda.synchronize()
    pair_ms, merges = {}, []
    for key, ev in ops.record:
        t = ev[0].elapsed_time(ev[1])
        if key == "merge":
            merges.append(t)
        else:
            pair_ms[key] = t
    clk = clocks.stop()
    status = ra.ra_get_device_status()
    ms = statistics.median(passes)
    merge_ms = statistics.mean(merges) if merges else 0.0
    steps = shard_step_estimate(pair_ms, n, args.order, merge_ms)
    xbytes = shard_exchange_bytes(w, args.order)
    nvlink_gbs = 770.0  # measured peer copy per direction on this kind of node
    launches = len(pair_ms) + len(merges)
    line = {"metric": "sequence-parallel pass TFLOP/s, all ranks on one GPU", "value": w.flops / (ms * 1e-3) / 1e12,
            "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded randn, bf16-rounded)",
            "config": dict(workload_config(w, args, L2_FLUSH_DESC),
                           parallelism=f"sequence-parallel {n} ranks, lockstep on one GPU"),
            "ranks": n, "pair_ms": {f"{a},{b}": t for (a, b), t in sorted(pair_ms.items())},
            "merge_ms": merge_ms,
            "one_rank_per_gpu_estimate": {
                "step_compute_ms": steps, "pass_ms": sum(steps),
                "TFLOP/s": w.flops / (sum(steps) * 1e-3) / 1e12,
                "exchange_bytes_per_rank_step": xbytes,
                "exchange_ms_per_step_at_770GBps": xbytes / (nvlink_gbs * 1e9) * 1e3,
                "note": "transfers assumed hidden under the step's compute when shorter; not measured across GPUs"},
            "peak_bf16_tflops": pk["bf16_tflops"], "peak_source": pk_kind, "clocks": clk,
            "gpu_launches": launches * args.steps, "device_status": ra.ra_status_string(status)}
    print(json.dumps(line))
    return 0 if status == 0 else 1


def launches_per_step(w, sched):
    """Kernels of ours launched by one ra_ring_attention call."""
    cast = 3 if w.in_dtype == "f32" else 0
    if sched in ("auto", "persistent"):
        return cast + 1
    out_cast = 1 if w.out_dtype == "bf16" else 0
    if sched == "fused":
        return cast + w.n_blocks + out_cast
    return cast + w.n_blocks + (w.n_blocks - 1) + out_cast


def forward_roofline(w, attn_ms, pk, pk_kind):
    """Roofline object of the attention kernel: achieved = the workload's
    causal-adjusted FLOPs over the kernel's mean launch time, against the
    measured dense bf16 peak (the sustained figure for launches over 100 ms,
    the burst one otherwise)."""
    sustained = attn_ms > 100.0
    peak = pk["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    achieved = w.flops / (attn_ms * 1e-3) / 1e12
    roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": None, "kernel": "attn_fwd_kernel",
            "peak_source": f"{pk_kind} {'sustained' if sustained else 'burst'} bf16 dense"}
    rec = attn_traffic(w.name)
    if rec is not None:
        roof["traffic"] = rec["dram_bytes_per_launch"]
        if rec.get("note"):
            roof["traffic_note"] = rec["note"]
    return roof


def time_forward(ra, dev, w, args, steps, warmup, flush, world, inputs=None):
    """Times `steps` ra_ring_attention calls on workload w, inputs resident in
    HBM, L2 flushed between calls (outside the events).  Returns a dict with
    the per-step device times, the slowest rank's total, the attention
    kernel's mean time, the clocks seen, and the device tensors."""
    import torch
    import torch.distributed as dist
    q_h, k_h, v_h = inputs if inputs is not None else workload_inputs(w)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    odt = torch.bfloat16 if w.out_dtype == "bf16" else torch.float32
    out = torch.empty((w.B, w.S, w.Hq, w.D), dtype=odt, device=dev)
    lse = torch.empty((w.B, w.S, w.Hq), dtype=torch.float32, device=dev)
    need = ra.ra_ring_attention_workspace(w.B, w.S, w.Hq, w.D, w.n_blocks, w.gqa_groups, w.partition, q.dtype,
                                          args.order, args.sched, odt)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(events=None):
        ra.ra_ring_attention(q, k, v, w.n_blocks, w.causal, w.partition, w.gqa_groups, out=out, lse=lse,
                             workspace=ws, order=args.order, sched=args.sched, attn_events=events,
                             tiling=args.tiling)

    for _ in range(warmup):
        flush()
        step()
    torch.cuda.synchronize()
    if ra.ra_get_device_status() != 0:
        raise SystemExit(f"{w.name}: device status not OK after warm-up")
    # The timed steps carry only their bracketing events (events the library
    # records inside the call cost about 10 us of GPU time per step).
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = Clocks(local_gpu_id(dev))
    time.sleep(0.3)
    for i in range(steps):
        flush()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(step_ms), dev)
    one_launch = args.sched in ("auto", "persistent") and w.in_dtype == "bf16"
    if one_launch:
        # the call is the one attention launch: the step events time it
        attn_ms = statistics.mean(step_ms)
    else:
        # the attention launches alone: events the library records around them
        Ka = min(steps, 200)
        av = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(Ka)]
        for i in range(Ka):
            flush()
            step(av[i])
        torch.cuda.synchronize()
        attn_ms = statistics.mean(a.elapsed_time(b) for a, b in av)
    status = ra.ra_get_device_status()
    return {"step_ms": step_ms, "total_ms": total_ms, "attn_ms": attn_ms, "clocks": clk, "status": status,
            "tensors": (q, k, v, out, lse, ws), "host": (q_h, k_h, v_h), "stream": stream}


def time_e2e(ra, dev, w, args, fw, steps, world):
    """The same call end to end through the public API with host buffers:
    every step copies its Q, K, V from pinned host memory, makes the call
    and reads out and lse back.  Two sets of device buffers and three streams
    let step i+1's upload, step i's call and step i-1's download overlap
    (PCIe is full duplex), as a caller streaming batches through the library
    would."""
    import torch
    import torch.distributed as dist
    q, k, v, out, lse, ws = fw["tensors"]
    q_h, k_h, v_h = fw["host"]
    stream = fw["stream"]
    qp, kp, vp = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
    bufs = [(q, k, v, out, lse, ws),
            (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(out),
             torch.empty_like(lse), torch.empty_like(ws))]
    host_out = [(torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                 torch.empty(lse.shape, dtype=lse.dtype).pin_memory()) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_steps(n, e_begin=None, e_end=None):
        ev_c, ev_o = [], []
        if e_begin is not None:
            e_begin.record(s_in)
        for i in range(n):
            qd, kd, vd, od, ld, wd = bufs[i % 2]
            if i >= 2:
                s_in.wait_event(ev_c[i - 2])  # step i-2's call has read these inputs
            with torch.cuda.stream(s_in):
                qd.copy_(qp, non_blocking=True)
                kd.copy_(kp, non_blocking=True)
                vd.copy_(vp, non_blocking=True)
            e_in = torch.cuda.Event()
            e_in.record(s_in)
            stream.wait_event(e_in)
            if i >= 2:
                stream.wait_event(ev_o[i - 2])  # step i-2's results are on the host
            ra.ra_ring_attention(qd, kd, vd, w.n_blocks, w.causal, w.partition, w.gqa_groups, out=od, lse=ld,
                                 workspace=wd, order=args.order, sched=args.sched, tiling=args.tiling,
                                 stream=stream)
            ev_c.append(torch.cuda.Event())
            ev_c[-1].record(stream)
            s_out.wait_event(ev_c[-1])
            with torch.cuda.stream(s_out):
                host_out[i % 2][0].copy_(od, non_blocking=True)
                host_out[i % 2][1].copy_(ld, non_blocking=True)
            ev_o.append(torch.cuda.Event())
            ev_o[-1].record(s_out)
        if e_end is not None:
            e_end.record(s_out)

    e2e_steps(3)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e2e_steps(steps, e0, e1)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    h2d = sum(t.numel() * t.element_size() for t in (q, k, v))
    d2h = out.numel() * out.element_size() + lse.numel() * lse.element_size()
    del bufs, host_out, qp, kp, vp
    return {"value": replica_throughput(w.flops, world, steps, e_ms), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps, "warmup": 3,
            "ms_per_step": e_ms / steps,
            "pipelining": "uploads, calls and downloads on three streams, two buffer sets"}


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    import blockwise_exact_attention_block_b200 as ra

    w = WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    flush = L2Flush(dev)
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    l2 = f"{L2_FLUSH_DESC} (L2 {l2_bytes >> 20} MiB)"
    pk, pk_kind = peaks()
    K = args.steps

    fw = time_forward(ra, dev, w, args, K, args.warmup, flush, world)
    status = fw["status"]
    roof = forward_roofline(w, fw["attn_ms"], pk, pk_kind)
    e2e = None
    if not args.no_e2e:
        # long calls: a few steps are enough for the pipeline's steady state
        Ke = max(3, min(K, 200 if fw["attn_ms"] < 100.0 else 3))
        e2e = time_e2e(ra, dev, w, args, fw, Ke, world)
    host = fw["host"]
    total_ms, attn_ms, clk = fw["total_ms"], fw["attn_ms"], fw["clocks"]
    del fw
    torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, host)
    del host

    # The other attention workloads, each timed the same way (its own steps,
    # warm-up, clocks and roofline).
    side = {}
    if not args.no_side:
        for name, steps in SIDE_WORKLOADS.items():
            if name == w.name:
                continue
            ws_ = WORKLOADS[name]
            r = time_forward(ra, dev, ws_, args, steps, 5, flush, world)
            status = status or r["status"]
            side[name] = {"value": replica_throughput(ws_.flops, world, steps, r["total_ms"]), "unit": "TFLOP/s",
                          "ms_per_step": r["total_ms"] / steps, "steps": steps, "warmup": 5,
                          "config": workload_config(ws_, args, l2),
                          "roofline": forward_roofline(ws_, r["attn_ms"], pk, pk_kind), "clocks": r["clocks"],
                          "gpu_launches": steps * launches_per_step(ws_, args.sched)}
            del r
            torch.cuda.empty_cache()

    merge = None
    if not args.no_merge:
        mclk = Clocks(local_gpu_id(dev))
        gbs, mms = bench_merge(ra, dev, 1048576, 2, 10, flush)
        merge = {"kernel": "merge_partial_kernel", "tokens": 1048576, "heads": 32, "D": 128, "partials": 2,
                 "GB/s": gbs, "ms": mms, "peak_GB/s": pk["hbm_gbs"], "frac": gbs / pk["hbm_gbs"],
                 "bytes_per_row": 12 * 128 + 12, "clocks": mclk.stop()}

    decode = None
    if not args.no_decode and world == 1:
        from seeded_inputs import DECODE_WORKLOADS
        dw = DECODE_WORKLOADS["decode1m"]
        dclk = Clocks(local_gpu_id(dev))
        gbs, dms, splits = bench_decode(ra, dev, dw, 10, flush)
        decode = {"kernel": "decode_partial_kernel + decode_combine_kernel", "workload": "decode1m", "B": dw.B,
                  "Tq": dw.Tq, "Skv": dw.Skv, "Hq": dw.Hq, "Hkv": dw.Hkv, "D": dw.D, "chunks": splits,
                  "GB/s": gbs, "ms": dms, "peak_GB/s": pk["hbm_gbs"], "frac": gbs / pk["hbm_gbs"],
                  "clocks": dclk.stop()}

    backward = None
    if not args.no_backward and world == 1:
        bw = WORKLOADS[args.backward_workload]
        bclk = Clocks(local_gpu_id(dev))
        tf, ktf, bms, bkms = bench_backward(ra, dev, bw, 20 if bw.S <= 32768 else 2, flush, args.order)
        bclk = bclk.stop()
        bpeak = pk["bf16_tflops_sustained" if bkms > 100.0 else "bf16_tflops"]
        brec = attn_traffic(bw.name, "attn_bwd_traffic.json", BWD_SOURCES)
        backward = {"kernel": "bwd_dkv_kernel + bwd_dq_kernel (+ bwd_prep_kernel in the call)",
                    "workload": bw.name, "flops_per_step": 2.5 * bw.flops, "TFLOP/s": tf, "kernels_TFLOP/s": ktf,
                    "ms": bms, "kernels_ms": bkms, "peak_TFLOP/s": bpeak, "frac": ktf / bpeak,
                    "traffic": brec["dram_bytes_per_launch"] if brec else None, "clocks": bclk}
    status = status or ra.ra_get_device_status()

    value = replica_throughput(w.flops, world, K, total_ms)
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": total_ms / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded randn, bf16-rounded)", "config": workload_config(w, args, l2),
            "pct_of_peak": 100.0 * roof["frac"], "attn_kernel_ms": attn_ms, "roofline": roof,
            "cpu_baseline": cpu, "e2e": e2e, "clocks": clk, "gpu_launches": K * launches_per_step(w, args.sched),
            "configs": side, "merge": merge, "decode": decode, "backward": backward,
            "device_status": ra.ra_status_string(status)}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0 if status == 0 else 1


def run_merge_sweep(args):
    import torch
    import blockwise_exact_attention_block_b200 as ra
    from seeded_inputs import MERGE_PARTIALS, MERGE_TOKENS
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    flush = L2Flush(dev)
    pk, pk_kind = peaks()
    sweep = []
    Ts = args.merge_T or MERGE_TOKENS
    ks = args.merge_k or MERGE_PARTIALS
    for T in Ts:
        for k in ks:
            reps = 10 if T <= 262144 else 3
            pw, pw_ms = bench_merge(ra, dev, T, k, reps, flush)
            kw, kw_ms = bench_merge(ra, dev, T, k, reps, flush, kway=True)
            sweep.append({"T": T, "k": k, "pairwise_GB/s": pw, "pairwise_ms_per_launch": pw_ms,
                          "pairwise_frac": pw / pk["hbm_gbs"], "kway_GB/s": kw, "kway_ms": kw_ms,
                          "kway_frac": None if kw is None else kw / pk["hbm_gbs"],
                          "bytes_per_pairwise_launch": T * 32 * (12 * 128 + 12)})
    top = max(sweep, key=lambda r: (r["T"], -r["k"]))
    line = {"metric": "merge GB/s (% of HBM peak)", "value": top["pairwise_GB/s"], "unit": "GB/s", "n_gpus": 1,
            "steps": None, "warmup": 2, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic (device randn / rand)",
            "config": {"workload": "merge sweep [T,32,128] fp32", "T": Ts, "k": ks,
                       "headline": {"T": top["T"], "k": top["k"]}, "l2": L2_FLUSH_DESC},
            "roofline": {"bound": "hbm", "achieved": top["pairwise_GB/s"], "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": top["pairwise_GB/s"] / pk["hbm_gbs"], "traffic": None,
                         "peak_source": f"{pk_kind} copy bandwidth"},
            "sweep": sweep}
    print(json.dumps(line))
    return 0


def timeline_summary(rec, event_ms, one_launch=True):
    """Summary of one launch's per-CTA records (start ns, end ns, SM id | work
    units << 32, SM cycles): span, the heaviest CTA, a least-squares fit of
    CTA duration to work units, how many CTAs started after the first wave,
    and the SM clock the CTAs ran at (cycles over time).  event_ms brackets
    this launch alone when one_launch, else more launches (the backward's two
    kernels): then no launch overhead is derived from it."""
    import numpy as np
    r = rec[rec[:, 1] > 0]
    t0 = int(r[:, 0].min())
    start, end = (r[:, 0] - t0) / 1e3, (r[:, 1] - t0) / 1e3
    sm = r[:, 2] & 0xFFFFFFFF
    dur, work = end - start, (r[:, 2] >> 32).astype(float)
    mhz = float(r[:, 3].sum()) / max(float(dur.sum()), 1e-9)
    span = float(end.max())
    i = int(np.argmax(dur))
    A = np.stack([np.ones_like(work), work], 1)
    fit = np.linalg.lstsq(A, dur, rcond=None)[0]
    later = start > 2.0
    n_sm = len(set(sm.tolist()))
    return {"ctas": int(len(r)), "sms": n_sm, "event_us": event_ms * 1e3, "span_us": span,
            "launch_overhead_us": event_ms * 1e3 - span if one_launch else None,
            "heaviest_cta": {"work": int(work[i]), "us": float(dur[i]), "of_span": float(dur[i]) / span},
            "fit_us": {"fixed": float(fit[0]), "per_unit": float(fit[1])},
            "ctas_after_first_wave": int(later.sum()),
            "last_end_of_first_wave_us": float(end[~later].max()),
            "mean_sm_busy_us": float(dur.sum()) / n_sm,
            "work_units": int(work.sum()),
            "sm_mhz_in_ctas": mhz,
            "cycles_per_unit": float(fit[1]) * mhz}


def run_cta_timeline(args):
    """--cta-timeline: after warm-up, one launch of each kernel with the
    per-CTA timeline on (ra_set_cta_timeline), summarised.  Times in us."""
    import torch
    import blockwise_exact_attention_block_b200 as ra
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    flush = L2Flush(dev)
    w = WORKLOADS[args.workload]
    q, k, v = (x.to(dev) for x in workload_inputs(w))
    odt = torch.bfloat16 if w.out_dtype == "bf16" else torch.float32
    rec = torch.zeros((1 << 16, 4), dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream(dev)

    def fwd(events=None):
        return ra.ra_ring_attention(q, k, v, w.n_blocks, w.causal, w.partition, w.gqa_groups, out_dtype=odt,
                                    order=args.order, sched=args.sched, tiling=args.tiling, attn_events=events)

    calls = {"attn_fwd": fwd}
    if args.backward:
        from seeded_inputs import backward_inputs
        _, _, _, do = backward_inputs(w.B, w.S, w.Hq, w.Hkv, w.D, w.in_dtype, seed=10)
        do = do.to(dev)
        o, l = fwd()

        def bwd(events=None):
            return ra.ra_ring_attention_backward(q, k, v, o, l, do, w.n_blocks, w.causal, w.partition, w.gqa_groups,
                                                 order=args.order, attn_events=events)
        calls["bwd_dkv"] = calls["bwd_dq"] = bwd
    clocks = Clocks(local_gpu_id(dev))
    out = {}
    for name, fn in calls.items():
        for _ in range(args.warmup + args.steps):  # warm-up, and clocks up to their load level
            flush()
            fn()
        best = None
        for _ in range(3):
            flush()
            rec.zero_()
            ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            ra.ra_set_cta_timeline(rec, name)
            try:
                fn(ev)
                torch.cuda.synchronize()
            finally:
                ra.ra_set_cta_timeline(None)
            summ = timeline_summary(rec.cpu().numpy(), ev[0].elapsed_time(ev[1]), one_launch=name == "attn_fwd" and args.sched in ("auto", "persistent")
                                    and w.in_dtype == "bf16")
            if best is None or summ["span_us"] < best["span_us"]:
                best = summ
        out[name] = best
    clk = clocks.stop()
    status = ra.ra_get_device_status()
    line = {"metric": "per-CTA timeline", "config": workload_config(w, args, L2_FLUSH_DESC), "kernels": out,
            "note": "the launch with the shortest CTA span of three; event_us from events the library records "
                    "around the kernels (the backward's pair of kernels for both backward entries)",
            "clocks": clk, "device_status": ra.ra_status_string(status)}
    print(json.dumps(line))
    return 0 if status == 0 else 1


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.cta_timeline:
        return run_cta_timeline(args)
    if args.merge_sweep:
        return run_merge_sweep(args)
    if args.decode:
        return run_decode(args)
    if args.backward:
        return run_backward(args)
    if args.shards:
        return run_shards(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
