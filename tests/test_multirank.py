"""The N > 1 path on the CPU: replicas timed by the slowest rank, and the
per-step estimate of the sequence-parallel bench mode.

bench.py --gpus N runs one replica of the workload per rank (weak scaling,
no exchange on the data path); the only collectives are the barrier and the
max over ranks of the timed region.  These tests run that logic as two gloo
ranks, and the reference arm under torchrun with two ranks.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mx = bench.max_over_ranks(times[rank])
        out[rank] = mx
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    port = free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    times = [12.5, 30.25]
    procs = [ctx.Process(target=_worker, args=(r, 2, port, times, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == max(times)


def test_max_over_ranks_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5


def test_replica_throughput_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    # 2 replicas of 1e12 FLOP per step, 10 steps in 1 s (slowest rank) -> 20 TFLOP/s
    assert bench.replica_throughput(1e12, 2, 10, 1000.0) == pytest.approx(20.0)


def test_reference_arm_under_torchrun_two_ranks():
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--workload", "tiny", "--steps", "1", "--warmup", "3"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


# ------------------------------------- sequence-parallel estimate (bench --shards)

@pytest.mark.parametrize("n", [1, 2, 3, 4, 8])
def test_shard_steps_cover_every_pair_once(n):
    sys.path.insert(0, ROOT)
    import bench
    for order, steps in (("ring", range(n)), ("tokenring", range(1, n + 1))):
        pairs = [p for s in steps for p in bench.shard_pairs(n, order, s)]
        assert sorted(pairs) == [(i, j) for i in range(n) for j in range(n)]
        for s in steps:  # one pair per rank and step: ranks own query blocks (ring) or KV blocks (TokenRing)
            own = [p[0] if order == "ring" else p[1] for p in bench.shard_pairs(n, order, s)]
            assert own == list(range(n))
    if n == 4:
        assert bench.shard_pairs(n, "ring", 1) == [(0, 3), (1, 0), (2, 1), (3, 2)]
        assert bench.shard_pairs(n, "tokenring", 2) == [(3, 0), (0, 1), (1, 2), (2, 3)]


def test_shard_step_estimate_takes_the_slowest_rank():
    sys.path.insert(0, ROOT)
    import bench
    n = 4
    # contiguous causal: only pairs kv <= q run; pair time grows with the query block
    pair_ms = {(i, j): 1.0 + i for i in range(n) for j in range(n) if j <= i}
    ring = bench.shard_step_estimate(pair_ms, n, "ring")
    # ring step s: rank r meets KV r - s, visible for r >= s; the slowest is rank 3
    assert ring == [4.0, 4.0, 4.0, 4.0]
    tok = bench.shard_step_estimate(pair_ms, n, "tokenring", merge_ms=0.5)
    # TokenRing step s: rank j computes query block j - s + 1 (mod n); visible when j <= it
    want = []
    for s in range(1, n + 1):
        ts = [1.0 + (j - s + 1) % n + (0.5 if s > 1 else 0.0) for j in range(n) if j <= (j - s + 1) % n]
        want.append(max(ts, default=0.0))
    assert tok == want
    assert bench.shard_step_estimate({}, n, "ring") == [0.0] * n


def test_shard_exchange_bytes():
    sys.path.insert(0, ROOT)
    import bench
    from seeded_inputs import WORKLOADS
    w = WORKLOADS["gqa24k"]  # 24,000 tokens, 4 blocks of 6,000, 32 query / 8 KV heads, D = 128
    assert bench.shard_exchange_bytes(w, "ring") == 2 * 6000 * 8 * 128 * 2
    assert bench.shard_exchange_bytes(w, "tokenring") == 6000 * 32 * 128 * 2 + 6000 * 32 * 129 * 4


def test_timeline_summary_on_a_known_schedule():
    # three SMs, five CTAs: CTA cost 2 us + 1 us per work unit; two CTAs start
    # after the first wave on the SMs that free up first
    import numpy as np
    import bench
    t0 = 10**12
    rows = []  # start ns, end ns, SM, work
    for sm, (start, work) in enumerate([(0.0, 6), (0.0, 3), (0.0, 2)]):
        rows.append((start, start + 2 + work, sm, work))
    rows.append((4.0, 4.0 + 2 + 1, 2, 1))   # after SM 2's first CTA (ends at 4)
    rows.append((5.0, 5.0 + 2 + 0, 1, 0))   # after SM 1's first CTA (ends at 5)
    # 1,500 cycles per us: a 1.5 GHz clock
    rec = np.array([(t0 + int(a * 1e3), t0 + int(b * 1e3), sm | (w << 32), int((b - a) * 1500))
                    for a, b, sm, w in rows] + [(0, 0, 0, 0)] * 3, dtype=np.int64)
    s = bench.timeline_summary(rec, event_ms=0.0105)
    assert s["ctas"] == 5 and s["sms"] == 3
    assert abs(s["span_us"] - 8.0) < 1e-9
    assert abs(s["launch_overhead_us"] - 2.5) < 1e-9
    assert s["heaviest_cta"] == {"work": 6, "us": 8.0, "of_span": 1.0}
    assert abs(s["fit_us"]["fixed"] - 2.0) < 1e-9 and abs(s["fit_us"]["per_unit"] - 1.0) < 1e-9
    assert s["ctas_after_first_wave"] == 2
    assert abs(s["last_end_of_first_wave_us"] - 8.0) < 1e-9
    assert abs(s["mean_sm_busy_us"] - (8 + 5 + 4 + 3 + 2) / 3) < 1e-9
    assert s["work_units"] == 12
    assert abs(s["sm_mhz_in_ctas"] - 1500.0) < 1e-6
    assert abs(s["cycles_per_unit"] - 1500.0) < 1e-6
