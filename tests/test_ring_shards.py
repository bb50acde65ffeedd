"""Sequence-parallel ring and TokenRing across ranks (one block per rank), on
the CPU.

The rank programs of blockwise_exact_attention_block_b200.ring are run with
their device work replaced by the oracle (fp64 block partials and the merge
rule), so these tests check the host logic: which block each rank holds at
each step, which messages travel where, the causal skips, and the merge
order.  They run in one process (the lockstep executor) and as gloo ranks
(torch.distributed point-to-point, 2 and 4 processes).  Each rank's block
result, gathered back to original positions, must equal the oracle's full
attention.  The same programs on the CUDA kernels are in
tests/test_gpu_parity.py.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from oracle import attention as F  # noqa: E402
from oracle import blockwise as K  # noqa: E402
from seeded_inputs import attention_inputs  # noqa: E402


def _ring():
    # the ring module alone: it loads the CUDA library only when BlockOps is built
    import importlib.util
    path = os.path.join(ROOT, "blockwise_exact_attention_block_b200", "ring.py")
    spec = importlib.util.spec_from_file_location("ring_host_logic", path)
    mod = importlib.util.module_from_spec(spec)
    sys.modules[spec.name] = mod
    spec.loader.exec_module(mod)
    return mod


R = _ring()


class OracleOps:
    """The device work of a step, done by the oracle in fp64 on the CPU.
    Records the (q_block, kv_block) pairs folded into each query block."""

    def __init__(self, S, n, causal, partition, groups):
        self.S, self.n, self.causal, self.groups = S, n, causal, groups
        self.pos = K.partition_perm(S, n, partition).reshape(n, S // n)
        self.merged = {}     # q block -> KV blocks in the order they were folded in
        self.computed = []   # (q block, KV block) in the order computed
        self.partials = {}   # (q block, KV block) -> block_lse, to recognise a partial that travelled

    def new_state(self, q):
        B, L, Hq, D = q.shape
        return (torch.zeros((B, L, Hq, D), dtype=torch.float64),
                torch.full((B, L, Hq), float("-inf"), dtype=torch.float64))

    def new_partial(self, q):
        B, L, Hq, D = q.shape
        buf = torch.empty(B * L * Hq * (D + 1), dtype=torch.float64)
        return buf, buf[: B * L * Hq * D].view(B, L, Hq, D), buf[B * L * Hq * D:].view(B, L, Hq)

    def _partial(self, q, k, v, qb, kb):
        self.computed.append((qb, kb))
        bo, bl = K.block_partial(q, k, v, self.pos[qb], self.pos[kb], self.causal, self.groups)
        self.partials[(qb, kb)] = bl
        return bo, bl

    def _fold(self, out, lse, bo, bl, pair):
        o, l = K.merge_rule(out.numpy(), lse.numpy(), bo, bl)
        out.copy_(torch.from_numpy(o))
        lse.copy_(torch.from_numpy(l))
        self.merged.setdefault(pair[0], []).append(pair[1])

    def attn_merge(self, q, k, v, qb, kb, out, lse):
        bo, bl = self._partial(q, k, v, qb, kb)
        self._fold(out, lse, bo, bl, (qb, kb))

    def attn(self, q, k, v, qb, kb, block_out, block_lse):
        bo, bl = self._partial(q, k, v, qb, kb)
        block_out.copy_(torch.from_numpy(bo))
        block_lse.copy_(torch.from_numpy(bl))

    def merge(self, out, lse, block_out, block_lse):
        # a message carries no pair index: the pair is recognised by its
        # block_lse among the partials computed in this process (lockstep)
        bl = block_lse.numpy()
        pair = next((key for key, x in self.partials.items() if np.array_equal(x, bl)), (None, None))
        self._fold(out, lse, block_out.numpy(), bl, pair)


def shard(x, S, n, partition, r):
    return torch.cat([x[:, p:p + l] for p, l in R.block_segments(S, n, partition, r)], dim=1).contiguous()


def gather(blocks, S, n, partition):
    B = blocks[0].shape[0]
    full = torch.empty((B, S) + tuple(blocks[0].shape[2:]), dtype=blocks[0].dtype)
    for r, blk in enumerate(blocks):
        row = 0
        for p, l in R.block_segments(S, n, partition, r):
            full[:, p:p + l] = blk[:, row:row + l]
            row += l
    return full


def inputs(S, Hq=4, Hkv=2, D=8, seed=3):
    q, k, v = attention_inputs(1, S, Hq, Hkv, D, dtype="bf16", seed=seed)
    return q.double(), k.double(), v.double()


CASES = [(n, order, part, causal) for n in (1, 2, 3, 4, 8) for order in R.ORDERS
         for part in ("contiguous", "zigzag") for causal in (True, False)]


@pytest.mark.parametrize("n,order,partition,causal", CASES)
def test_lockstep_ranks_equal_full_attention(n, order, partition, causal):
    S = 16 * n
    q, k, v = inputs(S)
    ops = OracleOps(S, n, causal, partition, 2)
    res = R.ring_attention_lockstep([shard(q, S, n, partition, r) for r in range(n)],
                                    [shard(k, S, n, partition, r) for r in range(n)],
                                    [shard(v, S, n, partition, r) for r in range(n)],
                                    S, causal, partition, order, ops=ops)
    out = gather([o for o, _ in res], S, n, partition).numpy()
    lse = gather([l for _, l in res], S, n, partition).numpy()
    ro, rl = F.full_attention(q, k, v, causal, 2)
    assert np.max(np.abs(out - ro)) <= 1e-12
    assert np.max(np.abs(lse - rl)) <= 1e-12
    # every visible pair computed exactly once, and no other
    want = sorted((qb, kb) for qb in range(n) for kb in range(n)
                  if R.pair_visible(S, n, partition, causal, qb, kb))
    assert sorted(ops.computed) == want


@pytest.mark.parametrize("n", [2, 3, 4, 5, 8, 16])
def test_steps_follow_the_pages_order(n):
    # Ring: at step s rank r meets KV block (r - s) mod n, folded in that
    # order.  TokenRing: at step s (1-based) rank j computes query block
    # (j - s + 1) mod n, so query block r meets KV blocks r, r + 1, ...
    S = 16 * n
    q, k, v = inputs(S)
    blocks = [[shard(x, S, n, "zigzag", r) for r in range(n)] for x in (q, k, v)]
    ops = OracleOps(S, n, True, "zigzag", 2)
    R.ring_attention_lockstep(*blocks, S, True, "zigzag", "ring", ops=ops)
    for r in range(n):
        # rank r computes the pairs of query block r, in step order
        assert [kb for qb, kb in ops.computed if qb == r] == [(r - s) % n for s in range(n)]
        assert ops.merged[r] == [(r - s) % n for s in range(n)]
    ops = OracleOps(S, n, True, "zigzag", 2)
    R.ring_attention_lockstep(*blocks, S, True, "zigzag", "tokenring", ops=ops)
    for j in range(n):
        # rank j computes the pairs of KV block j, in step order
        assert [qb for qb, kb in ops.computed if kb == j] == [(j - s + 1) % n for s in range(1, n + 1)]
        # and query block j is folded with KV blocks j, j + 1, ... (step 1 locally)
        assert ops.merged[j] == [(j + s) % n for s in range(n)]


def test_causal_contiguous_skips_pairs_and_messages():
    # contiguous causal: KV block j > q block i is fully masked; those pairs
    # run nothing and their partials are never sent
    n, S = 4, 64
    q, k, v = inputs(S)
    blocks = [[shard(x, S, n, "contiguous", r) for r in range(n)] for x in (q, k, v)]
    for order in R.ORDERS:
        ops = OracleOps(S, n, True, "contiguous", 2)
        R.ring_attention_lockstep(*blocks, S, True, "contiguous", order, ops=ops)
        assert len(ops.computed) == n * (n + 1) // 2
        assert all(kb <= qb for qb, kb in ops.computed)
    assert R.pair_visible(S, n, "zigzag", True, 0, n - 1)   # zigzag: every pair sees keys
    assert not R.pair_visible(S, n, "contiguous", True, 0, 1)


def _count_messages(order, n, S, partition, causal):
    q, k, v = inputs(S, Hq=2, Hkv=1, D=4)
    progs = [R.program(order, r, n, shard(q, S, n, partition, r), shard(k, S, n, partition, r),
                       shard(v, S, n, partition, r), OracleOps(S, n, causal, partition, 2), S, causal, partition)
             for r in range(n)]
    count = {"sends": 0}

    class Counting:
        def __init__(self, prog):
            self.prog = prog

        def send(self, x):
            msg = self.prog.send(x)
            if isinstance(msg, R.Post):
                count["sends"] += len(msg.sends)
            return msg

    R.run_lockstep([Counting(p) for p in progs])
    return count["sends"]


def test_message_counts():
    n, S = 4, 64
    # ring: every rank forwards K/V n - 1 times
    assert _count_messages("ring", n, S, "zigzag", True) == n * (n - 1)
    # TokenRing: Q forwarded n - 1 times per rank, plus one partial per remote pair
    assert _count_messages("tokenring", n, S, "zigzag", True) == n * (n - 1) + n * (n - 1)
    remote_visible = sum(1 for i in range(n) for j in range(n) if i != j and j <= i)
    assert _count_messages("tokenring", n, S, "contiguous", True) == n * (n - 1) + remote_visible


def test_lockstep_reports_unmatched_messages():
    def lonely():
        h = yield R.Post(recvs=[(torch.zeros(2), 1)])
        yield R.Wait(h)

    def idle():
        return None
        yield  # noqa: unreachable - makes this a generator

    with pytest.raises(RuntimeError, match="wait on messages"):
        R.run_lockstep([lonely(), idle()])


def test_lockstep_rejects_mismatched_shapes():
    def sender():
        h = yield R.Post(sends=[(torch.zeros(3), 1)])
        yield R.Wait(h)

    def receiver():
        h = yield R.Post(recvs=[(torch.zeros(2), 0)])
        yield R.Wait(h)

    with pytest.raises(RuntimeError, match="into"):
        R.run_lockstep([sender(), receiver()])


# ------------------------------------------------------------ gloo ranks

def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_worker(rank, world, port, order, partition, causal, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        S = 16 * world
        q, k, v = inputs(S)
        ops = OracleOps(S, world, causal, partition, 2)
        o, l = R.ring_attention_dist(shard(q, S, world, partition, rank), shard(k, S, world, partition, rank),
                                     shard(v, S, world, partition, rank), S, causal, partition, order, ops=ops)
        out[rank] = (o.numpy(), l.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,order,partition,causal", [
    (2, "ring", "zigzag", True), (2, "tokenring", "zigzag", True),
    (4, "ring", "contiguous", True), (4, "tokenring", "contiguous", True),
    (4, "tokenring", "zigzag", False)])
def test_gloo_ranks_equal_full_attention(world, order, partition, causal):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = free_port()
    procs = [ctx.Process(target=_gloo_worker, args=(r, world, port, order, partition, causal, out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    S = 16 * world
    q, k, v = inputs(S)
    res = [out[r] for r in range(world)]
    o = gather([torch.from_numpy(x) for x, _ in res], S, world, partition).numpy()
    l = gather([torch.from_numpy(x) for _, x in res], S, world, partition).numpy()
    ro, rl = F.full_attention(q, k, v, causal, 2)
    assert np.max(np.abs(o - ro)) <= 1e-12
    assert np.max(np.abs(l - rl)) <= 1e-12


def _subgroup_worker(rank, world, port, out):
    # a ring over ranks {0, 2} of three: block index = rank inside the group
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        group = dist.new_group([0, 2])
        if rank in (0, 2):
            S, n, part = 32, 2, "zigzag"
            q, k, v = inputs(S)
            r = dist.get_rank(group)
            ops = OracleOps(S, n, True, part, 2)
            o, l = R.ring_attention_dist(shard(q, S, n, part, r), shard(k, S, n, part, r), shard(v, S, n, part, r),
                                         S, True, part, "tokenring", group=group, ops=ops)
            out[r] = (o.numpy(), l.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_gloo_ring_over_a_subgroup():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = free_port()
    procs = [ctx.Process(target=_subgroup_worker, args=(r, 3, port, out)) for r in range(3)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    S, n, part = 32, 2, "zigzag"
    q, k, v = inputs(S)
    o = gather([torch.from_numpy(out[r][0]) for r in range(n)], S, n, part).numpy()
    l = gather([torch.from_numpy(out[r][1]) for r in range(n)], S, n, part).numpy()
    ro, rl = F.full_attention(q, k, v, True, 2)
    assert np.max(np.abs(o - ro)) <= 1e-12
    assert np.max(np.abs(l - rl)) <= 1e-12
