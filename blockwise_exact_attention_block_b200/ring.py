"""Sequence parallelism: one block of the sequence per rank, exchanged on a ring.

Anthology of the SOTA, SOTA-181 (ring attention, Liu et al. 2023): the
sequence is cut into blocks, one per device on a ring.  Every device keeps
its query block; at each step it computes attention against the key/value
block it holds and passes that block to the next device, so after n steps
every query block has met every key/value block, and the result is exact.

TokenRing review (pith.science, arXiv 2412.20501), "Core claim" and "What
carries the argument": TokenRing keeps K and V in place and sends the query
block forward instead; the partial result (block_out, block_lse) of each
step goes back to the query block's owner, which folds it in with the update
rule.  "Referee Report / major comments, Algorithm 1 (section 3.2)": at step
s (1-based) device j computes query block t = (j - s + 1) mod n against its
own key/value block j; the last partials go to device j - n + 1 (mod n).

A rank's work is a generator (a "program") that yields the messages of each
step and runs the step's device work between posting them and waiting for
them, so that transfers overlap compute:

    handle = yield Post(sends=[(tensor, peer)], recvs=[(tensor, peer)])
    ...device work of the step...
    yield Wait(handle)

Messages between two ranks are matched in the order they are posted.  A
program never writes a tensor it has posted for sending, and never reads one
posted for receiving, before the matching Wait.  Two executors run programs:

* run_dist      - torch.distributed point-to-point operations (NCCL between
                  GPUs, one process per GPU; gloo between CPU processes).
* run_lockstep  - the programs of all ranks in one process: each send is
                  copied into its receive once both are posted, and a rank
                  blocked in a Wait resumes once its step's messages are
                  all paired.  It checks the schedules and the device work
                  of all ranks on a single device.

The device work comes from an ``ops`` object; BlockOps, the default, calls
the CUDA library (ra_block_attn_merge for a pair whose result stays on the
rank, ra_block_attn + ra_merge_partial for a partial that travels).

Layout on every rank: q [B, L, Hq, D] and k, v [B, L, Hkv, D] (bf16) are the
rows of this rank's block in partition order (contiguous: tokens
[r L, (r + 1) L); zigzag: chunk r then chunk 2n - 1 - r, chunk c = S / 2n);
the result is (out fp32 [B, L, Hq, D], lse fp32 [B, L, Hq]) for the same
rows.  block_segments() gives the original positions of a block's rows.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

ORDERS = ("ring", "tokenring")


@dataclass
class Post:
    """Messages of one step: (tensor, peer rank) pairs."""
    sends: list = field(default_factory=list)
    recvs: list = field(default_factory=list)


@dataclass
class Wait:
    handle: object


# ------------------------------------------------------------- partition

def block_segments(S: int, n: int, partition: str, r: int):
    """Runs of original positions [(pos, len), ...] of block r, in row order."""
    if partition == "contiguous":
        if S % n:
            raise ValueError("contiguous partition needs S divisible by the ring size")
        L = S // n
        return [(r * L, L)]
    if partition == "zigzag":
        if S % (2 * n):
            raise ValueError("zigzag partition needs S divisible by twice the ring size")
        c = S // (2 * n)
        return [(r * c, c), ((2 * n - 1 - r) * c, c)]
    raise ValueError(f"unknown partition {partition!r}")


def pair_visible(S: int, n: int, partition: str, causal: bool, q_block: int, kv_block: int) -> bool:
    """False when no query of q_block may see any key of kv_block (causal
    mask over original positions): the pair contributes nothing and is
    skipped, with its messages."""
    if not causal:
        return True
    q_last = max(p + l - 1 for p, l in block_segments(S, n, partition, q_block))
    k_first = min(p for p, _ in block_segments(S, n, partition, kv_block))
    return k_first <= q_last


# ------------------------------------------------------------------- ops

class BlockOps:
    """Device work of a step on the CUDA library (bf16 inputs, fp32 results).

    Every launch goes to torch's current stream.  That is the stream the
    point-to-point operations of `run_dist` are ordered against (NCCL's own
    stream waits on it when a step is posted, and it waits on NCCL's stream
    at each Wait), so a receive never overwrites a buffer that a kernel of an
    earlier step is still reading.  To run on another stream, make it current
    (`with torch.cuda.stream(s):`) around the whole program."""

    def __init__(self, S: int, n: int, causal: bool, partition: str):
        from . import ra_block_attn, ra_block_attn_merge, ra_merge_partial
        self._attn, self._attn_merge, self._merge = ra_block_attn, ra_block_attn_merge, ra_merge_partial
        self.S, self.n, self.causal, self.partition = S, n, causal, partition

    def new_state(self, q):
        """Running (out, lse) of a query block before any pair: (0, -inf)."""
        B, L, Hq, D = q.shape
        out = torch.zeros((B, L, Hq, D), dtype=torch.float32, device=q.device)
        lse = torch.full((B, L, Hq), float("-inf"), dtype=torch.float32, device=q.device)
        return out, lse

    def new_partial(self, q):
        """One flat buffer holding (block_out, block_lse), so that a partial
        travels as one message; block_lse starts 16-byte aligned."""
        B, L, Hq, D = q.shape
        buf = torch.empty(B * L * Hq * (D + 1), dtype=torch.float32, device=q.device)
        return buf, buf[: B * L * Hq * D].view(B, L, Hq, D), buf[B * L * Hq * D:].view(B, L, Hq)

    def attn_merge(self, q, k, v, q_block, kv_block, out, lse):
        self._attn_merge(q, k, v, self.S, self.n, q_block, kv_block, self.causal, out, lse,
                         partition=self.partition)

    def attn(self, q, k, v, q_block, kv_block, block_out, block_lse):
        self._attn(q, k, v, self.S, self.n, q_block, kv_block, self.causal, partition=self.partition,
                   block_out=block_out, block_lse=block_lse)

    def merge(self, out, lse, block_out, block_lse):
        self._merge(out, lse, block_out, block_lse)


# -------------------------------------------------------------- programs

def ring_program(rank: int, n: int, q, k, v, ops, S: int, causal: bool, partition: str):
    """Ring order: K and V travel forward.  At step s (0-based) this rank
    holds KV block (rank - s) mod n, folds that pair into its running
    (out, lse), and meanwhile sends the block on to rank + 1 and receives the
    next one from rank - 1 (double-buffered).  Returns (out, lse)."""
    out, lse = ops.new_state(q)
    kv = [torch.stack((k, v)), None]
    if n > 1:
        kv[1] = torch.empty_like(kv[0])
    for s in range(n):
        cur = kv[s % 2]
        src = (rank - s) % n
        handle = None
        if s + 1 < n:
            handle = yield Post(sends=[(cur, (rank + 1) % n)], recvs=[(kv[(s + 1) % 2], (rank - 1) % n)])
        if pair_visible(S, n, partition, causal, rank, src):
            ops.attn_merge(q, cur[0], cur[1], rank, src, out, lse)
        if handle is not None:
            yield Wait(handle)
    return out, lse


def tokenring_program(rank: int, n: int, q, k, v, ops, S: int, causal: bool, partition: str):
    """TokenRing order: Q travels forward, partials travel back to the owner.

    At step s (1-based) this rank holds query block t = (rank - s + 1) mod n
    and computes it against its own KV block.  Step 1 is its own query block,
    folded straight into (out, lse).  For s >= 2 the partial travels back to
    rank t in the exchange posted at the start of step s + 1 (after step n, a
    last exchange: to rank + 1), which also brings this rank the partial of
    its own query block from the rank that held it at step s,
    (rank + s - 1) mod n; it is folded in once that exchange completes.
    Partials are therefore merged in KV order rank, rank + 1, ...,
    rank + n - 1.  Returns (out, lse)."""
    out, lse = ops.new_state(q)
    qbuf = [q.clone(), torch.empty_like(q) if n > 1 else None]
    send_part = [ops.new_partial(q), ops.new_partial(q)]
    recv_part = [ops.new_partial(q), ops.new_partial(q)]

    def exchange(s, q_fwd):
        """Messages posted at the start of step s (s = n + 1: the last one)."""
        sends, recvs = [], []
        if q_fwd:
            sends.append((qbuf[(s - 1) % 2], (rank + 1) % n))
            recvs.append((qbuf[s % 2], (rank - 1) % n))
        incoming = None
        if s >= 3:
            u = s - 1                       # the step whose partials move now
            t = (rank - u + 1) % n          # owner of the query block this rank held at step u
            if pair_visible(S, n, partition, causal, t, rank):
                sends.append((send_part[u % 2][0], t))
            h = (rank + u - 1) % n          # rank that held this rank's query block at step u
            if pair_visible(S, n, partition, causal, rank, h):
                incoming = recv_part[u % 2]
                recvs.append((incoming[0], h))
        return sends, recvs, incoming

    for s in range(1, n + 1):
        t = (rank - s + 1) % n
        sends, recvs, incoming = exchange(s, s < n)
        handle = (yield Post(sends=sends, recvs=recvs)) if sends or recvs else None
        held = qbuf[(s - 1) % 2]
        if pair_visible(S, n, partition, causal, t, rank):
            if s == 1:
                ops.attn_merge(held, k, v, t, rank, out, lse)
            else:
                _, bo, bl = send_part[s % 2]
                ops.attn(held, k, v, t, rank, bo, bl)
        if handle is not None:
            yield Wait(handle)
        if incoming is not None:
            ops.merge(out, lse, incoming[1], incoming[2])
    if n > 1:
        sends, recvs, incoming = exchange(n + 1, False)
        if sends or recvs:
            handle = yield Post(sends=sends, recvs=recvs)
            yield Wait(handle)
        if incoming is not None:
            ops.merge(out, lse, incoming[1], incoming[2])
    return out, lse


def program(order: str, rank: int, n: int, q, k, v, ops, S: int, causal: bool, partition: str):
    if order == "ring":
        return ring_program(rank, n, q, k, v, ops, S, causal, partition)
    if order == "tokenring":
        return tokenring_program(rank, n, q, k, v, ops, S, causal, partition)
    raise ValueError(f"unknown order {order!r}")


# ------------------------------------------------------------- executors

def run_dist(prog, group=None):
    """Runs one rank's program with torch.distributed point-to-point
    operations on `group` (default: the world); peers are group ranks.
    Returns the program's result."""
    import torch.distributed as dist

    def peer(p):
        return p if group is None else dist.get_global_rank(group, p)

    reply = None
    while True:
        try:
            msg = prog.send(reply)
        except StopIteration as stop:
            return stop.value
        if isinstance(msg, Post):
            p2p = [dist.P2POp(dist.isend, t, peer(p), group) for t, p in msg.sends]
            p2p += [dist.P2POp(dist.irecv, t, peer(p), group) for t, p in msg.recvs]
            reply = dist.batch_isend_irecv(p2p) if p2p else []
        elif isinstance(msg, Wait):
            for req in msg.handle:
                req.wait()
            reply = None
        else:
            raise TypeError(f"a program yielded {type(msg).__name__}")


class _Handle:
    """A posted step: the number of its messages not yet matched."""

    def __init__(self, count: int):
        self.pending = count


def run_lockstep(progs):
    """Runs the programs of all ranks (rank = list index) in one process and
    returns their results.  Sends and receives are paired per (sender,
    receiver) in posting order; a pair is copied as soon as both sides are
    posted, and a Wait returns once all of its step's messages are paired
    (a send completes only against its receive, as between GPUs).  Raises
    RuntimeError when the ranks cannot progress (a send or receive no rank
    matches) or a pair disagrees in shape or type."""
    from collections import deque
    n = len(progs)
    sendq, recvq = {}, {}
    results = [None] * n
    waiting = [None] * n   # handle each rank is blocked on
    replies = [None] * n
    live = set(range(n))

    def pair_up(key):
        sq, rq = sendq.get(key), recvq.get(key)
        while sq and rq:
            (src, hs), (dst, hr) = sq.popleft(), rq.popleft()
            if src.shape != dst.shape or src.dtype != dst.dtype:
                raise RuntimeError(f"message {key}: {tuple(src.shape)} {src.dtype} into "
                                   f"{tuple(dst.shape)} {dst.dtype}")
            dst.copy_(src)
            hs.pending -= 1
            hr.pending -= 1

    while live:
        progressed = False
        for r in sorted(live):
            if waiting[r] is not None:
                if waiting[r].pending:
                    continue
                waiting[r] = None
            progressed = True
            while True:
                try:
                    msg = progs[r].send(replies[r])
                except StopIteration as stop:
                    results[r] = stop.value
                    live.discard(r)
                    break
                if isinstance(msg, Post):
                    h = _Handle(len(msg.sends) + len(msg.recvs))
                    for t, p in msg.sends:
                        sendq.setdefault((r, p), deque()).append((t, h))
                        pair_up((r, p))
                    for t, p in msg.recvs:
                        recvq.setdefault((p, r), deque()).append((t, h))
                        pair_up((p, r))
                    replies[r] = h
                elif isinstance(msg, Wait):
                    replies[r] = None
                    if msg.handle.pending:
                        waiting[r] = msg.handle
                        break
                else:
                    raise TypeError(f"a program yielded {type(msg).__name__}")
        if live and not progressed:
            left = {k: len(v) for k, v in list(sendq.items()) + list(recvq.items()) if v}
            raise RuntimeError(f"ranks {sorted(live)} wait on messages no rank matches: {left}")
    return results


# ---------------------------------------------------------------- entry

def ring_attention_dist(q, k, v, S: int, causal: bool, partition: str = "contiguous", order: str = "ring",
                        group=None, ops=None):
    """Exact attention of this rank's query block over the whole sequence,
    with one block per rank of `group` (block index = group rank).  Call on
    every rank of the group with its own block.  Returns (out, lse) fp32."""
    import torch.distributed as dist
    rank, n = dist.get_rank(group), dist.get_world_size(group)
    ops = ops if ops is not None else BlockOps(S, n, causal, partition)
    return run_dist(program(order, rank, n, q, k, v, ops, S, causal, partition), group)


def ring_attention_lockstep(qs, ks, vs, S: int, causal: bool, partition: str = "contiguous",
                            order: str = "ring", ops=None):
    """All n ranks' blocks (lists indexed by block) in one process; returns
    the list of every block's (out, lse)."""
    n = len(qs)
    ops = ops if ops is not None else BlockOps(S, n, causal, partition)
    return run_lockstep([program(order, r, n, qs[r], ks[r], vs[r], ops, S, causal, partition)
                         for r in range(n)])
