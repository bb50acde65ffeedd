"""GPU parity: the CUDA path (through the C ABI) against the CPU fp64 oracle on
the same seeded inputs.

Tolerances (fixed for this method): bf16 attention inputs -> max-abs error
<= 2e-2 and relative L2 error <= 1e-2, on out and on lse separately; the fp32
merge kernels -> max-abs <= 1e-5 on out and |err| <= 1e-5 * max(1, |lse|) on
lse, against the fp64 rule applied to the same fp32 partials; the zigzag
permutation -> bit-exact.  Workloads too large for the full oracle are checked
on sampled query rows, each computed exactly against every key it may see.
"""
import numpy as np
import pytest
import torch

from oracle import attention as F
from oracle import blockwise as K
from seeded_inputs import DECODE_WORKLOADS, WORKLOADS, attention_inputs, decode_inputs, merge_inputs, workload_inputs

pytestmark = pytest.mark.gpu

ATOL, RTOL_L2 = 2e-2, 1e-2
MERGE_TOL = 1e-5


def assert_close_bf16(got, ref, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    gi, ri = np.isneginf(got), np.isneginf(ref)
    assert np.array_equal(gi, ri), f"{what}: -inf pattern differs"
    fin = ~ri
    if not fin.any():
        return
    err = np.abs(got[fin] - ref[fin])
    mx = float(err.max())
    rel = float(np.linalg.norm(got[fin] - ref[fin]) / max(np.linalg.norm(ref[fin]), 1e-30))
    assert mx <= ATOL, f"{what}: max-abs {mx:.3e} > {ATOL}"
    assert rel <= RTOL_L2, f"{what}: rel-L2 {rel:.3e} > {RTOL_L2}"


def to_np(t):
    return t.detach().float().cpu().numpy()


# -------------------------------------------------------------- permutation

@pytest.mark.parametrize("shape,n,dtype", [((1, 8, 1, 8), 2, torch.float32), ((2, 4096, 8, 128), 4, torch.bfloat16),
                                           ((1, 24000, 4, 128), 4, torch.bfloat16), ((3, 96, 3, 2), 6, torch.float32),
                                           ((1, 96, 3, 2), 3, torch.bfloat16)])
def test_zigzag_permute_bit_exact(cuda_lib, shape, n, dtype):
    ra = cuda_lib
    g = torch.Generator().manual_seed(0)
    x = torch.randn(shape, generator=g).to(dtype)
    perm = K.zigzag_perm(shape[1], n)
    d = ra.ra_zigzag_permute(x.cuda(), n, inverse=False)
    ref = x[:, torch.from_numpy(perm)]
    assert torch.equal(d.cpu(), ref)
    back = ra.ra_zigzag_permute(d, n, inverse=True)
    assert torch.equal(back.cpu(), x)


# ---------------------------------------------------------------- merge rule

def check_merge(got_o, got_l, ref_o, ref_l):
    go, gl = to_np(got_o).astype(np.float64), to_np(got_l).astype(np.float64)
    assert np.array_equal(np.isneginf(gl), np.isneginf(ref_l))
    assert float(np.max(np.abs(go - ref_o))) <= MERGE_TOL
    fin = np.isfinite(ref_l)
    assert np.all(np.abs(gl[fin] - ref_l[fin]) <= MERGE_TOL * np.maximum(1.0, np.abs(ref_l[fin])))


@pytest.mark.parametrize("T", [4096, 65536])
def test_merge_partial_matches_oracle(cuda_lib, T):
    ra = cuda_lib
    outs, lses = merge_inputs(T, 2)
    # empty partials on a few rows: the rule's -inf cases
    lses[1][0, :4] = float("-inf")
    lses[0][1, :4] = float("-inf")
    lses[0][2, :2] = float("-inf")
    lses[1][2, :2] = float("-inf")
    ref_o, ref_l = K.merge_rule(outs[0].double().numpy(), lses[0].double().numpy(), outs[1].double().numpy(),
                                lses[1].double().numpy())
    o, l = outs[0].cuda(), lses[0].cuda()
    ra.ra_merge_partial(o, l, outs[1].cuda(), lses[1].cuda())
    check_merge(o, l, ref_o, ref_l)


def test_merge_partial_full_size_sampled_rows(cuda_lib):
    """The bench's merge: two [1,048,576, 32, 128] fp32 partials (16 GiB each,
    drawn on the device from a seeded generator, with the workload's
    distributions).  Sampled rows, copied out before and after the merge, are
    checked against the fp64 rule."""
    ra = cuda_lib
    T, H, D = 1048576, 32, 128
    g = torch.Generator(device="cuda").manual_seed(7)
    out = torch.randn((T, H, D), device="cuda", generator=g)
    lse = torch.rand((T, H), device="cuda", generator=g) * 20 - 5
    bo = torch.randn((T, H, D), device="cuda", generator=g)
    bl = torch.rand((T, H), device="cuda", generator=g) * 20 - 5
    bl[T - 1, :3] = float("-inf")  # empty partials at the last token
    rng = np.random.default_rng(8)
    ti = torch.from_numpy(np.unique(np.concatenate([rng.integers(0, T, 2048), [0, T - 1]])))
    before = [x[ti.cuda()].double().cpu().numpy() for x in (out, lse, bo, bl)]
    ra.ra_merge_partial(out, lse, bo, bl)
    torch.cuda.synchronize()
    ref_o, ref_l = K.merge_rule(*before)
    check_merge(out[ti.cuda()], lse[ti.cuda()], ref_o, ref_l)
    assert ra.ra_get_device_status() == 0


@pytest.mark.parametrize("T,k", [(1048576, 4), (131072, 16)])
def test_merge_partials_large_sampled_rows(cuda_lib, T, k):
    """The k-way merge at the sweep's sizes (16 partials of 1M tokens would
    need 256 GiB, so k = 16 runs at 131,072 tokens): partials drawn on the
    device from a seeded generator, sampled rows against the fp64 k-way rule."""
    ra = cuda_lib
    H, D = 32, 128
    g = torch.Generator(device="cuda").manual_seed(9 + k)
    outs = [torch.randn((T, H, D), device="cuda", generator=g) for _ in range(k)]
    lses = [torch.rand((T, H), device="cuda", generator=g) * 20 - 5 for _ in range(k)]
    rng = np.random.default_rng(k)
    ti = torch.from_numpy(np.unique(np.concatenate([rng.integers(0, T, 1024), [0, T - 1]]))).cuda()
    ref_o, ref_l = K.merge_partials([o[ti].double().cpu().numpy() for o in outs],
                                    [l[ti].double().cpu().numpy() for l in lses])
    go, gl = ra.ra_merge_partials(outs, lses)
    torch.cuda.synchronize()
    check_merge(go[ti], gl[ti], ref_o, ref_l)
    assert ra.ra_get_device_status() == 0


@pytest.mark.parametrize("k", [2, 4, 8, 16])
def test_merge_partials_matches_oracle(cuda_lib, k):
    ra = cuda_lib
    outs, lses = merge_inputs(4096, k, seed=k)
    ref_o, ref_l = K.merge_partials([o.double().numpy() for o in outs], [l.double().numpy() for l in lses])
    go, gl = ra.ra_merge_partials([o.cuda() for o in outs], [l.cuda() for l in lses])
    check_merge(go, gl, ref_o, ref_l)
    # pairwise launches, folded left to right, give the same answer
    o, l = outs[0].cuda(), lses[0].cuda()
    for j in range(1, k):
        ra.ra_merge_partial(o, l, outs[j].cuda(), lses[j].cuda())
    check_merge(o, l, ref_o, ref_l)


# ----------------------------------------------------------- block attention

BLOCK_CASES = [
    # B, S, n, Hq, Hkv, D, causal, partition
    (2, 1200, 4, 4, 2, 128, True, "zigzag"),       # L=300: ragged tail, chunk (150) straddles a tile
    (1, 1024, 4, 2, 2, 64, True, "contiguous"),
    (1, 768, 2, 2, 1, 128, False, "contiguous"),
]


@pytest.mark.parametrize("case", BLOCK_CASES, ids=lambda c: f"B{c[0]}S{c[1]}n{c[2]}H{c[3]}/{c[4]}D{c[5]}{c[7]}{'C' if c[6] else ''}")
def test_block_attn_every_pair(cuda_lib, case):
    ra = cuda_lib
    B, S, n, Hq, Hkv, D, causal, part = case
    q, k, v = attention_inputs(B, S, Hq, Hkv, D, "bf16", seed=3)
    perm = K.partition_perm(S, n, part)
    L = S // n
    pos = perm.reshape(n, L)
    pt = torch.from_numpy(perm)
    qp, kp, vp = q[:, pt], k[:, pt], v[:, pt]
    for qb in range(n):
        qblk = qp[:, qb * L:(qb + 1) * L].contiguous()
        for kb in range(n):
            kblk = kp[:, kb * L:(kb + 1) * L].contiguous()
            vblk = vp[:, kb * L:(kb + 1) * L].contiguous()
            bo, bl = ra.ra_block_attn(qblk.cuda(), kblk.cuda(), vblk.cuda(), S, n, qb, kb, causal, part)
            ro, rl = K.block_partial(qblk, kblk, vblk, pos[qb], pos[kb], causal, Hq // Hkv)
            assert_close_bf16(to_np(bo), ro, f"block_out q{qb} kv{kb}")
            assert_close_bf16(to_np(bl), rl, f"block_lse q{qb} kv{kb}")


# ----------------------------------------------------------- whole method

SCHEDS = ["persistent", "fused", "unfused"]


@pytest.mark.parametrize("tiling", ["row_pairs", "kv_split", "cluster2"])
@pytest.mark.parametrize("order", ["ring", "tokenring"])
@pytest.mark.parametrize("sched", SCHEDS)
@pytest.mark.parametrize("case", [(2, 1200, 4, 4, 2, 128, True, "zigzag"), (1, 1024, 4, 2, 1, 64, True, "contiguous"),
                                  (1, 640, 5, 2, 2, 128, False, "zigzag"), (1, 2304, 2, 2, 2, 128, True, "contiguous")],
                         ids=lambda c: f"B{c[0]}S{c[1]}n{c[2]}D{c[5]}{c[7]}{'C' if c[6] else ''}")
def test_ring_attention_matches_full_oracle(cuda_lib, case, sched, order, tiling):
    ra = cuda_lib
    B, S, n, Hq, Hkv, D, causal, part = case
    q, k, v = attention_inputs(B, S, Hq, Hkv, D, "bf16", seed=4)
    ro, rl = F.full_attention(q, k, v, causal, Hq // Hkv)
    for out_dtype in (torch.float32, torch.bfloat16):
        o, l = ra.ra_ring_attention(q.cuda(), k.cuda(), v.cuda(), n, causal, part, out_dtype=out_dtype,
                                    order=order, sched=sched, tiling=tiling)
        assert_close_bf16(to_np(o), ro, f"out {sched}/{order}/{tiling}/{out_dtype}")
        assert_close_bf16(to_np(l), rl, f"lse {sched}/{order}/{tiling}/{out_dtype}")
    assert ra.ra_get_device_status() == 0


EDGE_CASES = [
    # B, S, Hq, Hkv, D, n, causal, partition
    (1, 256, 2, 2, 128, 1, True, "contiguous"),     # one block: plain attention
    (1, 256, 2, 2, 128, 1, True, "zigzag"),         # one block, two chunks
    (1, 512, 2, 1, 128, 16, True, "zigzag"),        # 16 blocks, chunks of 16 rows
    (1, 32, 1, 1, 128, 16, True, "zigzag"),         # chunks of a single row
    (3, 384, 6, 2, 64, 3, True, "zigzag"),          # batch 3, GQA 3, D=64, c=64
    (2, 640, 4, 4, 128, 5, False, "contiguous"),    # non-causal, L=128
    (1, 2000, 4, 1, 128, 4, True, "zigzag"),        # c=250: tiles straddle nothing, ragged tails
    (1, 1000, 2, 2, 64, 2, False, "zigzag"),        # non-causal zigzag
]


@pytest.mark.parametrize("sched", SCHEDS)
@pytest.mark.parametrize("case", EDGE_CASES, ids=lambda c: f"B{c[0]}S{c[1]}H{c[2]}/{c[3]}D{c[4]}n{c[5]}{c[7]}{'C' if c[6] else ''}")
def test_ring_attention_edge_cases(cuda_lib, case, sched):
    ra = cuda_lib
    B, S, Hq, Hkv, D, n, causal, part = case
    q, k, v = attention_inputs(B, S, Hq, Hkv, D, "bf16", seed=6)
    ro, rl = F.full_attention(q, k, v, causal, Hq // Hkv)
    for tiling in ("auto", "row_pairs", "kv_split", "cluster2"):
        o, l = ra.ra_ring_attention(q.cuda(), k.cuda(), v.cuda(), n, causal, part, out_dtype=torch.float32,
                                    sched=sched, tiling=tiling)
        assert_close_bf16(to_np(o), ro, f"out {sched}/{tiling}")
        assert_close_bf16(to_np(l), rl, f"lse {sched}/{tiling}")
    assert ra.ra_get_device_status() == 0


def test_block_attn_empty_and_full_pairs(cuda_lib):
    # causal zigzag, n=4: pairs whose KV block lies wholly after (every row
    # empty: lse = -inf, out = 0) or wholly before (no masking) the query block
    ra = cuda_lib
    B, S, n, Hq, Hkv, D = 1, 2048, 4, 2, 2, 128
    q, k, v = attention_inputs(B, S, Hq, Hkv, D, "bf16", seed=8)
    perm = K.zigzag_perm(S, n)
    L = S // n
    pos = perm.reshape(n, L)
    pt = torch.from_numpy(perm)
    qp, kp, vp = q[:, pt], k[:, pt], v[:, pt]
    seen_empty = seen_full = False
    for qb in range(n):
        for kb in range(n):
            qblk = qp[:, qb * L:(qb + 1) * L].contiguous()
            kblk = kp[:, kb * L:(kb + 1) * L].contiguous()
            vblk = vp[:, kb * L:(kb + 1) * L].contiguous()
            bo, bl = ra.ra_block_attn(qblk.cuda(), kblk.cuda(), vblk.cuda(), S, n, qb, kb, True, "zigzag")
            ro, rl = K.block_partial(qblk, kblk, vblk, pos[qb], pos[kb], True, 1)
            empty_rows = np.isneginf(rl)
            seen_empty |= bool(empty_rows.any())
            seen_full |= bool((~empty_rows).all())
            assert np.all(to_np(bo)[empty_rows] == 0.0)
            assert_close_bf16(to_np(bo), ro, f"block_out q{qb} kv{kb}")
            assert_close_bf16(to_np(bl), rl, f"block_lse q{qb} kv{kb}")
    assert seen_empty and seen_full


@pytest.mark.parametrize("case", BLOCK_CASES, ids=lambda c: f"B{c[0]}S{c[1]}n{c[2]}H{c[3]}/{c[4]}D{c[5]}{c[7]}{'C' if c[6] else ''}")
def test_block_attn_merge_folds_every_pair(cuda_lib, case):
    # every query block folds its n pairs, in a shuffled order, into (0, -inf)
    # with the fused entry point; the blocks gathered back to original order
    # are the full attention
    ra = cuda_lib
    B, S, n, Hq, Hkv, D, causal, part = case
    q, k, v = attention_inputs(B, S, Hq, Hkv, D, "bf16", seed=9)
    perm = K.partition_perm(S, n, part)
    L = S // n
    pt = torch.from_numpy(perm)
    qp, kp, vp = q[:, pt].cuda(), k[:, pt].cuda(), v[:, pt].cuda()
    out = torch.zeros((B, S, Hq, D), dtype=torch.float32, device="cuda")
    lse = torch.full((B, S, Hq), float("-inf"), dtype=torch.float32, device="cuda")
    rng = np.random.default_rng(1)
    for qb in range(n):
        rows = slice(qb * L, (qb + 1) * L)
        o, l = out[:, rows].contiguous(), lse[:, rows].contiguous()
        for kb in rng.permutation(n):
            before = (o.clone(), l.clone())
            kv = slice(int(kb) * L, (int(kb) + 1) * L)
            ra.ra_block_attn_merge(qp[:, rows].contiguous(), kp[:, kv].contiguous(), vp[:, kv].contiguous(), S, n,
                                   qb, int(kb), causal, o, l, partition=part)
            if K.pair_is_empty(perm.reshape(n, L)[qb], perm.reshape(n, L)[kb], causal):
                # a pair that sees no key leaves the running state untouched, bit for bit
                assert torch.equal(o, before[0]) and torch.equal(l, before[1])
        out[:, rows], lse[:, rows] = o, l
    ro, rl = F.full_attention(q, k, v, causal, Hq // Hkv)
    assert_close_bf16(K.permute_rows(to_np(out), perm, inverse=True), ro, "folded out")
    assert_close_bf16(K.permute_rows(to_np(lse), perm, inverse=True), rl, "folded lse")
    assert ra.ra_get_device_status() == 0


@pytest.mark.parametrize("order", ["ring", "tokenring"])
@pytest.mark.parametrize("case", [(1, 2048, 4, 4, 2, 128, True, "zigzag"), (1, 1024, 4, 2, 1, 64, True, "contiguous"),
                                  (2, 1200, 3, 2, 2, 128, False, "zigzag")],
                         ids=lambda c: f"B{c[0]}S{c[1]}n{c[2]}D{c[5]}{c[7]}{'C' if c[6] else ''}")
def test_ring_shards_lockstep_on_cuda(cuda_lib, case, order):
    # the sequence-parallel rank programs (one block per rank, K/V or Q and
    # partials exchanged between ranks) with every rank's device work on the
    # CUDA kernels, all ranks in one process; gathered, the full attention
    from blockwise_exact_attention_block_b200 import ring
    ra = cuda_lib
    B, S, n, Hq, Hkv, D, causal, part = case
    q, k, v = attention_inputs(B, S, Hq, Hkv, D, "bf16", seed=10)

    def shard(x, r):
        return torch.cat([x[:, p:p + l] for p, l in ring.block_segments(S, n, part, r)], dim=1).contiguous().cuda()

    res = ring.ring_attention_lockstep([shard(q, r) for r in range(n)], [shard(k, r) for r in range(n)],
                                       [shard(v, r) for r in range(n)], S, causal, part, order)
    out = np.empty((B, S, Hq, D))
    lse = np.empty((B, S, Hq))
    for r, (o, l) in enumerate(res):
        row = 0
        for p, ln in ring.block_segments(S, n, part, r):
            out[:, p:p + ln] = to_np(o)[:, row:row + ln]
            lse[:, p:p + ln] = to_np(l)[:, row:row + ln]
            row += ln
    ro, rl = F.full_attention(q, k, v, causal, Hq // Hkv)
    assert_close_bf16(out, ro, f"ring shards out {order}")
    assert_close_bf16(lse, rl, f"ring shards lse {order}")
    assert ra.ra_get_device_status() == 0


def test_tiny_workload(cuda_lib):
    # fp32 inputs: the library rounds them to bf16 on entry; the attention is
    # judged against the oracle on the same rounded values.
    ra = cuda_lib
    w = WORKLOADS["tiny"]
    q, k, v = workload_inputs(w)
    qr, kr, vr = (x.to(torch.bfloat16) for x in (q, k, v))
    ro, rl = F.full_attention(qr, kr, vr, w.causal, w.gqa_groups)
    for sched in SCHEDS:
        o, l = ra.ra_ring_attention(q.cuda(), k.cuda(), v.cuda(), w.n_blocks, w.causal, w.partition, sched=sched)
        assert_close_bf16(to_np(o), ro, f"tiny out {sched}")
        assert_close_bf16(to_np(l), rl, f"tiny lse {sched}")


@pytest.fixture(scope="module")
def zigzag4k():
    w = WORKLOADS["zigzag4k"]
    q, k, v = workload_inputs(w)
    ro, rl = F.full_attention(q, k, v, w.causal, w.gqa_groups)
    return w, (q, k, v), (ro, rl)


@pytest.mark.parametrize("tiling", ["auto", "row_pairs", "kv_split", "cluster2"])
@pytest.mark.parametrize("sched", SCHEDS)
@pytest.mark.parametrize("order", ["ring", "tokenring"])
def test_zigzag4k_workload_full_oracle(cuda_lib, zigzag4k, sched, order, tiling):
    ra = cuda_lib
    w, (q, k, v), (ro, rl) = zigzag4k
    o, l = ra.ra_ring_attention(q.cuda(), k.cuda(), v.cuda(), w.n_blocks, w.causal, w.partition, sched=sched,
                                order=order, tiling=tiling)
    assert_close_bf16(to_np(o), ro, "zigzag4k out")
    assert_close_bf16(to_np(l), rl, "zigzag4k lse")


def sample_rows(w, per_head=64, seed=0):
    """Seeded random rows plus the first / last row of every zigzag chunk and
    rows on 128-row tile boundaries of the blocks."""
    rng = np.random.default_rng(seed)
    perm = K.partition_perm(w.S, w.n_blocks, w.partition)
    L = w.S // w.n_blocks
    special = set()
    c = w.S // (2 * w.n_blocks)
    for ch in range(2 * w.n_blocks):
        special.update([ch * c, ch * c + c - 1])
    for r in rng.choice(w.n_blocks, size=min(4, w.n_blocks), replace=False):
        for t in rng.choice(np.arange(128, L, 128), size=min(4, (L - 1) // 128), replace=False):
            special.update([int(perm[r * L + t]), int(perm[r * L + t - 1])])
    special.update([0, w.S - 1])
    rows = []
    for b in range(w.B):
        for h in range(w.Hq):
            pick = set(int(x) for x in rng.integers(0, w.S, per_head)) | special
            rows.extend((b, i, h) for i in sorted(pick))
    return rows


def check_sampled(w, q, k, v, o, l, rows, what):
    ro, rl = F.attention_rows(q, k, v, rows, w.causal, w.gqa_groups)
    bi = torch.tensor([r[0] for r in rows])
    ii = torch.tensor([r[1] for r in rows])
    hi = torch.tensor([r[2] for r in rows])
    go = o.float().cpu()[bi, ii, hi].numpy()
    gl = l.cpu()[bi, ii, hi].numpy()
    assert_close_bf16(go, ro, what + " out")
    assert_close_bf16(gl, rl, what + " lse")


@pytest.mark.parametrize("sched", SCHEDS)
def test_gqa24k_workload_sampled_rows(cuda_lib, sched):
    ra = cuda_lib
    w = WORKLOADS["gqa24k"]
    q, k, v = workload_inputs(w)
    o, l = ra.ra_ring_attention(q.cuda(), k.cuda(), v.cuda(), w.n_blocks, w.causal, w.partition,
                                out_dtype=torch.float32, sched=sched)
    rows = sample_rows(w, per_head=16 if sched != "persistent" else 64)
    check_sampled(w, q, k, v, o, l, rows, f"gqa24k {sched}")
    assert ra.ra_get_device_status() == 0


def whole_tile_rows(w, seed=0):
    """Every row of whole 128-row query tiles, per head: the ragged last tile
    of chunk h mod 2n and one seeded interior tile of chunk (h + 3) mod 2n.
    Query tiles start at their chunk's first token (zigzag chunks of c tokens,
    tiles never straddle one), so these are exactly the rows one CTA's tile
    writes; across the heads every chunk's tail and many interior tiles are
    covered."""
    rng = np.random.default_rng(seed)
    nch = 2 * w.n_blocks
    c = w.S // nch
    ntiles = (c + 127) // 128
    rows = []
    for b in range(w.B):
        for h in range(w.Hq):
            tail = (h % nch) * c + (ntiles - 1) * 128
            rows.extend((b, i, h) for i in range(tail, (h % nch) * c + c))
            t = int(rng.integers(0, ntiles - 1))
            first = ((h + 3) % nch) * c + 128 * t
            rows.extend((b, i, h) for i in range(first, first + 128))
    return rows


def test_gqa24k_whole_tiles(cuda_lib):
    # Sampled rows could miss a fault confined to one tile of one head; here
    # every row of two whole tiles per head (32 heads, 5,888 rows) is checked
    # against the fp64 oracle, the ragged 56-row chunk tails included.
    ra = cuda_lib
    w = WORKLOADS["gqa24k"]
    q, k, v = workload_inputs(w)
    o, l = ra.ra_ring_attention(q.cuda(), k.cuda(), v.cuda(), w.n_blocks, w.causal, w.partition,
                                out_dtype=torch.float32)
    rows = whole_tile_rows(w)
    assert len(rows) == w.Hq * ((w.S // 8) % 128 + 128)
    check_sampled(w, q, k, v, o, l, rows, "gqa24k whole tiles")
    assert ra.ra_get_device_status() == 0


def test_long1m_workload_sampled_rows(cuda_lib):
    ra = cuda_lib
    w = WORKLOADS["long1m"]
    q, k, v = workload_inputs(w)
    o, l = ra.ra_ring_attention(q.cuda(), k.cuda(), v.cuda(), w.n_blocks, w.causal, w.partition,
                                out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    rows = sample_rows(w, per_head=24)
    check_sampled(w, q, k, v, o, l, rows, "long1m")
    assert ra.ra_get_device_status() == 0


# ------------------------------------------------------------------ decode

DECODE_CASES = [
    # B, Tq, Skv, Hq, Hkv, D, causal, n_splits
    (2, 1, 1000, 8, 2, 128, True, 0),       # ragged cache (not a multiple of 64), GQA 4
    (1, 3, 777, 4, 4, 64, True, 5),         # MHA, D=64, three causal tokens, explicit chunks
    (1, 16, 2048, 16, 4, 128, True, 3),     # 4 heads x 16 tokens = 64 rows per KV head (the limit)
    (3, 2, 130, 6, 2, 128, False, 1),       # non-causal, one chunk, ragged last tile
    (1, 1, 64, 2, 1, 128, True, 0),         # exactly one tile
    (1, 4, 4, 4, 2, 128, True, 0),          # Tq == Skv: the first token sees key 0 only
    (2, 2, 5000, 8, 8, 64, True, 40),       # many chunks
]


@pytest.mark.parametrize("case", DECODE_CASES,
                         ids=lambda c: f"B{c[0]}Tq{c[1]}S{c[2]}H{c[3]}/{c[4]}D{c[5]}{'C' if c[6] else ''}n{c[7]}")
def test_decode_matches_oracle(cuda_lib, case):
    ra = cuda_lib
    B, Tq, Skv, Hq, Hkv, D, causal, n = case
    q, k, v = decode_inputs(B, Tq, Skv, Hq, Hkv, D, seed=11)
    ro, rl = F.decode_attention(q, k, v, causal, Hq // Hkv)
    for out_dtype in (torch.float32, torch.bfloat16):
        o, l = ra.ra_decode_attention(q.cuda(), k.cuda(), v.cuda(), causal, n, out_dtype=out_dtype)
        assert_close_bf16(to_np(o), ro, f"decode out {out_dtype}")
        assert_close_bf16(to_np(l), rl, f"decode lse {out_dtype}")
    assert ra.ra_get_device_status() == 0


def test_decode_chunk_count_invariance(cuda_lib):
    # the chunks are stitched by the merge rule: any chunk count gives the
    # same attention (to rounding), and matches the oracle's own chunked form
    ra = cuda_lib
    B, Tq, Skv, Hq, Hkv, D = 1, 2, 3000, 8, 2, 128
    q, k, v = decode_inputs(B, Tq, Skv, Hq, Hkv, D, seed=12)
    ro, rl = K.decode_blockwise(q, k, v, True, Hq // Hkv, 7)
    base = None
    for n in (1, 2, 7, 23, 0):
        o, l = ra.ra_decode_attention(q.cuda(), k.cuda(), v.cuda(), True, n)
        assert_close_bf16(to_np(o), ro, f"decode out n={n}")
        assert_close_bf16(to_np(l), rl, f"decode lse n={n}")
        if base is None:
            base = (o.clone(), l.clone())
        assert float((o - base[0]).abs().max()) <= 2e-3
        assert float((l - base[1]).abs().max()) <= 2e-3


@pytest.mark.parametrize("name", sorted(DECODE_WORKLOADS))
def test_decode_workloads_full_oracle(cuda_lib, name):
    ra = cuda_lib
    w = DECODE_WORKLOADS[name]
    q, k, v = decode_inputs(w.B, w.Tq, w.Skv, w.Hq, w.Hkv, w.D)
    o, l = ra.ra_decode_attention(q.cuda(), k.cuda(), v.cuda(), w.causal, 0)
    ro, rl = F.decode_attention(q, k, v, w.causal, w.gqa_groups)
    assert_close_bf16(to_np(o), ro, f"{name} out")
    assert_close_bf16(to_np(l), rl, f"{name} lse")
    assert ra.ra_get_device_status() == 0
