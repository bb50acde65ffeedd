"""GPU parity of the backward (ra_ring_attention_backward, through the C ABI)
against the fp64 oracle on the same seeded inputs.

Tolerance (derived from the arithmetic): the kernels round P and dS to bf16
(relative error <= 2^-9 each) before the dV / dQ / dK products and accumulate
in fp32; the oracle gets the bf16 inputs the kernels read.  Gradients grow
with the score spread (|dS| ~ P |dO| |V|), so the bar is relative to the
result's scale: max-abs error <= 2e-2 * max(1, max |ref|) and relative L2
error <= 1e-2, on dq, dk and dv separately.

Full-size workloads are checked on sampled query rows (dq) and sampled late
keys (dk, dv: a key near the end is seen by few queries, each recomputed over
its whole row), and on identities that hold at any size:
    sum_j dV_j = sum_i dO_i          (softmax rows sum to one)
    sum_j dK_j = 0                   (every dS row sums to zero)
    sum_i dQ_i . Q_i = sum_j dK_j . K_j   (both are the derivative of the
                                           loss along a scaling of the scores)
    sum_j dV_j . V_j = sum_i dO_i . O_i
per batch and KV head (query sums run over the heads of the group).
"""
import numpy as np
import pytest
import torch

from oracle import attention as F
from oracle import backward as G
from seeded_inputs import WORKLOADS, backward_inputs

pytestmark = pytest.mark.gpu

ATOL_REL, RTOL_L2 = 2e-2, 1e-2


def assert_grad_close(got, ref, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    err = np.abs(got - ref)
    bar = ATOL_REL * max(1.0, float(np.abs(ref).max()))
    mx = float(err.max())
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert mx <= bar, f"{what}: max-abs {mx:.3e} > {bar:.3e}"
    assert rel <= RTOL_L2, f"{what}: rel-L2 {rel:.3e} > {RTOL_L2}"


def to_np(t):
    return t.detach().double().cpu().numpy()


def run(ra, q, k, v, do, n, causal, part, out_dtype, order="ring"):
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, l = ra.ra_ring_attention(qd, kd, vd, n, causal, part, out_dtype=out_dtype, order=order)
    dq, dk, dv = ra.ra_ring_attention_backward(qd, kd, vd, o, l, dod, n, causal, part, order=order)
    torch.cuda.synchronize()
    return o, l, dq, dk, dv


CASES = [
    # B, S, Hq, Hkv, D, n, causal, partition, in dtype, out dtype, order
    (1, 256, 2, 2, 64, 2, True, "contiguous", "bf16", torch.float32, "ring"),
    (2, 384, 4, 2, 128, 2, True, "zigzag", "bf16", torch.float32, "ring"),          # 96-row chunks: ragged tiles
    (1, 600, 2, 1, 64, 3, False, "contiguous", "bf16", torch.bfloat16, "tokenring"),  # 200-row blocks
    (1, 512, 4, 1, 128, 4, True, "zigzag", "f32", torch.bfloat16, "tokenring"),     # fp32 inputs, 4 groups
    (1, 1000, 3, 3, 64, 1, True, "contiguous", "bf16", torch.float32, "ring"),      # one block
    (1, 1200, 4, 2, 128, 4, True, "zigzag", "bf16", torch.float32, "ring"),         # 150-row chunks
    (1, 512, 2, 1, 128, 16, True, "zigzag", "bf16", torch.float32, "tokenring"),    # 16 blocks, 16-row chunks
    (1, 640, 2, 2, 128, 5, False, "zigzag", "bf16", torch.float32, "ring"),         # non-causal zigzag
    (1, 32, 2, 1, 64, 16, True, "zigzag", "bf16", torch.float32, "ring"),           # 1-row chunks
    (2, 200, 2, 2, 128, 1, True, "contiguous", "bf16", torch.bfloat16, "ring"),     # one ragged 200-row block
    (1, 96, 4, 4, 64, 3, False, "contiguous", "f32", torch.float32, "tokenring"),   # 32-row blocks, fp32
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}S{c[1]}H{c[2]}/{c[3]}D{c[4]}n{c[5]}{c[7]}"
                                                      f"{'C' if c[6] else ''}{c[8]}{c[10]}")
def test_backward_matches_oracle(cuda_lib, case):
    ra = cuda_lib
    B, S, Hq, Hkv, D, n, causal, part, idt, odt, order = case
    q, k, v, do = backward_inputs(B, S, Hq, Hkv, D, idt, seed=5)
    _, _, dq, dk, dv = run(ra, q, k, v, do, n, causal, part, odt, order)
    # the kernels read bf16: the oracle gets the same values
    qb, kb, vb, dob = (x.to(torch.bfloat16) for x in (q, k, v, do))
    rq, rk, rv = G.attention_backward(qb, kb, vb, dob, causal, Hq // Hkv)
    assert_grad_close(to_np(dq), rq, "dq")
    assert_grad_close(to_np(dk), rk, "dk")
    assert_grad_close(to_np(dv), rv, "dv")
    assert ra.ra_get_device_status() == 0


def test_backward_from_oracle_forward(cuda_lib):
    """The backward alone: out and lse from the oracle, the expected gradient
    from the oracle's block-pair sums over the same out and lse."""
    ra = cuda_lib
    B, S, Hq, Hkv, D, n = 1, 768, 4, 2, 128, 3
    q, k, v, do = backward_inputs(B, S, Hq, Hkv, D, "bf16", seed=6)
    ro, rl = F.full_attention(q, k, v, True, 2)
    o = torch.from_numpy(ro).float().cuda()
    l = torch.from_numpy(rl).float().cuda()
    dq, dk, dv = ra.ra_ring_attention_backward(q.cuda(), k.cuda(), v.cuda(), o, l, do.cuda(), n, True, "contiguous")
    rq, rk, rv = G.blockwise_backward(q, k, v, do, ro, rl, n, True, "contiguous", 2)
    assert_grad_close(to_np(dq), rq, "dq")
    assert_grad_close(to_np(dk), rk, "dk")
    assert_grad_close(to_np(dv), rv, "dv")


def test_backward_order_invariance(cuda_lib):
    """Ring and TokenRing orders sum the same block pairs: the results agree
    to fp32 accumulation rounding."""
    ra = cuda_lib
    B, S, Hq, Hkv, D, n = 1, 1024, 4, 2, 128, 4
    q, k, v, do = backward_inputs(B, S, Hq, Hkv, D, "bf16", seed=7)
    a = run(ra, q, k, v, do, n, True, "zigzag", torch.float32, "ring")[2:]
    b = run(ra, q, k, v, do, n, True, "zigzag", torch.float32, "tokenring")[2:]
    for x, y in zip(a, b):
        scale = float(y.abs().max())
        assert float((x - y).abs().max()) <= 1e-3 * max(1.0, scale)


def test_backward_deterministic(cuda_lib):
    """Every output row has one writer: two calls give identical bits."""
    ra = cuda_lib
    q, k, v, do = backward_inputs(1, 1024, 4, 1, 128, "bf16", seed=8)
    a = run(ra, q, k, v, do, 4, True, "zigzag", torch.float32)[2:]
    b = run(ra, q, k, v, do, 4, True, "zigzag", torch.float32)[2:]
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_backward_zero_upstream_gradient(cuda_lib):
    ra = cuda_lib
    q, k, v, do = backward_inputs(1, 512, 2, 2, 128, "bf16", seed=9)
    do.zero_()
    for g in run(ra, q, k, v, do, 2, True, "zigzag", torch.float32)[2:]:
        assert int(torch.count_nonzero(g)) == 0


def test_backward_accumulator_drains(cuda_lib):
    """Long walks drain the tensor-core accumulators into the fp32 outputs
    every 256 tiles.  Here the first key tile meets 64 query tiles of each of
    8 query heads (512 tiles: one drain in the dK/dV kernel), checked against
    the whole oracle gradient."""
    ra = cuda_lib
    B, S, Hq, Hkv, D, n = 1, 8192, 8, 1, 128, 2
    q, k, v, do = backward_inputs(B, S, Hq, Hkv, D, "bf16", seed=11)
    _, _, dq, dk, dv = run(ra, q, k, v, do, n, True, "zigzag", torch.float32)
    rq, rk, rv = G.attention_backward(q, k, v, do, True, Hq // Hkv)
    assert_grad_close(to_np(dq), rq, "dq")
    assert_grad_close(to_np(dk), rk, "dk")
    assert_grad_close(to_np(dv), rv, "dv")
    assert ra.ra_get_device_status() == 0


def test_backward_accumulator_drains_dq(cuda_lib):
    """dQ drains: the last query tile of a 40,960-token sequence walks 320 KV
    tiles (one drain); its rows against the oracle, row by row."""
    ra = cuda_lib
    B, S, Hq, Hkv, D, n = 1, 40960, 2, 1, 128, 4
    q, k, v, do = backward_inputs(B, S, Hq, Hkv, D, "bf16", seed=12)
    o, l, dq, dk, dv = run(ra, q, k, v, do, n, True, "contiguous", torch.float32)
    rows = [(0, i, h) for h in range(Hq) for i in (S - 1, S - 60, S - 128, S - 129, 33000, 100)]
    ref = G.backward_query_rows(q, k, v, do, rows, True, Hq // Hkv)
    bi, ii, hi = (torch.tensor([r[t] for r in rows]) for t in range(3))
    assert_grad_close(to_np(dq.cpu()[bi, ii, hi]), ref, "dq rows")
    check_identities(q, k, v, do, o, dq, dk, dv, Hq // Hkv, "S=40960")
    assert ra.ra_get_device_status() == 0


# ------------------------------------------------------ full-size workloads

def check_identities(q, k, v, do, o, dq, dk, dv, groups, what):
    B, S, Hq, D = q.shape
    Hkv = Hq // groups
    f = lambda t: t.cuda().double()  # noqa: E731
    q, k, v, do, o, dq, dk, dv = map(f, (q, k, v, do, o, dq, dk, dv))
    dog = do.view(B, S, Hkv, groups, D)
    # sum_j dV_j = sum_i dO_i
    lhs, rhs = dv.sum(1), dog.sum((1, 3))
    scale = dog.pow(2).sum((1, 3)).sqrt()
    assert bool(((lhs - rhs).abs() <= 1e-2 * scale.clamp_min(1.0)).all()), f"{what}: sum dV != sum dO"
    # sum_j dK_j = 0
    colsum, colnorm = dk.sum(1), dk.pow(2).sum(1).sqrt()
    assert bool((colsum.abs() <= 2e-2 * colnorm.clamp_min(1e-6)).all()), f"{what}: sum dK != 0"
    # sum_i dQ_i . Q_i = sum_j dK_j . K_j
    qq = (dq * q).sum(-1).view(B, S, Hkv, groups)
    kk = (dk * k).sum(-1)
    lhs, rhs = qq.sum((1, 3)), kk.sum(1)
    l1 = qq.abs().sum((1, 3)) + kk.abs().sum(1)
    assert bool(((lhs - rhs).abs() <= 1e-3 * l1).all()), f"{what}: dQ.Q != dK.K"
    # sum_j dV_j . V_j = sum_i dO_i . O_i
    vv = (dv * v).sum((1, 3))
    oo = (do * o).sum(-1).view(B, S, Hkv, groups)
    assert bool(((vv - oo.sum((1, 3))).abs() <= 1e-2 * oo.pow(2).sum((1, 3)).sqrt()).all()), \
        f"{what}: dV.V != dO.O"


def sampled_query_rows(w, per_head, seed):
    rng = np.random.default_rng(seed)
    c = w.S // (2 * w.n_blocks) if w.partition == "zigzag" else w.S // w.n_blocks
    special = {0, 1, w.S - 1} | {x for ch in range(w.S // c) for x in (ch * c, ch * c + c - 1)}
    rows = []
    for b in range(w.B):
        for h in range(w.Hq):
            pick = set(int(x) for x in rng.integers(0, w.S, per_head)) | set(rng.choice(sorted(special), 4).tolist())
            rows.extend((b, i, h) for i in sorted(pick))
    return rows


def sampled_late_keys(w, per_head, seed, window=40):
    rng = np.random.default_rng(seed)
    keys = []
    for b in range(w.B):
        for g in range(w.Hkv):
            pick = {w.S - 1} | set(int(x) for x in rng.integers(w.S - window, w.S, per_head))
            keys.extend((b, j, g) for j in sorted(pick))
    return keys


@pytest.mark.parametrize("name", ["zigzag4k", "gqa24k"])
def test_backward_workload(cuda_lib, name):
    ra = cuda_lib
    w = WORKLOADS[name]
    q, k, v, do = backward_inputs(w.B, w.S, w.Hq, w.Hkv, w.D, w.in_dtype, seed=10)
    o, l, dq, dk, dv = run(ra, q, k, v, do, w.n_blocks, w.causal, w.partition, torch.float32)
    assert ra.ra_get_device_status() == 0
    check_identities(q, k, v, do, o, dq, dk, dv, w.gqa_groups, name)
    if name == "zigzag4k":  # small enough for the whole oracle
        rq, rk, rv = G.attention_backward(q, k, v, do, w.causal, w.gqa_groups)
        assert_grad_close(to_np(dq), rq, "dq")
        assert_grad_close(to_np(dk), rk, "dk")
        assert_grad_close(to_np(dv), rv, "dv")
        return
    rows = sampled_query_rows(w, per_head=12, seed=1)
    ref = G.backward_query_rows(q, k, v, do, rows, w.causal, w.gqa_groups)
    bi, ii, hi = (torch.tensor([r[t] for r in rows]) for t in range(3))
    assert_grad_close(to_np(dq.cpu()[bi, ii, hi]), ref, f"{name} dq rows")
    keys = sampled_late_keys(w, per_head=3, seed=2)
    rk, rv = G.backward_key_rows(q, k, v, do, keys, w.causal, w.gqa_groups)
    bi, ji, gi = (torch.tensor([r[t] for r in keys]) for t in range(3))
    assert_grad_close(to_np(dk.cpu()[bi, ji, gi]), rk, f"{name} dk late keys")
    assert_grad_close(to_np(dv.cpu()[bi, ji, gi]), rv, f"{name} dv late keys")


def test_backward_long1m_workload(cuda_lib):
    """1,048,576 tokens, 8 zigzag blocks, GQA 8/2, bf16 out: the identities
    over the whole gradient, sampled dq rows, and dk, dv of late keys (each
    from the full rows of the few queries that see it).  The oracle gets one
    query head (or one KV group) at a time, sliced out, so it holds ~1 GB."""
    ra = cuda_lib
    w = WORKLOADS["long1m"]
    q, k, v, do = backward_inputs(w.B, w.S, w.Hq, w.Hkv, w.D, w.in_dtype, seed=10)
    o, l, dq, dk, dv = run(ra, q, k, v, do, w.n_blocks, w.causal, w.partition, torch.bfloat16)
    assert ra.ra_get_device_status() == 0
    check_identities(q, k, v, do, o, dq, dk, dv, w.gqa_groups, "long1m")
    o = l = None
    dq, dk, dv = dq.cpu(), dk.cpu(), dv.cpu()
    torch.cuda.empty_cache()
    rng = np.random.default_rng(3)
    G_ = w.gqa_groups
    for h in (0, w.Hq - 1):  # one query head of each KV group
        g = h // G_
        rows = sorted({int(x) for x in rng.integers(0, w.S, 3)} | {w.S - 1})
        ref = G.backward_query_rows(q[:, :, h:h + 1], k[:, :, g:g + 1], v[:, :, g:g + 1], do[:, :, h:h + 1],
                                    [(0, i, 0) for i in rows], True, 1)
        assert_grad_close(to_np(dq[0, rows, h]), ref, f"long1m dq rows head {h}")
    for g in range(w.Hkv):
        keys = [w.S - 1 - 5 * g]
        sl = slice(g * G_, (g + 1) * G_)
        rk, rv = G.backward_key_rows(q[:, :, sl], k[:, :, g:g + 1], v[:, :, g:g + 1], do[:, :, sl],
                                     [(0, j, 0) for j in keys], True, G_)
        assert_grad_close(to_np(dk[0, keys, g]), rk, f"long1m dk late keys group {g}")
        assert_grad_close(to_np(dv[0, keys, g]), rv, f"long1m dv late keys group {g}")
