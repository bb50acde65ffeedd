"""The per-CTA timeline (ra_set_cta_timeline), a tracing aid, on the GPU.

Each record must be well formed (end after start, an SM id below the SM
count), there must be exactly one record per CTA of the launch, and the work
units the CTAs report must be, as a multiset, the tile counts of the work
decomposition computed here from the partition alone:
  forward / dQ: per query tile, the KV tiles its last row sees, summed over
                every KV segment the tile meets;
  dK/dV:        per key tile, the query tiles with a row that sees the tile's
                first key, times the GQA group size.
A launch with the timeline off must leave the records untouched, and the
results must not depend on it.
"""
import numpy as np
import pytest
import torch

from seeded_inputs import attention_inputs, backward_inputs

pytestmark = pytest.mark.gpu

BM = 128


def segments(S, n, part):
    """(pos, len) of every segment of every block, in block order."""
    if part == "zigzag":
        c = S // (2 * n)
        return [s for r in range(n) for s in ((r * c, c), ((2 * n - 1 - r) * c, c))]
    L = S // n
    return [(r * L, L) for r in range(n)]


def visible(last, kpos, klen, causal):
    if not causal:
        return klen
    return min(max(last - kpos + 1, 0), klen)


def query_tile_work(S, n, part, causal, rows):
    segs = segments(S, n, part)
    out = []
    for pos, length in segs:
        for t in range(-(-length // rows)):
            last = pos + min((t + 1) * rows, length) - 1
            out.append(sum(-(-visible(last, kp, kl, causal) // BM) for kp, kl in segs))
    return out


def key_tile_work(S, n, part, causal, groups):
    segs = segments(S, n, part)
    out = []
    for kpos, klen in segs:
        for kt in range(-(-klen // BM)):
            first_k = kpos + kt * BM
            cnt = 0
            for qpos, qlen in segs:
                for t in range(-(-qlen // BM)):
                    q0, qr = qpos + t * BM, min(qlen - t * BM, BM)
                    if not causal or q0 + qr - 1 >= first_k:
                        cnt += 1
            out.append(cnt * groups)
    return out


def check_records(rec, expected_work, what):
    n_cta = len(expected_work)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    r = rec.cpu().numpy()
    used = r[:n_cta]
    assert (r[n_cta:] == 0).all(), f"{what}: records past the grid were written"
    assert (used[:, 0] > 0).all() and (used[:, 1] >= used[:, 0]).all(), f"{what}: start/end"
    sm, work = used[:, 2] & 0xFFFFFFFF, used[:, 2] >> 32
    assert (sm < sms).all(), f"{what}: SM ids"
    assert sorted(work.tolist()) == sorted(expected_work), f"{what}: work units"
    # every CTA of one launch runs within one span of well under a second
    assert used[:, 1].max() - used[:, 0].min() < 10**9, f"{what}: span"
    # cycles over ns: the clock the CTAs ran at, between 0.3 and 2.5 GHz
    ns = (used[:, 1] - used[:, 0]).sum()
    ghz = used[:, 3].sum() / max(ns, 1)
    assert 0.3 < ghz < 2.5, f"{what}: {ghz:.2f} GHz from the cycle counts"


@pytest.mark.parametrize("tiling,rows", [("kv_split", 128), ("row_pairs", 256)])
@pytest.mark.parametrize("S,n,part,causal", [(1200, 4, "zigzag", True), (1024, 2, "contiguous", False)])
def test_forward_timeline(cuda_lib, tiling, rows, S, n, part, causal):
    ra = cuda_lib
    B, Hq, Hkv, D = 1, 4, 2, 128
    q, k, v = (x.cuda() for x in attention_inputs(B, S, Hq, Hkv, D, "bf16", seed=21))
    ref_o, ref_l = ra.ra_ring_attention(q, k, v, n, causal, part, out_dtype=torch.float32, tiling=tiling)
    rec = torch.zeros((4096, 4), dtype=torch.int64, device="cuda")
    ra.ra_set_cta_timeline(rec, "attn_fwd")
    try:
        o, l = ra.ra_ring_attention(q, k, v, n, causal, part, out_dtype=torch.float32, tiling=tiling)
        torch.cuda.synchronize()
    finally:
        ra.ra_set_cta_timeline(None)
    assert torch.equal(o, ref_o) and torch.equal(l, ref_l), "the timeline changed the results"
    expected = query_tile_work(S, n, part, causal, rows) * (B * Hq)
    check_records(rec, expected, f"forward {tiling} S={S}")
    # off again: a further launch leaves the records alone
    rec.fill_(-1)
    ra.ra_ring_attention(q, k, v, n, causal, part, out_dtype=torch.float32, tiling=tiling)
    torch.cuda.synchronize()
    assert (rec == -1).all()
    assert ra.ra_get_device_status() == 0


def test_backward_timelines(cuda_lib):
    ra = cuda_lib
    B, S, Hq, Hkv, D, n, causal, part = 1, 1200, 4, 2, 128, 4, True, "zigzag"
    q, k, v, do = (x.cuda() for x in backward_inputs(B, S, Hq, Hkv, D, "bf16", seed=22))
    o, l = ra.ra_ring_attention(q, k, v, n, causal, part, out_dtype=torch.float32)
    ref = ra.ra_ring_attention_backward(q, k, v, o, l, do, n, causal, part)
    expected = {"bwd_dq": query_tile_work(S, n, part, causal, BM) * (B * Hq),
                "bwd_dkv": key_tile_work(S, n, part, causal, Hq // Hkv) * (B * Hkv)}
    for kernel, exp in expected.items():
        rec = torch.zeros((4096, 4), dtype=torch.int64, device="cuda")
        ra.ra_set_cta_timeline(rec, kernel)
        try:
            got = ra.ra_ring_attention_backward(q, k, v, o, l, do, n, causal, part)
            torch.cuda.synchronize()
        finally:
            ra.ra_set_cta_timeline(None)
        for a, b in zip(got, ref):
            assert torch.equal(a, b), f"{kernel}: the timeline changed the gradient"
        check_records(rec, exp, kernel)
    assert ra.ra_get_device_status() == 0
