"""The checked build (libra_b200_debug.so, compiled with -DRA_DEBUG_BOUNDS).

Every run-time-indexed global access of the kernels (TMA rows and heads,
output rows, lse / Delta entries, merge rows) and every segment-table read is
checked on the device against the extent it must lie in.  Here the edge cases
run on that build, in a child process that loads it (RA_DEBUG_BOUNDS=1): the
results must match the fp64 oracle and no check may fail.  A last case makes
the producer check a row past the end of the K tensor (fault_inject = 2, a
value only the checked build accepts): the copy is skipped, nothing faults,
and the status word must read RA_ERR_DEVICE_BOUNDS with the failed check's
record; the next call on the same context must be correct again.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import numpy as np
import torch
import blockwise_exact_attention_block_b200 as ra
from oracle import attention as F
from oracle import backward as G
from oracle import blockwise as K
from seeded_inputs import attention_inputs, backward_inputs, decode_inputs, merge_inputs

assert ra.ra_debug_build(), "the checked build was not loaded"
ATOL, RTOL = 2e-2, 1e-2

def close(got, ref, what, atol=ATOL):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.array_equal(np.isneginf(got), np.isneginf(ref)), what
    fin = ~np.isneginf(ref)
    err = np.abs(got[fin] - ref[fin])
    assert float(err.max()) <= atol, (what, float(err.max()))
    rel = np.linalg.norm(got[fin] - ref[fin]) / max(np.linalg.norm(ref[fin]), 1e-30)
    assert rel <= RTOL, (what, rel)

def clean(what):
    st = ra.ra_get_device_status()
    rec = ra.ra_get_bounds_record()
    assert st == 0 and rec == (0, 0, 0), (what, ra.ra_status_string(st), rec)

# forward: the edge cases of the release tests, every schedule and tiling
for (B, S, Hq, Hkv, D, n, causal, part) in [
        (1, 32, 1, 1, 128, 16, True, "zigzag"),      # chunks of a single row
        (1, 1200, 4, 2, 128, 4, True, "zigzag"),     # 150-row chunks: ragged tiles
        (1, 2000, 4, 1, 128, 4, True, "zigzag"),     # c = 250, ragged tails
        (3, 384, 6, 2, 64, 3, True, "zigzag"),       # batch 3, GQA 3, D = 64
        (2, 640, 4, 4, 64, 5, False, "contiguous")]:
    q, k, v = attention_inputs(B, S, Hq, Hkv, D, "bf16", seed=6)
    ro, rl = F.full_attention(q, k, v, causal, Hq // Hkv)
    for sched in ("persistent", "fused", "unfused"):
        for tiling in ("auto", "row_pairs", "kv_split", "cluster2"):
            o, l = ra.ra_ring_attention(q.cuda(), k.cuda(), v.cuda(), n, causal, part, out_dtype=torch.float32,
                                        sched=sched, tiling=tiling)
            what = f"forward S={S} n={n} D={D} {sched}/{tiling}"
            clean(what)
            close(o.cpu().numpy(), ro, what + " out")
            close(l.cpu().numpy(), rl, what + " lse")
    # one block pair through the block-local entry point
    L = S // n
    perm = K.partition_perm(S, n, part)
    pt = torch.from_numpy(perm)
    qb, kb = 0, n - 1
    qp, kp, vp = (x[:, pt] for x in (q, k, v))
    bo, bl = ra.ra_block_attn(qp[:, qb * L:(qb + 1) * L].contiguous().cuda(), kp[:, kb * L:(kb + 1) * L].contiguous().cuda(),
                              vp[:, kb * L:(kb + 1) * L].contiguous().cuda(), S, n, qb, kb, causal, part)
    torch.cuda.synchronize()
    clean(f"block pair S={S}")

# backward: ragged zigzag, GQA, D = 64 and 128, one-row chunks
for (B, S, Hq, Hkv, D, n, causal, part) in [
        (1, 1200, 4, 2, 128, 4, True, "zigzag"),
        (1, 32, 2, 1, 64, 16, True, "zigzag"),
        (2, 200, 2, 2, 128, 1, True, "contiguous")]:
    q, k, v, do = backward_inputs(B, S, Hq, Hkv, D, "bf16", seed=10)
    o, l = ra.ra_ring_attention(q.cuda(), k.cuda(), v.cuda(), n, causal, part, out_dtype=torch.float32)
    dq, dk, dv = ra.ra_ring_attention_backward(q.cuda(), k.cuda(), v.cuda(), o, l, do.cuda(), n, causal, part)
    clean(f"backward S={S}")
    rq, rk, rv = G.attention_backward(q, k, v, do, causal, Hq // Hkv)
    for got, ref, nm in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        close(got.cpu().numpy(), ref, f"backward S={S} {nm}", atol=2e-2 * max(1.0, float(np.abs(ref).max())))
    clean(f"backward S={S}")

# merges: pairwise and k-way, with empty partials
outs, lses = merge_inputs(4096, 5, seed=3)
lses[1][0, :4] = float("-inf")
ref_o, ref_l = K.merge_partials([x.double().numpy() for x in outs], [x.double().numpy() for x in lses])
go, gl = ra.ra_merge_partials([x.cuda() for x in outs], [x.cuda() for x in lses])
clean("k-way merge")
close(go.cpu().numpy(), ref_o, "k-way merge", atol=1e-5)
o, l = outs[0].cuda(), lses[0].cuda()
for j in range(1, 5):
    ra.ra_merge_partial(o, l, outs[j].cuda(), lses[j].cuda())
close(o.cpu().numpy(), ref_o, "pairwise merge", atol=1e-5)
clean("merges")

# decode over a ragged cache
q, k, v = decode_inputs(2, 3, 1000, 8, 2, 128, seed=11)
ro, rl = F.decode_attention(q, k, v, True, 4)
o, l = ra.ra_decode_attention(q.cuda(), k.cuda(), v.cuda(), True, 0, out_dtype=torch.float32)
clean("decode")
close(o.cpu().numpy(), ro, "decode out")

# an injected out-of-range row: recorded, skipped, no fault
q, k, v = attention_inputs(1, 1024, 2, 2, 128, "bf16", seed=12)
for tiling in ("row_pairs", "kv_split"):
    ra.ra_ring_attention(q.cuda(), k.cuda(), v.cuda(), 4, True, "zigzag", out_dtype=torch.float32,
                         tiling=tiling, fault_inject=2)
    torch.cuda.synchronize()
    st = ra.ra_get_device_status()
    line, idx, lim = ra.ra_get_bounds_record()
    assert st == ra.RA_ERR_DEVICE_BOUNDS, ra.ra_status_string(st)
    assert line > 0 and idx >= lim == 1024, (line, idx, lim)
    ro, rl = F.full_attention(q, k, v, True, 1)
    o, l = ra.ra_ring_attention(q.cuda(), k.cuda(), v.cuda(), 4, True, "zigzag", out_dtype=torch.float32,
                                tiling=tiling)
    close(o.cpu().numpy(), ro, f"after the injected check ({tiling})")
    clean(f"after the injected check ({tiling})")
print("CHECKED_BUILD_OK")
'''


def test_checked_build_edge_cases_and_injected_check():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = os.path.join(ROOT, "blockwise_exact_attention_block_b200", "libra_b200_debug.so")
    assert os.path.exists(lib), "libra_b200_debug.so is missing: build it (build.py --debug-bounds)"
    env = dict(os.environ, RA_DEBUG_BOUNDS="1", PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    res = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                         timeout=900)
    assert res.returncode == 0 and "CHECKED_BUILD_OK" in res.stdout, res.stdout[-3000:] + res.stderr[-3000:]
