"""ra_ring_attention_noalloc: the entry point for callers that cannot
allocate device memory at call time (their framework owns the GPU's memory
pool, or cudaMalloc's implicit synchronisation is not acceptable).  Its
scratch is a fixed device array inside the library.

Checked through the C ABI against ra_ring_attention with a caller-provided
workspace, on workloads that do need scratch, twice in a row (the second call
reuses the array as the first left it).  This file is collected last on
purpose: run alone (fresh process) or after every other test, it must pass.
"""
import ctypes

import numpy as np
import pytest
import torch

from seeded_inputs import WORKLOADS, attention_inputs, workload_inputs

pytestmark = pytest.mark.gpu

ATOL, RTOL_L2 = 2e-2, 1e-2


def close(got, ref, what):
    got = got.detach().float().cpu().numpy().astype(np.float64)
    ref = ref.detach().float().cpu().numpy().astype(np.float64)
    assert np.array_equal(np.isneginf(got), np.isneginf(ref)), what
    fin = ~np.isneginf(ref)
    err = np.abs(got[fin] - ref[fin])
    assert float(err.max()) <= ATOL, f"{what}: max-abs {float(err.max()):.3e}"
    rel = np.linalg.norm(got[fin] - ref[fin]) / max(np.linalg.norm(ref[fin]), 1e-30)
    assert rel <= RTOL_L2, f"{what}: rel-L2 {rel:.3e}"


def cases():
    # fp32 inputs: rounded to bf16 in scratch (the tiny workload)
    w = WORKLOADS["tiny"]
    q, k, v = workload_inputs(w)
    yield "tiny-f32-in", (q, k, v), dict(n_blocks=w.n_blocks, causal=w.causal, partition=w.partition,
                                         sched="persistent", out_dtype=torch.float32)
    # unfused schedule with bf16 output: fp32 running output and per-step partials in scratch
    q, k, v = attention_inputs(1, 2048, 4, 2, 128, "bf16", seed=5)
    yield "zigzag2k-unfused-bf16", (q, k, v), dict(n_blocks=4, causal=True, partition="zigzag", sched="unfused",
                                                   out_dtype=torch.bfloat16)
    yield "zigzag2k-fused-bf16", (q, k, v), dict(n_blocks=4, causal=True, partition="zigzag", sched="fused",
                                                 out_dtype=torch.bfloat16)


@pytest.mark.parametrize("name,inputs,kw", list(cases()), ids=lambda x: x if isinstance(x, str) else "")
def test_noalloc_matches_workspace_entry_point(cuda_lib, name, inputs, kw):
    ra = cuda_lib
    q, k, v = (t.cuda() for t in inputs)
    need = ra.ra_ring_attention_workspace(q.shape[0], q.shape[1], q.shape[2], q.shape[3], kw["n_blocks"],
                                          q.shape[2] // k.shape[2], kw["partition"], q.dtype, "ring", kw["sched"],
                                          kw["out_dtype"])
    assert 0 < need <= ra.ra_noalloc_scratch_bytes()  # the case really uses scratch
    ref_o, ref_l = ra.ra_ring_attention(q, k, v, kw["n_blocks"], kw["causal"], kw["partition"],
                                        out_dtype=kw["out_dtype"], sched=kw["sched"])
    out = torch.empty_like(ref_o)
    lse = torch.empty_like(ref_l)
    for call in range(2):
        out.fill_(float("nan"))
        lse.fill_(float("nan"))
        torch.cuda.synchronize()
        # The second call runs with every module already loaded: neither the
        # device's free memory nor torch's allocator may move across it.
        free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
        ra.ra_ring_attention_noalloc(q, k, v, kw["n_blocks"], kw["causal"], kw["partition"], out=out, lse=lse,
                                     sched=kw["sched"])
        torch.cuda.synchronize()
        if call == 1:
            assert torch.cuda.mem_get_info()[0] == free0, f"{name}: device free memory changed"
            assert torch.cuda.memory_allocated() == alloc0, f"{name}: torch allocated memory"
        close(out, ref_o, f"{name} out, call {call}")
        close(lse, ref_l, f"{name} lse, call {call}")
    assert ra.ra_get_device_status() == 0


def test_noalloc_rejects_scratch_beyond_its_array(cuda_lib):
    ra = cuda_lib
    fake = 1 << 20  # never dereferenced: the size check comes first
    unf = ra.ra_options(0, ra.RA_SCHED_UNFUSED, None, None, 0)
    # gqa24k, unfused, bf16 out: ~0.8 GB of fp32 running output and partials
    st = ra._lib.ra_ring_attention_noalloc(fake, fake, fake, ra.RA_BF16, 1, 24000, 32, 128, 4, 1, ra.RA_PART_ZIGZAG,
                                           4, fake, ra.RA_BF16, fake, ctypes.byref(unf), None)
    assert st == ra.RA_ERR_WORKSPACE
