"""Failure detection without a GPU fault: a bounded wait that runs out.

The block-attention kernel's waits are bounded (about 1 s of SM clocks).
With ra_options.fault_inject = 1 the TMA producer withholds one K tile, so
the tensor-core issuer's wait for it expires: the kernel must record
RA_ERR_TIMEOUT in the device status word, stop every CTA, drain its copies
and products and return, leaving the context usable.  Nothing here traps,
faults or hangs a GPU; the failure is a load that is never issued."""
import time

import numpy as np
import pytest
import torch

from oracle import attention as F
from seeded_inputs import attention_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("tiling", ["kv_split", "row_pairs"])
def test_bounded_wait_reports_timeout_and_context_survives(cuda_lib, tiling):
    ra = cuda_lib
    B, S, Hq, Hkv, D, n = 1, 2048, 4, 2, 128, 4
    q, k, v = attention_inputs(B, S, Hq, Hkv, D, "bf16", seed=21)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    assert ra.ra_get_device_status() == ra.RA_OK
    t0 = time.monotonic()
    ra.ra_ring_attention(qd, kd, vd, n, True, "zigzag", tiling=tiling, fault_inject=1)
    assert ra.ra_get_device_status() == ra.RA_ERR_TIMEOUT  # synchronises, then clears the word
    assert time.monotonic() - t0 < 60.0
    # the context is still usable: the same call without the fault is exact
    out, lse = ra.ra_ring_attention(qd, kd, vd, n, True, "zigzag", tiling=tiling)
    torch.cuda.synchronize()
    ro, rl = F.full_attention(q, k, v, True, Hq // Hkv)
    assert np.max(np.abs(out.cpu().double().numpy() - ro)) <= 2e-2
    assert np.max(np.abs(lse.cpu().double().numpy() - rl)) <= 2e-2
    assert ra.ra_get_device_status() == ra.RA_OK
