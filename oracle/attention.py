"""Full softmax attention, written out from its definition in fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

What the blockwise method must reproduce exactly (TokenRing review,
"Assumptions & free parameters": the merge "exactly reproduces standard
attention"; Anthology of the SOTA, SOTA-181: "the attention is unchanged and
exact").  For batch b, query head h and query token i, with KV head
g = h // gqa_groups (contiguous GQA groups, TokenRing review, "If this is
right", grouped / multi-query attention):

    s_ij   = (1 / sqrt(D)) * sum_d q[b,i,h,d] * k[b,j,g,d]
    visible: all j, or j <= i when causal (original token indices)
    lse_i  = ln sum_{j visible} exp(s_ij)
    out_i  = sum_{j visible} exp(s_ij - lse_i) * v[b,j,g,:]

The scale 1/sqrt(D) is the plain scaled dot product; the pages do not state a
scale.  Rows are processed in chunks so the S x S score matrix is never held;
the chunking is over independent query rows only and changes no arithmetic.
"""
from __future__ import annotations

import math

import numpy as np


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor (any dtype, including bf16)
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def softmax_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)


def full_attention(q, k, v, causal: bool, gqa_groups: int = 1, row_chunk: int = 512):
    """Exact attention over the whole sequence.

    q: [B, S, Hq, D]; k, v: [B, S, Hkv, D] with Hq = Hkv * gqa_groups.
    Returns (out [B, S, Hq, D], lse [B, S, Hq]) in fp64, natural log.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if Hq != Hkv * gqa_groups:
        raise ValueError("Hq must equal Hkv * gqa_groups")
    scale = softmax_scale(D)
    out = np.zeros((B, S, Hq, D), dtype=np.float64)
    lse = np.full((B, S, Hq), -np.inf, dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            g = h // gqa_groups
            kk = k[b, :, g, :]
            vv = v[b, :, g, :]
            for i0 in range(0, S, row_chunk):
                i1 = min(S, i0 + row_chunk)
                # causal rows i0..i1-1 see keys 0..i1-1 at most
                jmax = i1 if causal else S
                s = (q[b, i0:i1, h, :] @ kk[:jmax].T) * scale
                if causal:
                    rows = np.arange(i0, i1)[:, None]
                    cols = np.arange(jmax)[None, :]
                    s = np.where(cols <= rows, s, -np.inf)
                m = s.max(axis=1, keepdims=True)
                e = np.exp(s - m)
                tot = e.sum(axis=1, keepdims=True)
                lse[b, i0:i1, h] = (m + np.log(tot))[:, 0]
                out[b, i0:i1, h, :] = (e / tot) @ vv[:jmax]
    return out, lse


def attention_rows(q, k, v, rows, causal: bool, gqa_groups: int = 1, batch: int = 32):
    """Exact attention for selected query rows only.

    rows: iterable of (b, i, h).  Returns (out [R, D], lse [R]) in fp64.
    Used where the full oracle is too large: each sampled row is computed
    against every key it may see.  ``batch`` bounds how many rows are
    evaluated together (memory only; the result does not depend on it).
    """
    rows = list(rows)
    D = q.shape[-1]
    scale = softmax_scale(D)
    out = np.zeros((len(rows), D), dtype=np.float64)
    lse = np.zeros((len(rows),), dtype=np.float64)
    # Rows that share (batch, KV head) are evaluated together against that
    # head's keys (a matrix product instead of one matrix-vector product per
    # row); each row still sees every key it may see, in one softmax.
    groups = {}
    for r, (b, i, h) in enumerate(rows):
        groups.setdefault((b, h // gqa_groups), []).append(r)
    for (b, g), idx in groups.items():
        jall = max(rows[r][1] for r in idx) + 1 if causal else q.shape[1]
        kk = _f64(k[b, :jall, g, :])
        vv = _f64(v[b, :jall, g, :])
        for s0 in range(0, len(idx), batch):
            sel = idx[s0:s0 + batch]
            ii = np.array([rows[r][1] for r in sel])
            jmax = int(ii.max()) + 1 if causal else q.shape[1]
            qq = np.stack([_f64(q[b, rows[r][1], rows[r][2], :]) for r in sel])
            s = (qq @ kk[:jmax].T) * scale
            if causal:
                s = np.where(np.arange(jmax)[None, :] <= ii[:, None], s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            tot = e.sum(axis=1, keepdims=True)
            lse[sel] = (m + np.log(tot))[:, 0]
            out[sel] = (e / tot) @ vv[:jmax]
    return out, lse


def decode_attention(q, k, v, causal: bool, gqa_groups: int = 1):
    """Attention of the last Tq tokens of a sequence over its Skv cached keys.

    q: [B, Tq, Hq, D] holds the queries of tokens Skv - Tq .. Skv - 1;
    k, v: [B, Skv, Hkv, D] the key/value cache of tokens 0 .. Skv - 1.
    Query i (position Skv - Tq + i) sees key j iff j <= Skv - Tq + i when
    causal, every key otherwise.  Returns (out [B, Tq, Hq, D], lse [B, Tq, Hq])
    in fp64.  TokenRing review, "Reading between the lines": the decode-phase
    KV-cache variant; the computation is plain softmax attention per query.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Tq, Hq, D = q.shape
    Skv = k.shape[1]
    if Tq > Skv:
        raise ValueError("more queries than cached tokens")
    scale = softmax_scale(D)
    out = np.zeros((B, Tq, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Tq, Hq), dtype=np.float64)
    pos = Skv - Tq + np.arange(Tq)
    for b in range(B):
        for h in range(Hq):
            g = h // gqa_groups
            s = (q[b, :, h, :] @ k[b, :, g, :].T) * scale
            if causal:
                s = np.where(np.arange(Skv)[None, :] <= pos[:, None], s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            tot = e.sum(axis=1, keepdims=True)
            lse[b, :, h] = (m + np.log(tot))[:, 0]
            out[b, :, h, :] = (e / tot) @ v[b, :, g, :]
    return out, lse
