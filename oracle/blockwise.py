"""Blockwise attention with the pages' merge rule, fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring).  This module shares no
code with ``oracle.attention``: the per-block softmax below is written again
here on purpose, so that the identity "blockwise + merge == full attention"
checks two independent computations.

Steps, in the pages' order and notation:

1. Partition (TokenRing review, "Referee Report / Summary": Q, K, V split
   along the token dimension).  Contiguous: block r holds tokens
   [r*L, (r+1)*L).  Zigzag (same page, "If this is right", zigzag causal
   partition; the pages give no pseudo-code, "minor comments, section 3.3.2"):
   with c = S / (2n), block r holds chunk r followed by chunk 2n-1-r.
2. Schedule (order of (q block, kv block) pairs).  Ring (Anthology of the
   SOTA, SOTA-181): at step s = 0..n-1, query block r meets KV block
   (r - s) mod n.  TokenRing (TokenRing review, "Core claim" and "major
   comments, Algorithm 1 (section 3.2)"): KV block j stays put; at step
   = 1..n it meets query block t = (j - step + 1) mod n (step is read as
   1-based, every rank index taken mod n).
3. Per pair, a block partial (block_out, block_lse): softmax attention of the
   query block over the KV block's keys, masked with original token positions
   (key visible iff kpos <= qpos under causal).  A row that sees no key in the
   block gets block_lse = -inf and block_out = 0.
4. Merge (TokenRing review, "What carries the argument"):
       out <- out - sigma(block_lse - lse) * (out - block_out)
       lse <- lse - ln sigma(lse - block_lse)
   starting from out = 0, lse = -inf.
5. Scatter rows back to original token order.
"""
from __future__ import annotations

import math

import numpy as np


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------- partitions

def zigzag_perm(S: int, n: int) -> np.ndarray:
    """perm[p] = original token index of permuted row p (block-major order).

    Block r = chunk r then chunk 2n-1-r, chunk size c = S / (2n).
    """
    if S % (2 * n) != 0:
        raise ValueError("zigzag needs S divisible by 2 * n_blocks")
    c = S // (2 * n)
    perm = []
    for r in range(n):
        perm.extend(range(r * c, (r + 1) * c))
        first = 2 * n - 1 - r
        perm.extend(range(first * c, (first + 1) * c))
    return np.asarray(perm, dtype=np.int64)


def contiguous_perm(S: int, n: int) -> np.ndarray:
    if S % n != 0:
        raise ValueError("contiguous partition needs S divisible by n_blocks")
    return np.arange(S, dtype=np.int64)


def partition_perm(S: int, n: int, partition: str) -> np.ndarray:
    if partition == "zigzag":
        return zigzag_perm(S, n)
    if partition == "contiguous":
        return contiguous_perm(S, n)
    raise ValueError(partition)


def permute_rows(x, perm: np.ndarray, inverse: bool = False) -> np.ndarray:
    """Gather (dst[:, p] = src[:, perm[p]]) or its inverse scatter along axis 1."""
    x = np.asarray(x)
    if not inverse:
        return x[:, perm]
    y = np.empty_like(x)
    y[:, perm] = x
    return y


# ----------------------------------------------------------------- schedules

def ring_schedule(n: int):
    """Steps of the ring: step s pairs query block r with KV block (r - s) mod n."""
    return [[(r, (r - s) % n) for r in range(n)] for s in range(n)]


def tokenring_schedule(n: int):
    """Steps of TokenRing: at step (1-based) KV block j meets Q block (j - step + 1) mod n."""
    return [[((j - step + 1) % n, j) for j in range(n)] for step in range(1, n + 1)]


def schedule(n: int, order: str):
    if order == "ring":
        return ring_schedule(n)
    if order == "tokenring":
        return tokenring_schedule(n)
    raise ValueError(order)


# ------------------------------------------------------------- merge rule

def sigmoid(x):
    """sigma(x) = 1 / (1 + e^-x), evaluated without overflow on either side."""
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore", invalid="ignore"):
        e = np.exp(-np.abs(x))  # in (0, 1]; e^-x for x >= 0, e^x for x < 0
        return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def log_sigmoid(x):
    """ln sigma(x) = -ln(1 + e^-x), evaluated without overflow on either side."""
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore", invalid="ignore"):
        return np.minimum(x, 0.0) - np.log1p(np.exp(-np.abs(x)))


def merge_rule(out, lse, block_out, block_lse):
    """One application of the pages' update; returns the new (out, lse).

    out/block_out: [..., D]; lse/block_lse: [...].  lse = -inf marks an empty
    partial (no key seen yet): merging an empty partial changes nothing, and
    merging into an empty state copies the partial.  Those two cases are where
    the literal formula would form -inf - (-inf).
    """
    out = np.asarray(out, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    block_out = np.asarray(block_out, dtype=np.float64)
    block_lse = np.asarray(block_lse, dtype=np.float64)
    with np.errstate(invalid="ignore"):
        w = sigmoid(block_lse - lse)
        new_out = out - w[..., None] * (out - block_out)
        new_lse = lse - log_sigmoid(lse - block_lse)
    block_empty = np.isneginf(block_lse)
    state_empty = np.isneginf(lse) & ~block_empty
    new_out = np.where(block_empty[..., None], out, new_out)
    new_lse = np.where(block_empty, lse, new_lse)
    new_out = np.where(state_empty[..., None], block_out, new_out)
    new_lse = np.where(state_empty, block_lse, new_lse)
    return new_out, new_lse


def merge_partials(outs, lses):
    """Fold k partials left to right with the merge rule (accumulator = partial 0)."""
    out = np.asarray(outs[0], dtype=np.float64).copy()
    lse = np.asarray(lses[0], dtype=np.float64).copy()
    for o, l in zip(outs[1:], lses[1:]):
        out, lse = merge_rule(out, lse, o, l)
    return out, lse


# ------------------------------------------------------------ block partial

def block_partial(qb, kb, vb, qpos, kpos, causal: bool, gqa_groups: int = 1):
    """Softmax attention of one query block over one KV block.

    qb: [B, Lq, Hq, D]; kb, vb: [B, Lk, Hkv, D]; qpos [Lq], kpos [Lk] are the
    original token indices of the rows.  Returns (block_out [B, Lq, Hq, D],
    block_lse [B, Lq, Hq]); rows with no visible key give (0, -inf).
    """
    qb, kb, vb = _f64(qb), _f64(kb), _f64(vb)
    B, Lq, Hq, D = qb.shape
    scale = 1.0 / math.sqrt(D)
    bo = np.zeros((B, Lq, Hq, D), dtype=np.float64)
    bl = np.full((B, Lq, Hq), -np.inf, dtype=np.float64)
    if causal:
        vis = np.asarray(kpos)[None, :] <= np.asarray(qpos)[:, None]
    else:
        vis = np.ones((Lq, kb.shape[1]), dtype=bool)
    any_vis = vis.any(axis=1)
    if not any_vis.any():
        return bo, bl
    for b in range(B):
        for h in range(Hq):
            g = h // gqa_groups
            logits = (qb[b, :, h, :] @ kb[b, :, g, :].T) * scale
            logits = np.where(vis, logits, -np.inf)
            rmax = np.where(any_vis, logits.max(axis=1), 0.0)
            with np.errstate(invalid="ignore"):
                ex = np.exp(logits - rmax[:, None])
            ex = np.where(vis, ex, 0.0)
            den = ex.sum(axis=1)
            ok = den > 0
            safe = np.where(ok, den, 1.0)
            bo[b, :, h, :] = np.where(ok[:, None], (ex / safe[:, None]) @ vb[b, :, g, :], 0.0)
            bl[b, :, h] = np.where(ok, rmax + np.log(safe), -np.inf)
    return bo, bl


# ------------------------------------------------------------ whole method

def pair_is_empty(qpos_blk, kpos_blk, causal: bool) -> bool:
    """True when no key of the KV block is visible to any query of the Q block."""
    return causal and int(np.min(kpos_blk)) > int(np.max(qpos_blk))


def blockwise_attention(q, k, v, n_blocks: int, causal: bool, partition: str = "contiguous",
                        gqa_groups: int = 1, order: str = "ring", pairs=None,
                        return_partials: bool = False):
    """The blockwise method end to end; returns (out, lse) in original token order.

    ``pairs`` overrides the schedule with an explicit sequence of
    (q_block, kv_block) pairs (used to test order invariance).  Pairs whose
    blocks see no key at all under the causal mask are skipped.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, S, Hq, D = q.shape
    n = n_blocks
    perm = partition_perm(S, n, partition)
    L = S // n
    qp = permute_rows(q, perm)
    kp = permute_rows(k, perm)
    vp = permute_rows(v, perm)
    pos = perm.reshape(n, L)
    out = np.zeros((B, S, Hq, D), dtype=np.float64)
    lse = np.full((B, S, Hq), -np.inf, dtype=np.float64)
    if pairs is None:
        pairs = [p for step in schedule(n, order) for p in step]
    partials = []
    for (qi, kj) in pairs:
        if pair_is_empty(pos[qi], pos[kj], causal):
            continue
        qs = slice(qi * L, (qi + 1) * L)
        ks = slice(kj * L, (kj + 1) * L)
        bo, bl = block_partial(qp[:, qs], kp[:, ks], vp[:, ks], pos[qi], pos[kj], causal, gqa_groups)
        if return_partials:
            partials.append(((qi, kj), bo, bl))
        out[:, qs], lse[:, qs] = merge_rule(out[:, qs], lse[:, qs], bo, bl)
    out = permute_rows(out, perm, inverse=True)
    lse = permute_rows(lse, perm, inverse=True)
    if return_partials:
        return out, lse, partials
    return out, lse


def visible_pairs_per_block(S: int, n: int, partition: str) -> np.ndarray:
    """Number of causal (query, key) pairs whose query lies in each block."""
    pos = partition_perm(S, n, partition).reshape(n, S // n)
    return (pos + 1).sum(axis=1)


def kv_splits(Skv: int, n_splits: int):
    """Contiguous chunks of the KV cache: chunk i = [i*Lk, min((i+1)*Lk, Skv)),
    Lk = ceil(Skv / n_splits); the last chunk may be shorter."""
    Lk = -(-Skv // n_splits)
    return [(i * Lk, min((i + 1) * Lk, Skv)) for i in range(n_splits) if i * Lk < Skv]


def decode_blockwise(q, k, v, causal: bool, gqa_groups: int, n_splits: int):
    """Decode attention by KV-cache chunks: one partial per chunk
    (block_partial), folded with the merge rule (merge_partials).  Query i has
    position Skv - Tq + i.  TokenRing review, "Reading between the lines"."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    Tq, Skv = q.shape[1], k.shape[1]
    qpos = Skv - Tq + np.arange(Tq)
    outs, lses = [], []
    for (j0, j1) in kv_splits(Skv, n_splits):
        bo, bl = block_partial(q, k[:, j0:j1], v[:, j0:j1], qpos, np.arange(j0, j1), causal, gqa_groups)
        outs.append(bo)
        lses.append(bl)
    return merge_partials(outs, lses)
