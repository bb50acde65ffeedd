"""Gradients of exact blockwise attention, fp64.  TEST INFRASTRUCTURE ONLY
(see the package docstring: only tests, the smoke check and the bench's CPU
baseline may use it; it shares no code with the CUDA path).

Anthology of the SOTA, SOTA-181: ring attention trains models (million-token
language modelling), so the blockwise computation has a backward pass.  The
forward keeps, per query row, the log-sum-exp of the whole row (TokenRing
review, "What carries the argument": the merged lse); with it every
(query block, KV block) pair's share of the gradient is independent of the
other pairs, and the shares add up.

Definition, per batch b and query head h reading KV head g = h // groups,
scale s = 1 / sqrt(D), P = softmax(s Q K^T + mask) by rows, O = P V, and an
upstream gradient dO:

    dV = P^T dO
    dP = dO V^T
    dS = P * (dP - Delta),   Delta_i = sum_d dO[i, d] O[i, d]
    dQ = s dS K
    dK = s dS^T Q

(Delta_i equals sum_j P_ij dP_ij.)  dK and dV of a KV head sum over the query
heads that read it.

* ``attention_backward`` - the definition over whole rows.
* ``blockwise_backward`` - the same gradient as sums over the (query block,
  KV block) pairs of a partition, each pair's probabilities rebuilt from the
  full-row lse: P_ij = exp(s Q_i K_j^T - lse_i).  It shares no code with
  ``attention_backward``.
* ``backward_query_rows`` / ``backward_key_rows`` - the definition evaluated
  one row at a time, for sampled rows of workloads too large for the whole
  matrices: dq of a query row needs only that row's keys; dk, dv of a key need
  every query row that sees it, each with its own full row.
"""
from __future__ import annotations

import math

import numpy as np


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def attention_backward(q, k, v, dout, causal: bool, gqa_groups: int = 1):
    """(dq, dk, dv) of full softmax attention for the upstream gradient dout.

    q, dout: [B, S, Hq, D]; k, v: [B, S, Hkv, D].  Returns fp64 arrays of the
    same shapes as q, k, v.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, S, Hq, D = q.shape
    s = 1.0 / math.sqrt(D)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    mask = np.tril(np.ones((S, S), dtype=bool)) if causal else np.ones((S, S), dtype=bool)
    for b in range(B):
        for h in range(Hq):
            g = h // gqa_groups
            logits = np.where(mask, (q[b, :, h] @ k[b, :, g].T) * s, -np.inf)
            m = logits.max(axis=1, keepdims=True)
            e = np.exp(logits - m)
            p = e / e.sum(axis=1, keepdims=True)
            o = p @ v[b, :, g]
            dv[b, :, g] += p.T @ do[b, :, h]
            dp = do[b, :, h] @ v[b, :, g].T
            delta = (do[b, :, h] * o).sum(axis=1, keepdims=True)
            ds = p * (dp - delta)
            dq[b, :, h] = s * (ds @ k[b, :, g])
            dk[b, :, g] += s * (ds.T @ q[b, :, h])
    return dq, dk, dv


def blockwise_backward(q, k, v, dout, out, lse, n_blocks: int, causal: bool, partition: str = "contiguous",
                       gqa_groups: int = 1):
    """The gradient as a sum over the (query block, KV block) pairs of the
    partition, given the forward's out and full-row lse (natural log).

    Blocks follow the forward's partition (contiguous, or zigzag: block r =
    chunk r then chunk 2n-1-r); the mask uses original positions.  For every
    pair: P = exp(s Q_i K_j^T - lse_i) on visible keys, dV_j += P^T dO_i,
    dP = dO_i V_j^T, dS = P (dP - Delta_i), dQ_i += s dS K_j, dK_j += s dS^T Q_i.
    """
    q, k, v, do, o, lse = _f64(q), _f64(k), _f64(v), _f64(dout), _f64(out), _f64(lse)
    B, S, Hq, D = q.shape
    s = 1.0 / math.sqrt(D)
    n = n_blocks
    if partition == "zigzag":
        c = S // (2 * n)
        blocks = [np.concatenate([np.arange(r * c, (r + 1) * c), np.arange((2 * n - 1 - r) * c, (2 * n - r) * c)])
                  for r in range(n)]
    else:
        L = S // n
        blocks = [np.arange(r * L, (r + 1) * L) for r in range(n)]
    delta = (do * o).sum(axis=3)  # [B, S, Hq]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for qi in blocks:
        for kj in blocks:
            vis = (kj[None, :] <= qi[:, None]) if causal else np.ones((len(qi), len(kj)), dtype=bool)
            if not vis.any():
                continue
            for b in range(B):
                for h in range(Hq):
                    g = h // gqa_groups
                    qb, kb, vb, dob = q[b, qi, h], k[b, kj, g], v[b, kj, g], do[b, qi, h]
                    p = np.where(vis, np.exp((qb @ kb.T) * s - lse[b, qi, h][:, None]), 0.0)
                    dv[b, kj, g] += p.T @ dob
                    ds = p * (dob @ vb.T - delta[b, qi, h][:, None])
                    dq[b, qi, h] += s * (ds @ kb)
                    dk[b, kj, g] += s * (ds.T @ qb)
    return dq, dk, dv


def _row(q_row, keys, vals, do_row, s):
    """One query row against its visible keys: (p, dp, delta)."""
    logits = (keys @ q_row) * s
    e = np.exp(logits - logits.max())
    p = e / e.sum()
    o = p @ vals
    return p, vals @ do_row, float(do_row @ o)


def backward_query_rows(q, k, v, dout, rows, causal: bool, gqa_groups: int = 1) -> np.ndarray:
    """dq at the (b, i, h) triples of ``rows``, one fp64 [D] vector each."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    S, D = q.shape[1], q.shape[3]
    s = 1.0 / math.sqrt(D)
    out = np.zeros((len(rows), D))
    for n, (b, i, h) in enumerate(rows):
        g = h // gqa_groups
        end = i + 1 if causal else S
        keys, vals = k[b, :end, g], v[b, :end, g]
        p, dp, delta = _row(q[b, i, h], keys, vals, do[b, i, h], s)
        out[n] = s * ((p * (dp - delta)) @ keys)
    return out


def backward_key_rows(q, k, v, dout, keys, causal: bool, gqa_groups: int = 1):
    """(dk, dv) at the (b, j, g) triples of ``keys``: sums over every query
    head of group g and every query row that sees key j (i >= j when causal),
    each row's probabilities normalised over its own visible keys."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    S, D = q.shape[1], q.shape[3]
    s = 1.0 / math.sqrt(D)
    dk = np.zeros((len(keys), D))
    dv = np.zeros((len(keys), D))
    for n, (b, j, g) in enumerate(keys):
        for h in range(g * gqa_groups, (g + 1) * gqa_groups):
            for i in range(j if causal else 0, S):
                end = i + 1 if causal else S
                p, dp, delta = _row(q[b, i, h], k[b, :end, g], v[b, :end, g], do[b, i, h], s)
                dv[n] += p[j] * do[b, i, h]
                dk[n] += s * p[j] * (dp[j] - delta) * q[b, i, h]
    return dk, dv
