"""Pins for the CPU fp64 oracle (no GPU).

Each test ties the oracle to something other than itself: brute force with
exactly rounded sums, a library routine (torch's scaled-dot-product attention
in fp64), closed forms, and the invariants the pages fix (the merge reproduces
full attention exactly; order and block count do not matter; zigzag keeps the
causal mask and balances the work).  The last group plants plausible mistakes
in copies of the oracle and checks that the pins catch each one.
"""
import itertools
import math

import numpy as np
import pytest
import torch

from oracle import attention as F
from oracle import blockwise as K
from seeded_inputs import WORKLOADS, attention_inputs, workload_inputs

TOL = 1e-12


def brute_attention(q, k, v, causal, groups):
    """Triple loops over plain Python floats with math.fsum (exactly rounded sums)."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, S, Hq, D = q.shape
    out = np.zeros_like(q)
    lse = np.zeros((B, S, Hq))
    for b in range(B):
        for h in range(Hq):
            g = h // groups
            for i in range(S):
                js = range(i + 1) if causal else range(S)
                s = [math.fsum(q[b, i, h, d] * k[b, j, g, d] for d in range(D)) / math.sqrt(D)
                     for j in js]
                m = max(s)
                w = [math.exp(x - m) for x in s]
                tot = math.fsum(w)
                lse[b, i, h] = m + math.log(tot)
                for d in range(D):
                    out[b, i, h, d] = math.fsum(w[t] * v[b, j, g, d] for t, j in enumerate(js)) / tot
    return out, lse


def small(B, S, Hq, Hkv, D, seed=1):
    q, k, v = attention_inputs(B, S, Hq, Hkv, D, dtype="f32", seed=seed)
    return q.double().numpy(), k.double().numpy(), v.double().numpy()


# ------------------------------------------------------------ full attention

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 5, 1, 1, 3), (2, 16, 2, 1, 8), (1, 11, 4, 2, 4)])
def test_full_matches_brute_force(causal, shape):
    B, S, Hq, Hkv, D = shape
    q, k, v = small(B, S, Hq, Hkv, D)
    out, lse = F.full_attention(q, k, v, causal, Hq // Hkv, row_chunk=4)
    bo, bl = brute_attention(q, k, v, causal, Hq // Hkv)
    assert np.max(np.abs(out - bo)) < TOL
    assert np.max(np.abs(lse - bl)) < TOL


@pytest.mark.parametrize("causal", [False, True])
def test_full_matches_torch_sdpa_fp64(causal):
    B, S, Hq, Hkv, D = 2, 96, 4, 2, 16
    q, k, v = small(B, S, Hq, Hkv, D, seed=3)
    out, lse = F.full_attention(q, k, v, causal, Hq // Hkv, row_chunk=32)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal,
                                                           enable_gqa=True)
    ref = ref.permute(0, 2, 1, 3).numpy()
    tk_rep = tk.repeat_interleave(Hq // Hkv, dim=1)
    sc = (tq @ tk_rep.transpose(-1, -2)) / math.sqrt(D)
    if causal:
        sc = sc.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
    ref_lse = torch.logsumexp(sc, dim=-1).permute(0, 2, 1).numpy()
    assert np.max(np.abs(out - ref)) < 1e-12
    assert np.max(np.abs(lse - ref_lse)) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_full_zero_query_closed_form(causal):
    # q = 0: every visible key gets the same weight, out = mean of visible V rows,
    # lse = ln(number of visible keys).
    B, S, Hq, Hkv, D = 1, 40, 2, 1, 8
    _, k, v = small(B, S, Hq, Hkv, D)
    q = np.zeros((B, S, Hq, D))
    out, lse = F.full_attention(q, k, v, causal, 2, row_chunk=16)
    for i in range(S):
        nvis = i + 1 if causal else S
        assert abs(lse[0, i, 0] - math.log(nvis)) < TOL
        assert np.max(np.abs(out[0, i, 1] - v[0, :nvis, 0].mean(axis=0))) < TOL


def test_full_equal_keys_closed_form():
    # all key rows equal: scores are constant along j, so weights are uniform and
    # lse = s + ln(#visible).
    B, S, Hq, D = 1, 24, 1, 8
    q, k, v = small(B, S, Hq, Hq, D)
    k[:] = k[:, :1]
    out, lse = F.full_attention(q, k, v, True, 1, row_chunk=8)
    for i in range(S):
        s = float(q[0, i, 0] @ k[0, 0, 0]) / math.sqrt(D)
        assert abs(lse[0, i, 0] - (s + math.log(i + 1))) < TOL
        assert np.max(np.abs(out[0, i, 0] - v[0, : i + 1, 0].mean(axis=0))) < TOL


def test_full_single_visible_key():
    # causal row 0 sees only key 0: out = v_0 and lse = s_00.
    q, k, v = small(1, 8, 2, 2, 8)
    out, lse = F.full_attention(q, k, v, True, 1)
    for h in range(2):
        assert np.max(np.abs(out[0, 0, h] - v[0, 0, h])) < TOL
        assert abs(lse[0, 0, h] - float(q[0, 0, h] @ k[0, 0, h]) / math.sqrt(8)) < TOL


def test_attention_rows_match_full():
    q, k, v = small(2, 64, 4, 2, 16)
    out, lse = F.full_attention(q, k, v, True, 2)
    rows = [(0, 0, 0), (1, 63, 3), (0, 17, 2), (1, 31, 1)]
    ro, rl = F.attention_rows(q, k, v, rows, True, 2)
    for r, (b, i, h) in enumerate(rows):
        assert np.max(np.abs(ro[r] - out[b, i, h])) < TOL
        assert abs(rl[r] - lse[b, i, h]) < TOL


# ---------------------------------------------------------------- merge rule

def test_merge_equal_partials():
    rng = np.random.default_rng(0)
    o = rng.standard_normal((7, 5))
    l = rng.uniform(-5, 15, 7)
    no, nl = K.merge_rule(o, l, o, l)
    assert np.max(np.abs(no - o)) < TOL
    assert np.max(np.abs(nl - (l + math.log(2)))) < TOL


def test_merge_zero_gap_is_average():
    # bl - l = 0 => sigma = 1/2: the new output is the plain average.
    rng = np.random.default_rng(1)
    o, bo = rng.standard_normal((2, 6, 4))
    l = rng.uniform(-5, 15, 6)
    no, nl = K.merge_rule(o, l, bo, l)
    assert np.max(np.abs(no - 0.5 * (o + bo))) < TOL
    assert np.max(np.abs(nl - (l + math.log(2)))) < TOL


def test_merge_two_point_closed_form():
    # Partial A = softmax over one key with logit a, partial B over one key with
    # logit b: exact union gives weights e^a/(e^a+e^b), e^b/(e^a+e^b) and
    # lse = ln(e^a + e^b).
    for a, b in [(0.3, -1.2), (10.0, 12.5), (-4.0, 14.9), (7.0, 7.0)]:
        va, vb = np.array([[1.0, -2.0]]), np.array([[0.5, 3.0]])
        no, nl = K.merge_rule(va, np.array([a]), vb, np.array([b]))
        wa = math.exp(a) / (math.exp(a) + math.exp(b))
        assert np.max(np.abs(no - (wa * va + (1 - wa) * vb))) < TOL
        assert abs(nl[0] - math.log(math.exp(a) + math.exp(b))) < TOL


def test_merge_empty_partials():
    rng = np.random.default_rng(2)
    o, bo = rng.standard_normal((2, 3, 4))
    l = np.array([1.0, -np.inf, -np.inf])
    bl = np.array([-np.inf, 2.0, -np.inf])
    no, nl = K.merge_rule(o, l, bo, bl)
    assert np.array_equal(no[0], o[0]) and nl[0] == 1.0          # empty block: no-op
    assert np.array_equal(no[1], bo[1]) and nl[1] == 2.0         # empty state: copy
    assert np.array_equal(no[2], o[2]) and np.isneginf(nl[2])    # both empty
    assert np.all(np.isfinite(no))


def test_merge_extreme_gap_no_overflow():
    o, bo = np.array([[1.0]]), np.array([[5.0]])
    no, nl = K.merge_rule(o, np.array([-800.0]), bo, np.array([800.0]))
    assert no[0, 0] == 5.0 and nl[0] == 800.0
    no, nl = K.merge_rule(o, np.array([800.0]), bo, np.array([-800.0]))
    assert no[0, 0] == 1.0 and nl[0] == 800.0


# ------------------------------------------------- blockwise == full (exact)

def test_tiny_workload_blockwise_equals_full():
    w = WORKLOADS["tiny"]
    q, k, v = workload_inputs(w)
    out, lse = F.full_attention(q, k, v, w.causal, w.gqa_groups)
    for order in ("ring", "tokenring"):
        bo, bl = K.blockwise_attention(q, k, v, w.n_blocks, w.causal, w.partition, w.gqa_groups, order)
        assert np.max(np.abs(bo - out)) < TOL
        assert np.max(np.abs(bl - lse)) < TOL


@pytest.mark.parametrize("partition", ["contiguous", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
def test_blockwise_equals_full_gqa(partition, causal):
    q, k, v = small(2, 96, 4, 2, 16, seed=5)
    out, lse = F.full_attention(q, k, v, causal, 2)
    bo, bl = K.blockwise_attention(q, k, v, 4, causal, partition, 2, "tokenring")
    assert np.max(np.abs(bo - out)) < TOL
    assert np.max(np.abs(bl - lse)) < TOL


def test_zigzag4k_shape_reduced_heads_equals_full():
    # The 4k zigzag workload's sequence and block layout (S=4096, n=4, c=512),
    # one head to keep the CPU time short.
    q, k, v = attention_inputs(1, 4096, 1, 1, 32, dtype="bf16", seed=0)
    out, lse = F.full_attention(q, k, v, True, 1)
    bo, bl = K.blockwise_attention(q, k, v, 4, True, "zigzag", 1, "ring")
    assert np.max(np.abs(bo - out)) < 1e-11
    assert np.max(np.abs(bl - lse)) < 1e-11


@pytest.mark.parametrize("causal", [False, True])
def test_order_invariance_all_permutations(causal):
    n = 4
    q, k, v = small(1, 64, 2, 1, 8, seed=7)
    out, lse = F.full_attention(q, k, v, causal, 2)
    for kv_order in itertools.permutations(range(n)):
        pairs = [(r, kv_order[(r + s) % n]) for s in range(n) for r in range(n)]
        bo, bl = K.blockwise_attention(q, k, v, n, causal, "zigzag", 2, pairs=pairs)
        assert np.max(np.abs(bo - out)) < TOL
        assert np.max(np.abs(bl - lse)) < TOL


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
def test_block_count_invariance(n):
    q, k, v = small(1, 128, 2, 2, 8, seed=9)
    out, lse = F.full_attention(q, k, v, True, 1)
    for partition in ("contiguous", "zigzag"):
        for order in ("ring", "tokenring"):
            bo, bl = K.blockwise_attention(q, k, v, n, True, partition, 1, order)
            assert np.max(np.abs(bo - out)) < TOL
            assert np.max(np.abs(bl - lse)) < TOL


def test_merge_partials_matches_union_softmax():
    # k partials from disjoint key sets, merged left to right, equal the softmax
    # over the union (full attention over all keys, non-causal).
    q, k, v = small(1, 8, 1, 1, 4, seed=11)
    kk = np.concatenate([k] * 2, axis=1)
    vv = np.concatenate([v, -v], axis=1)
    S = 16
    out, lse = F.full_attention(np.repeat(q[:, :1], S, axis=1), kk, vv, False, 1)
    outs, lses = [], []
    pos = np.arange(S)
    for j in range(4):
        ks = slice(4 * j, 4 * j + 4)
        bo, bl = K.block_partial(np.repeat(q[:, :1], S, axis=1), kk[:, ks], vv[:, ks], pos, pos[ks], False)
        outs.append(bo)
        lses.append(bl)
    mo, ml = K.merge_partials(outs, lses)
    assert np.max(np.abs(mo - out)) < TOL
    assert np.max(np.abs(ml - lse)) < TOL


# ------------------------------------------------------------------ zigzag

def test_zigzag_worked_example():
    # S = 8, n = 2, c = 2: block 0 = chunk 0 (tokens 0,1) + chunk 3 (6,7);
    # block 1 = chunk 1 (2,3) + chunk 2 (4,5).
    assert K.zigzag_perm(8, 2).tolist() == [0, 1, 6, 7, 2, 3, 4, 5]


@pytest.mark.parametrize("S,n", [(8, 2), (4096, 4), (24000, 4), (1048576, 8), (48, 6)])
def test_zigzag_is_bijection(S, n):
    p = K.zigzag_perm(S, n)
    assert np.array_equal(np.sort(p), np.arange(S))
    x = np.arange(S)[None, :] * 3 + 1
    assert np.array_equal(K.permute_rows(K.permute_rows(x, p), p, inverse=True), x)


def test_zigzag_rejects_ragged():
    with pytest.raises(ValueError):
        K.zigzag_perm(100, 3)


@pytest.mark.parametrize("S,n", [(4096, 4), (24000, 4), (1048576, 8), (8, 2)])
def test_zigzag_balance_invariant(S, n):
    # Every block sees 2n*c^2 + c causal pairs; they add up to S(S+1)/2.
    c = S // (2 * n)
    per = K.visible_pairs_per_block(S, n, "zigzag")
    assert np.all(per == 2 * n * c * c + c)
    assert per.sum() == S * (S + 1) // 2
    if (S, n) == (4096, 4):
        assert per[0] == 2_097_664


def test_contiguous_is_unbalanced():
    per = K.visible_pairs_per_block(4096, 4, "contiguous")
    assert per[0] < per[-1]
    assert per.sum() == 4096 * 4097 // 2


# ---------------------------------------------------------------- schedules

@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_schedules_cover_every_pair_once(n):
    for order in ("ring", "tokenring"):
        steps = K.schedule(n, order)
        assert len(steps) == n
        flat = [p for s in steps for p in s]
        assert sorted(flat) == [(a, b) for a in range(n) for b in range(n)]
        for s in steps:  # each step keeps every rank busy exactly once
            assert sorted(q for q, _ in s) == list(range(n))
            assert sorted(kv for _, kv in s) == list(range(n))


def test_schedule_first_steps():
    assert K.ring_schedule(4)[1] == [(0, 3), (1, 0), (2, 1), (3, 2)]
    assert K.tokenring_schedule(4)[0] == [(0, 0), (1, 1), (2, 2), (3, 3)]
    assert K.tokenring_schedule(4)[1] == [(3, 0), (0, 1), (1, 2), (2, 3)]


# ------------------------------------------------------ planted mistakes

def _mutant_merges():
    def wrong_sigma_sign(out, lse, bo, bl):
        w = K.sigmoid(lse - bl)
        return out - w[..., None] * (out - bo), lse - K.log_sigmoid(lse - bl)

    def wrong_lse_arg(out, lse, bo, bl):
        w = K.sigmoid(bl - lse)
        return out - w[..., None] * (out - bo), lse - K.log_sigmoid(bl - lse)

    def dropped_lse_term(out, lse, bo, bl):
        w = K.sigmoid(bl - lse)
        return out - w[..., None] * (out - bo), np.maximum(lse, bl)

    def swapped_out_operands(out, lse, bo, bl):
        w = K.sigmoid(bl - lse)
        return bo - w[..., None] * (bo - out), lse - K.log_sigmoid(lse - bl)

    return [wrong_sigma_sign, wrong_lse_arg, dropped_lse_term, swapped_out_operands]


@pytest.mark.parametrize("mutant", _mutant_merges(), ids=lambda f: f.__name__)
def test_identity_pin_catches_merge_mutants(mutant, monkeypatch):
    q, k, v = small(1, 32, 1, 1, 8, seed=13)
    out, lse = F.full_attention(q, k, v, False, 1)

    def guarded(o, l, bo, bl):  # keep the -inf bootstrap, mutate the finite case
        fin = np.isfinite(l)
        mo, ml = mutant(o, np.where(fin, l, 0.0), bo, bl)
        return np.where(fin[..., None], mo, bo), np.where(fin, ml, bl)

    monkeypatch.setattr(K, "merge_rule", guarded)
    bo, bl = K.blockwise_attention(q, k, v, 4, False, "contiguous", 1)
    assert max(np.max(np.abs(bo - out)), np.max(np.abs(bl - lse))) > 1e-6


def _planted_full_attention(q, k, v, causal, groups, mistake=None):
    """A copy of the oracle's full attention, step for step, with one planted
    mistake: "transposed" (scores from k against q), "unscaled" (the 1/sqrt(D)
    dropped), "strict_mask" (causal keeps j < i instead of j <= i) or
    "wrong_group" (query head h reads KV head h % Hkv instead of h // groups).
    With mistake=None it is the oracle's computation."""
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    scale = 1.0 if mistake == "unscaled" else 1.0 / math.sqrt(D)
    out = np.zeros((B, S, Hq, D))
    lse = np.zeros((B, S, Hq))
    for b in range(B):
        for h in range(Hq):
            g = h % Hkv if mistake == "wrong_group" else h // groups
            kk, vv, qq = k[b, :, g, :], v[b, :, g, :], q[b, :, h, :]
            s = (kk @ qq.T if mistake == "transposed" else qq @ kk.T) * scale
            if causal:
                rows, cols = np.arange(S)[:, None], np.arange(S)[None, :]
                keep = cols < rows if mistake == "strict_mask" else cols <= rows
                s = np.where(keep, s, -np.inf)
            with np.errstate(invalid="ignore"):
                m = s.max(axis=1, keepdims=True)
                e = np.exp(s - m)
                tot = e.sum(axis=1, keepdims=True)
                lse[b, :, h] = (m + np.log(tot))[:, 0]
                out[b, :, h, :] = (e / tot) @ vv
    return out, lse


def _pin_holds(got, ref):
    """The brute-force pin's test; NaN (a row left with no key) fails it."""
    return bool(np.max(np.abs(got[0] - ref[0])) < TOL and np.max(np.abs(got[1] - ref[1])) < TOL)


@pytest.mark.parametrize("mistake", [None, "transposed", "unscaled", "strict_mask", "wrong_group"])
def test_brute_force_pin_catches_planted_mistakes(mistake):
    # D = 8 (so a dropped 1/sqrt(D) is not a factor a test input could hide),
    # 4 query heads over 2 KV heads (so the head grouping matters), causal.
    q, k, v = small(1, 10, 4, 2, 8, seed=17)
    ref = brute_attention(q, k, v, True, 2)
    got = _planted_full_attention(q, k, v, True, 2, mistake)
    if mistake is None:
        assert _pin_holds(got, ref)  # the copy itself is faithful
        assert _pin_holds(got, F.full_attention(q, k, v, True, 2))
    else:
        assert not _pin_holds(got, ref), mistake


def test_strict_mask_changes_every_causal_row():
    # The off-by-one mask is caught on every row, not only the first (row 0
    # is left with no key at all; any later row loses its diagonal term).
    q, k, v = small(1, 8, 1, 1, 4, seed=19)
    bo, bl = brute_attention(q, k, v, True, 1)
    po, pl = _planted_full_attention(q, k, v, True, 1, "strict_mask")
    with np.errstate(invalid="ignore"):
        for i in range(1, 8):
            assert abs(pl[0, i, 0] - bl[0, i, 0]) > 1e-6, i
    assert not np.isfinite(pl[0, 0, 0])


# --------------------------------------------------------- decode (KV cache)

@pytest.mark.parametrize("causal", [False, True])
def test_decode_equals_last_rows_of_full_attention(causal):
    # the decode queries are the last Tq tokens: same rows of full attention
    B, S, Hq, Hkv, D, Tq = 2, 80, 4, 2, 16, 7
    q, k, v = small(B, S, Hq, Hkv, D, seed=21)
    fo, fl = F.full_attention(q, k, v, causal, 2, row_chunk=16)
    do, dl = F.decode_attention(q[:, S - Tq:], k, v, causal, 2)
    assert np.max(np.abs(do - fo[:, S - Tq:])) < TOL
    assert np.max(np.abs(dl - fl[:, S - Tq:])) < TOL


def test_decode_single_token_brute_force():
    B, S, Hq, D = 1, 9, 2, 4
    q, k, v = small(B, S, Hq, Hq, D, seed=23)
    bo, bl = brute_attention(q, k, v, True, 1)
    do, dl = F.decode_attention(q[:, -1:], k, v, True, 1)
    assert np.max(np.abs(do[:, 0] - bo[:, -1])) < TOL
    assert np.max(np.abs(dl[:, 0] - bl[:, -1])) < TOL


@pytest.mark.parametrize("n_splits", [1, 2, 3, 7, 16])
@pytest.mark.parametrize("causal", [False, True])
def test_decode_blockwise_equals_decode(n_splits, causal):
    B, S, Hq, Hkv, D, Tq = 1, 100, 4, 1, 8, 5
    q, k, v = small(B, S, Hq, Hkv, D, seed=25)
    ro, rl = F.decode_attention(q[:, -Tq:], k, v, causal, 4)
    bo, bl = K.decode_blockwise(q[:, -Tq:], k, v, causal, 4, n_splits)
    assert np.max(np.abs(bo - ro)) < TOL
    assert np.max(np.abs(bl - rl)) < TOL


def test_kv_splits_cover_the_cache():
    for Skv, n in [(100, 3), (4096, 16), (7, 16), (10000, 7)]:
        sp = K.kv_splits(Skv, n)
        assert sp[0][0] == 0 and sp[-1][1] == Skv
        assert all(a1 == b0 for (_, a1), (b0, _) in zip(sp, sp[1:]))


# ---------------------------------------------------------------- backward

from oracle import backward as G  # noqa: E402


def autograd_backward(q, k, v, dout, causal, groups):
    """torch's scaled-dot-product attention in fp64, differentiated by autograd."""
    qt, kt, vt = (torch.as_tensor(np.asarray(x, dtype=np.float64)).permute(0, 2, 1, 3).clone().requires_grad_(True)
                  for x in (q, k, v))
    kr = kt.repeat_interleave(groups, dim=1)
    vr = vt.repeat_interleave(groups, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kr, vr, is_causal=causal)
    o.backward(torch.as_tensor(np.asarray(dout, dtype=np.float64)).permute(0, 2, 1, 3))
    return tuple(t.grad.permute(0, 2, 1, 3).numpy() for t in (qt, kt, vt))


def rand64(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("groups", [1, 2])
def test_backward_matches_autograd(causal, groups):
    B, S, Hq, D = 2, 40, 4, 16
    q, do = rand64((B, S, Hq, D), 1), rand64((B, S, Hq, D), 2)
    k, v = rand64((B, S, Hq // groups, D), 3), rand64((B, S, Hq // groups, D), 4)
    got = G.attention_backward(q, k, v, do, causal, groups)
    ref = autograd_backward(q, k, v, do, causal, groups)
    for a, r, nm in zip(got, ref, "qkv"):
        assert np.max(np.abs(a - r)) <= 1e-10 * max(1.0, np.max(np.abs(r))), nm


def test_backward_finite_differences():
    # central differences of L = sum(dO * O) on a tiny problem
    B, S, Hq, Hkv, D = 1, 5, 2, 1, 3
    q, k, v = rand64((B, S, Hq, D), 5), rand64((B, S, Hkv, D), 6), rand64((B, S, Hkv, D), 7)
    do = rand64((B, S, Hq, D), 8)
    dq, dk, dv = G.attention_backward(q, k, v, do, True, 2)

    def loss(qq, kk, vv):
        o, _ = F.full_attention(qq, kk, vv, True, 2)
        return float(np.sum(do * o))

    eps = 1e-6
    for x, g in ((q, dq), (k, dk), (v, dv)):
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [xp if x is y else y for y in (q, k, v)]
            args_m = [xm if x is y else y for y in (q, k, v)]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - g[idx]) <= 1e-6, (idx, fd, g[idx])


def test_backward_closed_forms():
    B, S, Hq, Hkv, D = 1, 24, 4, 2, 8
    q, k, v = rand64((B, S, Hq, D), 9), rand64((B, S, Hkv, D), 10), rand64((B, S, Hkv, D), 11)
    # no upstream gradient, no gradient
    for gr in G.attention_backward(q, k, v, np.zeros((B, S, Hq, D)), True, 2):
        assert np.all(gr == 0.0)
    do = rand64((B, S, Hq, D), 12)
    dq, dk, dv = G.attention_backward(q, k, v, do, True, 2)
    # softmax rows sum to one: the keys' dV adds up to the queries' dO of the group
    assert np.allclose(dv.sum(axis=1), do.reshape(B, S, Hkv, 2, D).sum(axis=(1, 3)), atol=1e-12)
    # every dS row sums to zero: the keys' dK adds up to zero
    assert np.allclose(dk.sum(axis=1), 0.0, atol=1e-12)


@pytest.mark.parametrize("partition,n", [("contiguous", 1), ("contiguous", 4), ("zigzag", 2), ("zigzag", 4)])
@pytest.mark.parametrize("causal", [True, False])
def test_blockwise_backward_equals_full(partition, n, causal):
    B, S, Hq, Hkv, D = 2, 64, 4, 2, 8
    q, k, v = attention_inputs(B, S, Hq, Hkv, D, "f32", seed=13)
    do = torch.as_tensor(rand64((B, S, Hq, D), 14))
    o, lse = F.full_attention(q, k, v, causal, 2)
    ref = G.attention_backward(q, k, v, do, causal, 2)
    got = G.blockwise_backward(q, k, v, do, o, lse, n, causal, partition, 2)
    for a, r in zip(got, ref):
        assert np.max(np.abs(a - r)) <= TOL * max(1.0, np.max(np.abs(r)))


def _backward_mutant(kind):
    """A copy of the definition with one plausible mistake planted."""
    def f(q, k, v, dout, causal, groups):
        q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dout))
        B, S, Hq, D = q.shape
        s = 1.0 / math.sqrt(D)
        dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        mask = np.tril(np.ones((S, S), dtype=bool)) if causal else np.ones((S, S), dtype=bool)
        for b in range(B):
            for h in range(Hq):
                g = h // groups
                lg = np.where(mask, (q[b, :, h] @ k[b, :, g].T) * s, -np.inf)
                e = np.exp(lg - lg.max(axis=1, keepdims=True))
                p = e / e.sum(axis=1, keepdims=True)
                o = p @ v[b, :, g]
                dv[b, :, g] += p.T @ do[b, :, h]
                dp = do[b, :, h] @ v[b, :, g].T
                delta = 0.0 if kind == "no_delta" else (do[b, :, h] * o).sum(axis=1, keepdims=True)
                ds = p * (dp - delta)
                dq[b, :, h] = (1.0 if kind == "no_scale" else s) * (ds @ k[b, :, g])
                dk[b, :, g] += s * ((ds if kind == "ds_not_transposed" else ds.T) @ q[b, :, h])
        return dq, dk, dv
    return f


@pytest.mark.parametrize("kind", ["no_delta", "no_scale", "ds_not_transposed"])
def test_backward_pins_catch_planted_mistakes(kind):
    B, S, Hq, D = 1, 16, 2, 16
    q, do = rand64((B, S, Hq, D), 15), rand64((B, S, Hq, D), 16)
    k, v = rand64((B, S, Hq, D), 17), rand64((B, S, Hq, D), 18)
    ref = autograd_backward(q, k, v, do, True, 1)
    got = _backward_mutant(kind)(q, k, v, do, True, 1)
    assert any(np.max(np.abs(a - r)) > 1e-6 for a, r in zip(got, ref))
    good = _backward_mutant("none")(q, k, v, do, True, 1)
    assert all(np.max(np.abs(a - r)) <= 1e-10 for a, r in zip(good, ref))


@pytest.mark.parametrize("causal", [True, False])
def test_backward_rows_match_autograd(causal):
    B, S, Hq, Hkv, D = 2, 30, 4, 2, 8
    q, do = rand64((B, S, Hq, D), 19), rand64((B, S, Hq, D), 20)
    k, v = rand64((B, S, Hkv, D), 21), rand64((B, S, Hkv, D), 22)
    dq, dk, dv = autograd_backward(q, k, v, do, causal, 2)
    rows = [(0, 0, 0), (1, 7, 3), (0, 29, 1), (1, 15, 2)]
    got = G.backward_query_rows(q, k, v, do, rows, causal, 2)
    for n, (b, i, h) in enumerate(rows):
        assert np.max(np.abs(got[n] - dq[b, i, h])) <= 1e-10
    keys = [(0, 0, 0), (1, 29, 1), (0, 13, 1), (1, 28, 0)]
    gk, gv = G.backward_key_rows(q, k, v, do, keys, causal, 2)
    for n, (b, j, g) in enumerate(keys):
        assert np.max(np.abs(gk[n] - dk[b, j, g])) <= 1e-10
        assert np.max(np.abs(gv[n] - dv[b, j, g])) <= 1e-10
