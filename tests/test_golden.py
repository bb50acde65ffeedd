"""Hand-derived worked examples (tests/golden/) against the oracle.

Each fixture states the passage it follows and how its expected values were
derived by hand (closed forms such as ln 5 or (v0 + e^3 v1) / (1 + e^3));
none of them comes from the oracle or from the CUDA path.  The oracle's
update rule, its full attention and its blockwise path, and its zigzag
permutation must reproduce them to fp64 rounding.
"""
import json
import os

import numpy as np
import pytest

from oracle import attention as F
from oracle import blockwise as K

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def num(x):
    """Fixture number: a float, or the string '-inf'."""
    if isinstance(x, str):
        assert x == "-inf", x
        return float("-inf")
    return float(x)


def arr(x):
    return np.array(x, dtype=np.float64)


MERGE = load("merge_rule_worked.json")
ATT = load("attention_worked.json")
PERM = load("zigzag_perm.json")


@pytest.mark.parametrize("case", MERGE["cases"], ids=lambda c: c["name"])
def test_merge_rule_worked_examples(case):
    out, lse = K.merge_rule(arr(case["out"]), num(case["lse"]), arr(case["block_out"]), num(case["block_lse"]))
    want_lse = num(case["expect_lse"])
    if np.isneginf(want_lse):
        assert np.isneginf(lse)
    else:
        assert abs(float(lse) - want_lse) <= 1e-15 * max(1.0, abs(want_lse))
    np.testing.assert_allclose(out, arr(case["expect_out"]), rtol=0, atol=1e-15)


@pytest.mark.parametrize("causal", [True, False])
def test_full_attention_worked_example(causal):
    q, k, v = arr(ATT["q"])[None], arr(ATT["k"])[None], arr(ATT["v"])[None]
    want = ATT["causal" if causal else "full"]
    out, lse = F.full_attention(q, k, v, causal, gqa_groups=2)
    np.testing.assert_allclose(out[0], arr(want["out"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0], arr(want["lse"]), rtol=0, atol=1e-14)


@pytest.mark.parametrize("order", ["ring", "tokenring"])
@pytest.mark.parametrize("causal", [True, False])
def test_blockwise_path_worked_example(causal, order):
    # two one-token blocks: every row's result is stitched from two partials
    # by the update rule (or one, where the causal mask empties a pair)
    q, k, v = arr(ATT["q"])[None], arr(ATT["k"])[None], arr(ATT["v"])[None]
    want = ATT["causal" if causal else "full"]
    out, lse = K.blockwise_attention(q, k, v, 2, causal, "contiguous", gqa_groups=2, order=order)
    np.testing.assert_allclose(out[0], arr(want["out"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0], arr(want["lse"]), rtol=0, atol=1e-14)


@pytest.mark.parametrize("case", PERM["cases"], ids=lambda c: f"S{c['S']}n{c['n']}")
def test_zigzag_permutation_worked_examples(case):
    perm = K.zigzag_perm(case["S"], case["n"])
    assert perm.tolist() == case["perm"]
