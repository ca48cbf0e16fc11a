"""Closed-form pin: the oracle's visibility count reproduces the README's
analytic KV-cache figures ("mSeek" README, section "Results").

The cache stores, per LBCA layer and kv head, the P(T) pooled entries a query
at the end of a T-token context can see plus the raw tokens from P(T)*m on.
Only the block-aligned partition reading gives exactly 304,343 tokens in the
154,624-dense-token budget; the literal "every completed block plus the last w
tokens" reading gives 304,365.
"""
import json
import os

import pytest

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "cache_accounting.json")))
M = GOLD["model"]


def _bytes(orc, T, m):
    return orc.kv_cache_bytes(T, M["n_layers"], M["n_lbca_layers"], m, M["n_win"],
                              M["n_kv_heads"], M["head_dim"], M["elt_bytes"])


def _dense(orc, T):
    return orc.kv_cache_bytes(T, M["n_layers"], 0, 64, M["n_win"], M["n_kv_heads"], M["head_dim"],
                              M["elt_bytes"])


def test_cache_at_128k(orc):
    T = 131072
    assert round(_dense(orc, T) / 2**30, GOLD["gib_decimals"]) == GOLD["dense_gib_128k"]
    assert round(_bytes(orc, T, 64) / 2**30, GOLD["gib_decimals"]) == GOLD["lbca_gib_128k"]


def test_reduction_percentages(orc):
    tol = GOLD["reduction_tolerance"]
    r4k = 1 - _bytes(orc, 4096, 16) / _dense(orc, 4096)
    assert abs(r4k - GOLD["reduction_4k_m16"]) <= tol
    for T in (16384, 32768, 65536, 131072):
        r = 1 - _bytes(orc, T, 64) / _dense(orc, T)
        assert abs(r - GOLD["reduction_from_16k_m64"]) <= tol


def test_capacity_in_dense_budget(orc):
    budget = _dense(orc, GOLD["dense_tokens_in_budget"])
    want = GOLD["lbca_tokens_in_budget"]
    assert _bytes(orc, want, 64) <= budget
    # the largest fitting context: every longer one up to two blocks further exceeds the budget
    assert all(_bytes(orc, T, 64) > budget for T in range(want + 1, want + 2 * 64 + M["n_win"]))
    assert round(want / GOLD["dense_tokens_in_budget"], 2) == GOLD["capacity_ratio"]


@pytest.mark.parametrize("L,m,w,P", [(0, 4, 0, 0), (3, 4, 0, 0), (4, 4, 0, 1), (10, 4, 3, 1),
                                     (11, 4, 3, 2), (128, 64, 128, 0), (191, 64, 128, 0),
                                     (192, 64, 128, 1), (32769, 64, 128, 510), (131073, 128, 128, 1023)])
def test_visible_block_counts(orc, L, m, w, P):
    """P(L) = max(0, floor((L - w)/m)); raw visible tokens L - P*m lie in
    [min(L, w), w + m - 1]."""
    assert orc.visible_blocks(L, m, w) == P
    raw = L - P * m
    assert min(L, w) <= raw <= max(w + m - 1, 0) or L == 0
