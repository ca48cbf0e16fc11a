"""The algorithmic work behind every roofline figure, on the CPU.

bench.py divides algorithmic bytes (decode) and FLOPs (prefill) by measured
time.  Both count the visible (query, entry) pairs of the block-aligned
reading ("mSeek" README, "How LBCA works": pooled entries j < P(L), raw tokens
[P m, L)); here they are recounted from the NumPy brute force's visible set,
which finds P by search and checks that the pooled prefix and the raw window
partition the history, so a slip in the closed form (an off-by-one in P, a
raw window counted from the wrong token, a series or a sequence dropped)
shows up as a wrong roofline.
"""
import numpy as np
import pytest

import bench
from block_compressed_long_b200 import synth
from oracle import brute

W = synth.WORKLOADS


def _pairs_by_search(rows, m, w):
    total = 0
    for t in rows:
        P, raw = brute.visible(t + 1, m, w)
        total += P + len(raw)
    return total


@pytest.mark.parametrize("m,w,T", [(1, 0, 7), (1, 5, 9), (4, 0, 19), (4, 3, 23), (5, 16, 40), (16, 128, 100),
                                   (8, 200, 50), (3, 2, 3)])
def test_prefill_pairs_match_the_visible_sets(m, w, T):
    wk = synth.scaled(W["tiny_f32_prefill"], block_m=m, n_win=w, seq_len=T)
    assert bench.prefill_pairs(wk) == _pairs_by_search(range(T), m, w)


def test_tiny_f32_prefill_flops():
    w = W["tiny_f32_prefill"]
    pairs = _pairs_by_search(range(w.seq_len), w.block_m, w.n_win)
    assert bench.prefill_pairs(w) == pairs
    assert bench.prefill_flops(w) == 4.0 * w.head_dim * w.n_q_heads * pairs * w.batch


def test_16k_prefill_pairs_on_sampled_rows():
    w = W["gqa_prefill_16k"]
    rows = np.unique(np.linspace(0, w.seq_len - 1, 97).astype(np.int64)).tolist() + [0, 127, 128, 143, 144]
    for t in rows:
        assert bench.prefill_pairs(w, [t]) == _pairs_by_search([t], w.block_m, w.n_win), t


@pytest.mark.parametrize("name", ["gqa_decode_32k", "hca_mqa_decode_128k", "ragged_gqa_decode_append"])
def test_decode_bytes_match_the_visible_sets(name):
    w = W[name]
    lens = synth.contexts(w)[:4] + 1  # the query sees its own new token
    esize = 2 if w.dtype == "bf16" else 4
    series = 1 if w.shared_kv else 2
    want = 0
    for L in lens:
        P, raw = brute.visible(int(L), w.block_m, w.n_win)
        want += (P + len(raw)) * w.n_kv_heads * w.head_dim * esize * series
    want += 2 * len(lens) * w.n_q_heads * w.head_dim * esize  # queries read, outputs written
    assert bench.bytes_per_decode(w, lens) == want
