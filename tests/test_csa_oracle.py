"""Pins of the CSA part of the fp64 oracle, on the CPU (no GPU needed).

The CSA form (CSA page, "What is implemented") adds three steps to the
block-compressed path: dual overlapped pooling (Eqs 9-12), the lightning
indexer's relevance and top-k block selection (Eqs 13-17), and shared-KV core
attention over the selected entries plus an overlapping raw window and the
sink (Eqs 18-19, Eq 27).  Each oracle function is checked against the NumPy
brute force and against closed forms or special cases that reduce to the
already-pinned single-series pooling and attention, chosen so that a
plausible slip (two separate softmaxes instead of one joint softmax, the
wrong preceding block, a dropped ReLU or head weight, a window that starts at
the wrong token, a selection that sees incomplete blocks) fails at least one.
"""
import numpy as np
import pytest

from oracle import brute
from oracle import oracle as orc


def _rng(seed):
    return np.random.default_rng(seed)


def _series(rng, B, T, G, D, m):
    xa, za, xb, zb = (rng.standard_normal((B, T, G, D)) for _ in range(4))
    bpa, bpb = (0.3 * rng.standard_normal((m, G * D)) for _ in range(2))
    return xa, za, xb, zb, bpa, bpb


def _cfg(**kw):
    base = dict(n_q_heads=4, n_kv_heads=1, head_dim=16, shared_kv=True, block_m=4, n_win=8, rope_dims=8,
                rmsnorm=True)
    base.update(kw)
    return orc.Config(**base)


# ------------------------------------------------------------- dual pooling ----
@pytest.mark.parametrize("m,T,G", [(4, 4 * 7 + 3, 1), (1, 9, 2), (3, 3 * 5, 2), (8, 8 * 3 + 7, 1)])
def test_pool_dual_matches_brute_force(orc, m, T, G):
    rng = _rng(1)
    c = _cfg(n_kv_heads=G, n_q_heads=2 * G, block_m=m, rmsnorm=False, rope_dims=0)
    xa, za, xb, zb, bpa, bpb = _series(rng, 2, T, G, 16, m)
    got = orc.pool_dual(c, orc.VALUE, xa, za, xb, zb, bpa, bpb)
    for b in range(2):
        want = brute.pool_dual_series(xa[b], za[b], xb[b], zb[b], bpa, bpb, m)
        np.testing.assert_allclose(got[b], want, rtol=0, atol=1e-12)


def test_pool_dual_key_series_is_finalised_at_the_block_start(orc):
    rng = _rng(2)
    m, T, D = 4, 4 * 6, 16
    c = _cfg(block_m=m)
    xa, za, xb, zb, bpa, bpb = _series(rng, 1, T, 1, D, m)
    g = 1 + 0.1 * rng.standard_normal(D)
    got = orc.pool_dual(c, orc.KEY, xa, za, xb, zb, bpa, bpb, gamma=g)[0, :, 0]
    raw = brute.pool_dual_series(xa[0], za[0], xb[0], zb[0], bpa, bpb, m)[:, 0]
    want = brute._rot(brute._rms(raw, g, c.rms_eps), np.arange(T // m) * m, c.rope_dims, c.rope_theta)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_pool_dual_without_the_b_series_is_single_series_pooling(orc):
    """b-series logits at -1e30: every entry pools its own block alone, which
    is the (separately pinned) single-series pooling of the a-series."""
    rng = _rng(3)
    m, T, G, D = 4, 4 * 5 + 2, 2, 16
    c = _cfg(n_kv_heads=G, n_q_heads=4, block_m=m)
    xa, za, xb, _, bpa, bpb = _series(rng, 2, T, G, D, m)
    zb = np.full_like(za, -1e30)
    got = orc.pool_dual(c, orc.KEY, xa, za, xb, zb, bpa, bpb)
    want = orc.pool(c, orc.KEY, xa, za, bpa)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_pool_dual_first_entry_has_no_preceding_block(orc):
    rng = _rng(4)
    m, T = 4, 16
    c = _cfg(block_m=m, rmsnorm=False, rope_dims=0)
    xa, za, xb, zb, bpa, bpb = _series(rng, 1, T, 1, 16, m)
    got = orc.pool_dual(c, orc.VALUE, xa, za, xb, zb, bpa, bpb)[0, 0]
    want = orc.pool(c, orc.VALUE, xa[:, :m], za[:, :m], bpa)[0, 0]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_pool_dual_uniform_logits_give_the_mean_of_both_blocks(orc):
    rng = _rng(5)
    m, T = 4, 4 * 4
    c = _cfg(block_m=m, rmsnorm=False, rope_dims=0)
    xa, _, xb, _, _, _ = _series(rng, 1, T, 1, 16, m)
    z = np.full_like(xa, 0.7)
    zero = np.zeros((m, 16))
    got = orc.pool_dual(c, orc.VALUE, xa, z, xb, z, zero, zero)[0, :, 0]
    for i in range(1, T // m):
        want = (xa[0, i * m:(i + 1) * m, 0].sum(0) + xb[0, (i - 1) * m:i * m, 0].sum(0)) / (2 * m)
        np.testing.assert_allclose(got[i], want, rtol=0, atol=1e-12)


def test_pool_dual_one_softmax_over_both_series(orc):
    """Raising every a-series logit of an entry by c multiplies the a-series
    share of the weight by e^c relative to the b-series: with one joint
    softmax the entry moves to (e^c A + B) / (e^c Sa + Sb); two separate
    softmaxes would not move at all."""
    rng = _rng(6)
    m, T = 4, 4 * 3
    c = _cfg(block_m=m, rmsnorm=False, rope_dims=0)
    xa, za, xb, zb, bpa, bpb = _series(rng, 1, T, 1, 16, m)
    base = orc.pool_dual(c, orc.VALUE, xa, za, xb, zb, bpa, bpb)[0, :, 0]
    cc = 1.3
    moved = orc.pool_dual(c, orc.VALUE, xa, za + cc, xb, zb, bpa, bpb)[0, :, 0]
    i = 2
    la = za[0, i * m:(i + 1) * m, 0] + bpa
    lb = zb[0, (i - 1) * m:i * m, 0] + bpb
    ea, eb = np.exp(la), np.exp(lb)
    A = (ea * xa[0, i * m:(i + 1) * m, 0]).sum(0)
    Bv = (eb * xb[0, (i - 1) * m:i * m, 0]).sum(0)
    np.testing.assert_allclose(base[i], (A + Bv) / (ea.sum(0) + eb.sum(0)), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(moved[i], (np.exp(cc) * A + Bv) / (np.exp(cc) * ea.sum(0) + eb.sum(0)),
                               rtol=1e-12, atol=1e-12)
    assert np.abs(moved[i] - base[i]).max() > 1e-3
    # a common shift of both series' logits changes nothing
    same = orc.pool_dual(c, orc.VALUE, xa, za + cc, xb, zb + cc, bpa, bpb)[0, :, 0]
    np.testing.assert_allclose(same, base, rtol=0, atol=1e-12)


def test_pool_dual_one_hot_b_logit_selects_the_preceding_block_token(orc):
    rng = _rng(7)
    m, T, i, r = 4, 4 * 5, 3, 2
    c = _cfg(block_m=m, rmsnorm=False, rope_dims=0)
    xa, za, xb, zb, bpa, bpb = _series(rng, 1, T, 1, 16, m)
    zb = zb.copy()
    zb[0, (i - 1) * m + r] = 200.0
    got = orc.pool_dual(c, orc.VALUE, xa, za, xb, zb, bpa, bpb)[0, i, 0]
    np.testing.assert_allclose(got, xb[0, (i - 1) * m + r, 0], rtol=0, atol=1e-12)


def test_pool_dual_is_a_convex_combination(orc):
    rng = _rng(8)
    m, T = 4, 4 * 6
    c = _cfg(block_m=m, rmsnorm=False, rope_dims=0)
    xa, za, xb, zb, bpa, bpb = _series(rng, 1, T, 1, 16, m)
    got = orc.pool_dual(c, orc.VALUE, xa, za, xb, zb, bpa, bpb)[0, :, 0]
    for i in range(1, T // m):
        vals = np.concatenate([xa[0, i * m:(i + 1) * m, 0], xb[0, (i - 1) * m:i * m, 0]])
        assert np.all(got[i] <= vals.max(0) + 1e-12) and np.all(got[i] >= vals.min(0) - 1e-12)


# ---------------------------------------------------------------- indexer ----
def test_indexer_matches_brute_force(orc):
    rng = _rng(9)
    B, NB, HI, DI = 3, 20, 5, 8
    q, kx = rng.standard_normal((B, HI, DI)), rng.standard_normal((B, NB, DI))
    w = rng.standard_normal((B, HI))
    nvis = np.array([0, 7, 20])
    got = orc.indexer_scores(q, w, kx, nvis)
    for b in range(B):
        n = int(nvis[b])
        np.testing.assert_allclose(got[b, :n], brute.indexer(q[b], w[b], kx[b], n), rtol=0, atol=1e-12)


def test_indexer_masks_the_blocks_a_query_cannot_see(orc):
    """Entry j of a query that sees n complete blocks is finite for j < n and
    -inf from n on (n = 0: every entry masked; n = NB: none)."""
    rng = _rng(12)
    B, NB, HI, DI = 4, 9, 3, 5
    q, kx, w = rng.standard_normal((B, HI, DI)), rng.standard_normal((B, NB, DI)), rng.standard_normal((B, HI))
    nvis = np.array([0, 1, 6, NB])
    got = orc.indexer_scores(q, w, kx, nvis)
    for b in range(B):
        n = int(nvis[b])
        assert np.all(np.isfinite(got[b, :n])) and np.all(np.isneginf(got[b, n:])), (b, n)


def test_indexer_relu_closed_forms(orc):
    """ReLU(x) - ReLU(-x) = x: I(q) - I(-q) = sum_h w_h q_h . k_j exactly; one
    head with weight 1 gives ReLU(q . k_j); scores are linear in w."""
    rng = _rng(10)
    B, NB, HI, DI = 2, 11, 4, 6
    q, kx, w = rng.standard_normal((B, HI, DI)), rng.standard_normal((B, NB, DI)), rng.standard_normal((B, HI))
    nv = np.full(B, NB)
    diff = orc.indexer_scores(q, w, kx, nv) - orc.indexer_scores(-q, w, kx, nv)
    np.testing.assert_allclose(diff, np.einsum("bh,bhd,bjd->bj", w, q, kx), rtol=0, atol=1e-12)
    one = orc.indexer_scores(q[:, :1], np.ones((B, 1)), kx, nv)
    np.testing.assert_allclose(one, np.maximum(np.einsum("bd,bjd->bj", q[:, 0], kx), 0), rtol=0, atol=1e-12)
    w2 = rng.standard_normal((B, HI))
    lin = orc.indexer_scores(q, 2 * w - 3 * w2, kx, nv)
    np.testing.assert_allclose(lin, 2 * orc.indexer_scores(q, w, kx, nv) - 3 * orc.indexer_scores(q, w2, kx, nv),
                               rtol=0, atol=1e-10)


def test_topk_selects_the_highest_visible_blocks(orc):
    rng = _rng(11)
    scores = rng.standard_normal((3, 30))
    nvis = np.array([30, 5, 0])
    got = orc.topk_blocks(scores, nvis, 8)
    assert got[0].tolist() == brute.topk(list(scores[0]), 8)
    assert sorted(got[1, :5].tolist()) == list(range(5)) and got[1, 5:].tolist() == [-1] * 3
    assert got[2].tolist() == [-1] * 8
    tied = np.zeros((1, 6))
    assert orc.topk_blocks(tied, [6], 3)[0].tolist() == [0, 1, 2]


def test_complete_blocks_only():
    assert orc.complete_blocks(15, 4) == 3 and orc.complete_blocks(16, 4) == 4 and orc.complete_blocks(3, 4) == 0


# -------------------------------------------------------- sparse attention ----
def _csa_inputs(rng, T, D=16, m=4):
    c_hist = rng.standard_normal((1, T, 1, D))
    z = rng.standard_normal((1, T, 1, D))
    xb, zb = rng.standard_normal((1, T, 1, D)), rng.standard_normal((1, T, 1, D))
    bpa, bpb = 0.3 * rng.standard_normal((m, D)), 0.3 * rng.standard_normal((m, D))
    return c_hist, z, xb, zb, bpa, bpb


@pytest.mark.parametrize("L,w,sel", [(23, 8, [3, 0, -1, 4]), (40, 5, [9, 2, 7]), (6, 16, [0]), (12, 3, [])])
def test_attend_sparse_matches_brute_force(orc, L, w, sel):
    rng = _rng(12)
    D, m = 16, 4
    c = _cfg(n_win=w)
    c_hist, z, xb, zb, bpa, bpb = _csa_inputs(rng, L, D, m)
    ek = orc.pool_dual(c, orc.KEY, c_hist, z, xb, zb, bpa, bpb)
    q = rng.standard_normal((1, 4, D))
    sink = rng.standard_normal(4)
    gq, gk = 1 + 0.1 * rng.standard_normal(D), 1 + 0.1 * rng.standard_normal(D)
    selv = np.array([sel], dtype=np.int64).reshape(1, len(sel))
    got = orc.attend_sparse(c, q, ek, selv, c_hist, [L], sink, gq, gk)[0]
    want = brute.attention_sparse(q[0], ek[0, :, 0], sel, c_hist[0, :, 0], L - 1, w=w, rope_dims=c.rope_dims,
                                  rmsnorm=True, eps=c.rms_eps, sink=sink, gamma_q=gq, gamma_kv=gk)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_attend_sparse_window_alone_is_causal_attention(orc):
    """No selected entry and a window covering the whole history: causal dense
    attention over the finalised raw tokens, the same as the (pinned)
    block-compressed attention whose window covers everything."""
    rng = _rng(13)
    L, D = 19, 16
    c = _cfg(n_win=64)
    c_hist = rng.standard_normal((1, L, 1, D))
    q = rng.standard_normal((1, 4, D))
    sink = rng.standard_normal(4)
    got = orc.attend_sparse(c, q, None, np.zeros((1, 0), np.int64), c_hist, [L], sink)
    want = orc.attend(c, q[:, None], np.array([[L - 1]]), None, None, c_hist, None, [L], sink)[:, 0]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_attend_sparse_every_block_and_no_window_is_dense_over_entries(orc):
    """All complete blocks selected, no window, L a multiple of m: the same
    visible set as the block-aligned attention with n_win = 0, whose pinned
    oracle then attends exactly the same entries."""
    rng = _rng(14)
    L, D, m = 24, 16, 4
    c = _cfg(n_win=0, block_m=m)
    c_hist, z, xb, zb, bpa, bpb = _csa_inputs(rng, L, D, m)
    ek = orc.pool_dual(c, orc.KEY, c_hist, z, xb, zb, bpa, bpb)
    q = rng.standard_normal((1, 4, D))
    sel = np.arange(L // m)[None]
    got = orc.attend_sparse(c, q, ek, sel, c_hist, [L])
    want = orc.attend(c, q[:, None], np.array([[L - 1]]), ek, None, c_hist, None, [L])[:, 0]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_attend_sparse_selection_order_and_padding_do_not_matter(orc):
    rng = _rng(15)
    L, D = 30, 16
    c = _cfg(n_win=6)
    c_hist, z, xb, zb, bpa, bpb = _csa_inputs(rng, L, D)
    ek = orc.pool_dual(c, orc.KEY, c_hist, z, xb, zb, bpa, bpb)
    q = rng.standard_normal((1, 4, D))
    a = orc.attend_sparse(c, q, ek, np.array([[5, 1, 6]]), c_hist, [L])
    b = orc.attend_sparse(c, q, ek, np.array([[-1, 6, 5, -1, 1]]), c_hist, [L])
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_attend_sparse_single_row_sink_closed_form(orc):
    """One visible row (window of 1, nothing selected): the output is the row
    weighted by sigma(s - sink), rotated back by -t."""
    rng = _rng(16)
    L, D = 9, 16
    c = _cfg(n_win=1, rmsnorm=False, rope_dims=0)
    c_hist = rng.standard_normal((1, L, 1, D))
    q = rng.standard_normal((1, 4, D))
    sink = rng.standard_normal(4)
    got = orc.attend_sparse(c, q, None, np.zeros((1, 0), np.int64), c_hist, [L], sink)[0]
    row = c_hist[0, L - 1, 0]
    s = q[0] @ row / np.sqrt(D)
    want = (1.0 / (1.0 + np.exp(sink - s)))[:, None] * row[None]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
