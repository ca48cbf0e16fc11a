"""Pins of the fp64 oracle against things other than itself.

Each test fixes part of the oracle by an independent route: the NumPy brute
force (different machinery, same definition), special cases that reduce to a
library routine (torch's scaled_dot_product_attention, torch's rms_norm,
complex multiplication), closed forms and invariants the pages' method must
satisfy ("mSeek" README, "How LBCA works": strict causality and dense-limit
behaviour).  No GPU is used.
"""
import itertools

import numpy as np
import pytest
import torch
from scipy.special import expit

from oracle import brute

RNG = np.random.default_rng(12345)


def _cfg(orc, **kw):
    return orc.Config(**kw)


def _inputs(rng, T, Hq, G, D, m, shared, bstd=0.3):
    q = rng.standard_normal((1, T, Hq, D))
    k = rng.standard_normal((1, T, G, D))
    zk = rng.standard_normal((1, T, G, D))
    bpk = rng.standard_normal((m, G * D)) * bstd
    if shared:
        return q, k, None, zk, None, bpk, None
    v = rng.standard_normal((1, T, G, D))
    zv = rng.standard_normal((1, T, G, D))
    bpv = rng.standard_normal((m, G * D)) * bstd
    return q, k, v, zk, zv, bpk, bpv


def _grid():
    cases = []
    for m in (1, 2, 3, 4, 16):
        for w in sorted({0, 1, max(m - 1, 0), m, 5, 128}):
            for T in (1, 2 * m + 3, 37):
                cases.append((m, w, T))
    return cases


@pytest.mark.parametrize("m,w,T", _grid())
def test_oracle_matches_brute_force(orc, m, w, T):
    """C oracle == NumPy brute force to 1e-12 (fp64), over both kv forms and
    every feature toggle, mirroring the README's float64 equivalence grid."""
    rng = np.random.default_rng(1000 * m + 10 * w + T)
    for shared, rope, rms, sink in itertools.product((False, True), (0, 4, 8), (False, True), (False, True)):
        if not shared and rms and rope == 4:
            continue  # keep the grid small; the other combinations cover it
        Hq, G, D = (4, 1, 8) if shared else (4, 2, 8)
        q, k, v, zk, zv, bpk, bpv = _inputs(rng, T, Hq, G, D, m, shared)
        s = rng.standard_normal(Hq) if sink else None
        gq = 1 + 0.1 * rng.standard_normal(D) if rms else None
        gk = 1 + 0.1 * rng.standard_normal(D) if rms else None
        cfg = _cfg(orc, n_q_heads=Hq, n_kv_heads=G, head_dim=D, shared_kv=shared, block_m=m, n_win=w,
                   rope_dims=rope, rmsnorm=rms, rope_theta=50.0)
        got = orc.forward(cfg, q, k, v, zk, zv, bpk, bpv, s, gq, gk)[0]
        want = brute.attention(q[0], k[0], None if shared else v[0], zk[0], None if shared else zv[0],
                               bpk, bpv, m=m, w=w, shared_kv=shared, rope_dims=rope, theta=50.0,
                               rmsnorm=rms, sink=s, gamma_q=gq, gamma_kv=gk)
        np.testing.assert_allclose(got, want, atol=1e-12, rtol=1e-12)


def test_m1_pooling_is_identity(orc):
    """m = 1: the one-position softmax weight is exactly 1, so pooling returns X."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal((2, 9, 3, 16))
    z = rng.standard_normal(x.shape)
    cfg = _cfg(orc, n_q_heads=3, n_kv_heads=3, head_dim=16, shared_kv=False, block_m=1, n_win=0)
    for bpos in (np.zeros((1, 48)), rng.standard_normal((1, 48))):
        assert np.array_equal(orc.pool(cfg, orc.VALUE, x, z, bpos), x)


def _torch_rope(x, pos, rho, theta):
    """RoPE as complex multiplication with torch.polar (RoFormer's complex form)."""
    if rho == 0:
        return x
    D = x.shape[-1]
    head, tail = x[..., :D - rho], x[..., D - rho:]
    zc = torch.view_as_complex(tail.reshape(*tail.shape[:-1], rho // 2, 2).contiguous())
    freq = theta ** (-torch.arange(rho // 2, dtype=torch.float64) * 2 / rho)
    ang = pos.to(torch.float64)[..., None] * freq
    zc = zc * torch.polar(torch.ones_like(ang), ang)
    return torch.cat([head, torch.view_as_real(zc).reshape(tail.shape)], dim=-1)


def _dense_reference(q, k, v, shared, rope, rms, theta, gq=None, gk=None):
    """Causal dense attention via torch SDPA (fp64 CPU) with the query/key
    treatment applied beforehand and the shared-form output rotation after."""
    q, k = torch.from_numpy(q[0]), torch.from_numpy(k[0])      # [T,H,D]
    T, Hq, D = q.shape
    G = k.shape[1]
    if rms:
        q = torch.nn.functional.rms_norm(q, (D,), torch.from_numpy(gq) if gq is not None else None, 1e-6)
        k = torch.nn.functional.rms_norm(k, (D,), torch.from_numpy(gk) if gk is not None else None, 1e-6)
    pos = torch.arange(T)
    q = _torch_rope(q, pos[:, None].expand(T, Hq), rope, theta)
    k = _torch_rope(k, pos[:, None].expand(T, G), rope, theta)
    val = k if shared else torch.from_numpy(v[0])
    o = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(0, 1), k.transpose(0, 1), val.transpose(0, 1), is_causal=True,
        enable_gqa=True).transpose(0, 1)
    if shared:
        o = _torch_rope(o, -pos[:, None].expand(T, Hq), rope, theta)
    return o.numpy()


@pytest.mark.parametrize("shared,rope,rms", [(False, 0, False), (False, 8, False), (False, 8, True),
                                             (True, 0, False), (True, 4, True), (True, 8, False)])
@pytest.mark.parametrize("w", [0, 3, 100])
def test_m1_reduces_to_causal_dense_attention(orc, shared, rope, rms, w):
    """m = 1 with zero bias: every token is its own pooled entry, so the method
    is causal dense attention for any window (README: dense-limit behaviour)."""
    rng = np.random.default_rng(7 + w)
    T, D = 23, 8
    Hq, G = (4, 1) if shared else (4, 2)
    q, k, v, zk, zv, _, _ = _inputs(rng, T, Hq, G, D, 1, shared)
    gq = 1 + 0.2 * rng.standard_normal(D) if rms else None
    gk = 1 + 0.2 * rng.standard_normal(D) if rms else None
    cfg = _cfg(orc, n_q_heads=Hq, n_kv_heads=G, head_dim=D, shared_kv=shared, block_m=1, n_win=w,
               rope_dims=rope, rmsnorm=rms, rope_theta=30.0)
    z0 = np.zeros((1, G * D))
    got = orc.forward(cfg, q, k, v, zk, zv, z0, None if shared else z0, None, gq, gk)[0]
    want = _dense_reference(q, k, v, shared, rope, rms, 30.0, gq, gk)
    np.testing.assert_allclose(got, want, atol=1e-12, rtol=1e-11)


@pytest.mark.parametrize("m", [2, 5, 16])
def test_window_covering_all_tokens_is_causal_attention(orc, m):
    """n_win >= L: no pooled entry is ever visible, so the output is causal
    softmax attention over the raw tokens, whatever m and the pooling inputs."""
    rng = np.random.default_rng(m)
    T, Hq, G, D = 31, 6, 2, 8
    q, k, v, zk, zv, bpk, bpv = _inputs(rng, T, Hq, G, D, m, False)
    cfg = _cfg(orc, n_q_heads=Hq, n_kv_heads=G, head_dim=D, shared_kv=False, block_m=m, n_win=T,
               rope_dims=8, rope_theta=100.0)
    got = orc.forward(cfg, q, k, v, zk, zv, bpk, bpv)[0]
    want = _dense_reference(q, k, v, False, 8, False, 100.0)
    np.testing.assert_allclose(got, want, atol=1e-12, rtol=1e-11)


def test_uniform_logits_give_block_mean(orc):
    """Z constant within each (block, channel) and zero bias: weights are 1/m."""
    rng = np.random.default_rng(3)
    m, nb, G, D = 8, 5, 2, 16
    x = rng.standard_normal((2, nb * m + 3, G, D))
    zc = rng.standard_normal((2, nb, 1, G, D)) * 5
    z = np.concatenate([np.broadcast_to(zc, (2, nb, m, G, D)).reshape(2, nb * m, G, D),
                        rng.standard_normal((2, 3, G, D))], axis=1)
    cfg = _cfg(orc, n_q_heads=G, n_kv_heads=G, head_dim=D, shared_kv=False, block_m=m, n_win=0)
    got = orc.pool(cfg, orc.VALUE, x, z, np.zeros((m, G * D)))
    want = x[:, :nb * m].reshape(2, nb, m, G, D).mean(axis=2)
    np.testing.assert_allclose(got, want, atol=1e-14, rtol=1e-13)


def test_pooling_is_a_convex_combination(orc):
    """Weights are positive and sum to one: pooling ones gives ones, and each
    pooled channel lies within its block's min and max."""
    rng = np.random.default_rng(4)
    m, G, D = 16, 3, 8
    x = rng.standard_normal((1, 5 * m, G, D))
    z = rng.standard_normal(x.shape) * 3
    bpos = rng.standard_normal((m, G * D))
    cfg = _cfg(orc, n_q_heads=G, n_kv_heads=G, head_dim=D, shared_kv=False, block_m=m, n_win=0)
    ones = orc.pool(cfg, orc.VALUE, np.ones_like(x), z, bpos)
    np.testing.assert_allclose(ones, 1.0, atol=1e-14)
    got = orc.pool(cfg, orc.VALUE, x, z, bpos)[0]
    blocks = x[0].reshape(5, m, G, D)
    assert np.all(got <= blocks.max(axis=1) + 1e-14)
    assert np.all(got >= blocks.min(axis=1) - 1e-14)


def test_one_hot_bias_and_logits_select_positions(orc):
    """A dominant positional bias at in-block offset i selects token i of every
    block; a dominant content logit selects its own token.  Pins that B_pos is
    indexed [offset, g*D + c] and Z by (token, g, c)."""
    rng = np.random.default_rng(5)
    m, G, D, nb = 4, 2, 4, 3
    x = rng.standard_normal((1, nb * m, G, D))
    z = rng.standard_normal(x.shape) * 0.1
    cfg = _cfg(orc, n_q_heads=G, n_kv_heads=G, head_dim=D, shared_kv=False, block_m=m, n_win=0)
    for i in range(m):
        bpos = np.zeros((m, G * D))
        bpos[i, :] = 800.0
        got = orc.pool(cfg, orc.VALUE, x, z, bpos)[0]
        np.testing.assert_allclose(got, x[0].reshape(nb, m, G, D)[:, i], atol=1e-12)
    # content: per (block, g, c) pick a random offset and make its logit dominate
    pick = rng.integers(0, m, size=(nb, G, D))
    z2 = np.zeros((nb, m, G, D))
    np.put_along_axis(z2, pick[:, None], 900.0, axis=1)
    got = orc.pool(cfg, orc.VALUE, x, z2.reshape(1, nb * m, G, D), np.zeros((m, G * D)))[0]
    want = np.take_along_axis(x[0].reshape(nb, m, G, D), pick[:, None], axis=1)[:, 0]
    np.testing.assert_allclose(got, want, atol=1e-12)


def test_logit_shift_invariance(orc):
    """Adding a constant per (block, channel) to Z leaves the pooled entry unchanged."""
    rng = np.random.default_rng(6)
    m, G, D, nb = 8, 2, 8, 4
    x = rng.standard_normal((1, nb * m, G, D))
    z = rng.standard_normal(x.shape)
    bpos = rng.standard_normal((m, G * D)) * 0.5
    shift = np.repeat(rng.standard_normal((1, nb, 1, G, D)) * 20, m, axis=2).reshape(x.shape)
    cfg = _cfg(orc, n_q_heads=G, n_kv_heads=G, head_dim=D, shared_kv=False, block_m=m, n_win=0,
               rope_dims=8, rmsnorm=True)
    for series in (orc.KEY, orc.VALUE):
        a = orc.pool(cfg, series, x, z, bpos)
        b = orc.pool(cfg, series, x, z + shift, bpos)
        np.testing.assert_allclose(a, b, atol=1e-13)


def test_sink_closed_form_and_limit(orc):
    """One visible token: o = v * sigmoid(s - sigma) with s = q.k / sqrt(D).
    sigma -> -inf recovers the sink-free output exactly."""
    rng = np.random.default_rng(8)
    D = 16
    q, k, v, zk, zv, bpk, bpv = _inputs(rng, 1, 2, 1, D, 4, False)
    sink = np.array([0.3, -1.7])
    cfg = _cfg(orc, n_q_heads=2, n_kv_heads=1, head_dim=D, shared_kv=False, block_m=4, n_win=4)
    got = orc.forward(cfg, q, k, v, zk, zv, bpk, bpv, sink)[0, 0]
    s = q[0, 0] @ k[0, 0, 0] / np.sqrt(D)
    want = v[0, 0, 0][None, :] * expit(s - sink)[:, None]
    np.testing.assert_allclose(got, want, atol=1e-14, rtol=1e-13)
    q, k, v, zk, zv, bpk, bpv = _inputs(rng, 40, 4, 2, 8, 4, False)
    cfg = _cfg(orc, n_q_heads=4, n_kv_heads=2, head_dim=8, shared_kv=False, block_m=4, n_win=6)
    a = orc.forward(cfg, q, k, v, zk, zv, bpk, bpv, np.full(4, -1e300))
    b = orc.forward(cfg, q, k, v, zk, zv, bpk, bpv, None)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("shared", [False, True])
def test_strict_causality(orc, shared):
    """Perturbing any input at positions > t leaves row t unchanged (README:
    strict causality; incomplete blocks never leak future tokens)."""
    rng = np.random.default_rng(9)
    T, m, w = 45, 4, 6
    Hq, G, D = (4, 1, 8) if shared else (4, 2, 8)
    q, k, v, zk, zv, bpk, bpv = _inputs(rng, T, Hq, G, D, m, shared)
    cfg = _cfg(orc, n_q_heads=Hq, n_kv_heads=G, head_dim=D, shared_kv=shared, block_m=m, n_win=w,
               rope_dims=4, rmsnorm=shared)
    base = orc.forward(cfg, q, k, v, zk, zv, bpk, bpv)
    for t in (0, 5, 17, 30, 43):
        arrs = [a.copy() if a is not None else None for a in (q, k, v, zk, zv)]
        for a in arrs:
            if a is not None:
                a[:, t + 1:] += rng.standard_normal(a[:, t + 1:].shape) * 3
        got = orc.forward(cfg, *arrs, bpk, bpv)
        assert np.array_equal(got[:, :t + 1], base[:, :t + 1])
        if t + 1 < T:
            assert not np.allclose(got[:, t + 1:], base[:, t + 1:])


def test_rope_preserves_norm_and_rmsnorm_gives_unit_rms(orc):
    """Pooled key entries: RoPE is a rotation (norms match the unrotated
    pooled values); RMSNorm leaves mean(e^2) = ms / (ms + eps)."""
    rng = np.random.default_rng(10)
    m, G, D = 4, 2, 16
    x = rng.standard_normal((1, 6 * m, G, D))
    z = rng.standard_normal(x.shape)
    bpos = rng.standard_normal((m, G * D))
    cfg = _cfg(orc, n_q_heads=G, n_kv_heads=G, head_dim=D, shared_kv=False, block_m=m, n_win=0,
               rope_dims=16, rope_theta=10.0)
    rot = orc.pool(cfg, orc.KEY, x, z, bpos, pos0=8)
    plain = orc.pool(cfg, orc.VALUE, x, z, bpos)
    np.testing.assert_allclose(np.linalg.norm(rot, axis=-1), np.linalg.norm(plain, axis=-1), rtol=1e-13)
    assert not np.allclose(rot, plain)
    cfg = _cfg(orc, n_q_heads=G, n_kv_heads=G, head_dim=D, shared_kv=False, block_m=m, n_win=0,
               rmsnorm=True, rms_eps=1e-3)
    e = orc.pool(cfg, orc.KEY, x, z, bpos)
    ms = np.mean(plain ** 2, axis=-1)
    np.testing.assert_allclose(np.mean(e ** 2, axis=-1), ms / (ms + 1e-3), rtol=1e-12)


def test_pool_block_start_positions(orc):
    """Entries pooled from a slice that starts at pos0 carry RoPE at
    pos0 + j*m: they equal the matching entries of the whole sequence."""
    rng = np.random.default_rng(11)
    m, G, D = 4, 1, 8
    x = rng.standard_normal((1, 10 * m, G, D))
    z = rng.standard_normal(x.shape)
    bpos = rng.standard_normal((m, G * D))
    cfg = _cfg(orc, n_q_heads=2, n_kv_heads=G, head_dim=D, shared_kv=True, block_m=m, n_win=0,
               rope_dims=8, rmsnorm=True)
    whole = orc.pool(cfg, orc.KEY, x, z, bpos)
    part = orc.pool(cfg, orc.KEY, x[:, 3 * m:7 * m], z[:, 3 * m:7 * m], bpos, pos0=3 * m)
    np.testing.assert_allclose(part, whole[:, 3:7], atol=1e-14)


@pytest.mark.parametrize("shared", [False, True])
def test_stream_equals_prefill_rows(orc, shared):
    """Token-by-token generation through the cache (pool each block once when
    it completes) reproduces every prefill row."""
    rng = np.random.default_rng(12)
    T, m, w = 50, 8, 5
    Hq, G, D = (4, 1, 8) if shared else (6, 2, 8)
    q, k, v, zk, zv, bpk, bpv = _inputs(rng, T, Hq, G, D, m, shared)
    sink = rng.standard_normal(Hq)
    cfg = _cfg(orc, n_q_heads=Hq, n_kv_heads=G, head_dim=D, shared_kv=shared, block_m=m, n_win=w,
               rope_dims=8, rmsnorm=shared)
    want = orc.forward(cfg, q, k, v, zk, zv, bpk, bpv, sink)[0]
    st = orc.Stream(cfg, bpk, bpv)
    for t in range(T):
        st.extend(k[0, t:t + 1], zk[0, t:t + 1], None if shared else v[0, t:t + 1],
                  None if shared else zv[0, t:t + 1])
        np.testing.assert_allclose(st.query(q[0, t], sink), want[t], atol=1e-13)


def test_decode_ragged_equals_prefill_rows(orc):
    """decode() of ragged sequences equals the prefill row at lens-1."""
    rng = np.random.default_rng(13)
    Tm, m, w = 60, 4, 7
    q, k, v, zk, zv, bpk, bpv = _inputs(rng, Tm, 4, 2, 8, m, False)
    k, v, zk, zv = (np.concatenate([a, rng.standard_normal(a.shape)]) for a in (k, v, zk, zv))
    qd = rng.standard_normal((2, 4, 8))
    lens = np.array([60, 23])
    cfg = _cfg(orc, n_q_heads=4, n_kv_heads=2, head_dim=8, shared_kv=False, block_m=m, n_win=w, rope_dims=8)
    got = orc.decode(cfg, qd, k, v, zk, zv, bpk, bpv, lens)
    for b in range(2):
        L = lens[b]
        qq = np.zeros((1, L, 4, 8)); qq[0, L - 1] = qd[b]
        want = orc.forward(cfg, qq, k[b:b + 1, :L], v[b:b + 1, :L], zk[b:b + 1, :L], zv[b:b + 1, :L],
                           bpk, bpv, rows=[L - 1])[0, 0]
        np.testing.assert_allclose(got[b], want, atol=1e-14)


def test_oracle_rejects_bad_arguments(orc):
    cfg = _cfg(orc, n_q_heads=3, n_kv_heads=2, head_dim=8, shared_kv=False, block_m=4, n_win=0)
    with pytest.raises(ValueError):
        orc.pool(cfg, orc.VALUE, np.zeros((1, 8, 2, 8)), np.zeros((1, 8, 2, 8)), np.zeros((4, 16)))


@pytest.mark.parametrize("rms", [False, True])
def test_pooled_entry_takes_rope_at_block_start(orc, rms):
    """A block of identical tokens pools to that token, so its key entry must
    equal the token's own key treatment at the block-start position j*m
    (CSA page, "Deviations from paper": block-start RoPE positions), here
    computed with torch's rms_norm and complex rotation."""
    rng = np.random.default_rng(14)
    m, G, D, nb = 8, 2, 16, 5
    tok = rng.standard_normal((1, nb, 1, G, D))
    x = np.broadcast_to(tok, (1, nb, m, G, D)).reshape(1, nb * m, G, D)
    z = rng.standard_normal(x.shape)
    bpos = rng.standard_normal((m, G * D))
    cfg = _cfg(orc, n_q_heads=G, n_kv_heads=G, head_dim=D, shared_kv=False, block_m=m, n_win=0,
               rope_dims=12, rmsnorm=rms, rope_theta=20.0)
    got = orc.pool(cfg, orc.KEY, x, z, bpos, pos0=3 * m)[0]
    e = torch.from_numpy(tok[0, :, 0].copy())
    if rms:
        e = torch.nn.functional.rms_norm(e, (D,), None, 1e-6)
    pos = (torch.arange(nb) * m + 3 * m)[:, None].expand(nb, G)
    want = _torch_rope(e, pos, 12, 20.0).numpy()
    np.testing.assert_allclose(got, want, atol=1e-13)
