"""Pins of the oracle's backward (gradients of the prefill with respect to
every input), on the CPU.

The forward oracle is pinned elsewhere; here its gradient is checked against
central finite differences of that same forward in fp64 (an independent
route: no reverse-mode step is shared), on both forms and every feature
(RMSNorm, partial RoPE, sink, -t output rotation, GQA head map, a ragged last
block), plus two exact properties of the pooling softmax: the logits'
gradient sums to zero over every block (a softmax is invariant to a shared
shift), and with m = 1 and no bias pooling is the identity, so no gradient
reaches the logits at all.
"""
import numpy as np
import pytest

from oracle import oracle as orc


def _inputs(rng, shared, B=1, T=14, Hq=4, G=2, D=8, m=3):
    G = 1 if shared else G
    f = lambda *s: rng.standard_normal(s)  # noqa: E731
    x = dict(q=f(B, T, Hq, D), k=f(B, T, G, D), zk=f(B, T, G, D), bpos_k=0.5 * f(m, G * D))
    x.update(v=None, zv=None, bpos_v=None) if shared else x.update(v=f(B, T, G, D), zv=f(B, T, G, D),
                                                                   bpos_v=0.5 * f(m, G * D))
    x.update(sink=f(Hq), gamma_q=1 + 0.2 * f(D), gamma_kv=1 + 0.2 * f(D))
    return x


def _loss(c, x, dout):
    o = orc.forward(c, x["q"], x["k"], x["v"], x["zk"], x["zv"], x["bpos_k"], x["bpos_v"], x["sink"],
                    x["gamma_q"], x["gamma_kv"])
    return float((o * dout).sum())


NAMES = {"q": "dq", "k": "dk", "v": "dv", "zk": "dzk", "zv": "dzv", "bpos_k": "dbk", "bpos_v": "dbv",
         "sink": "dsink"}


@pytest.mark.parametrize("shared,rms,rope,w", [(False, False, 8, 4), (False, True, 4, 2), (True, True, 4, 3),
                                               (True, False, 0, 20)], ids=["gqa", "gqa-rms", "shared", "shared-wide"])
def test_gradients_match_finite_differences(orc, shared, rms, rope, w):
    rng = np.random.default_rng(21)
    m = 3
    c = orc.Config(4, 1 if shared else 2, 8, shared, m, w, rope, rms)
    x = _inputs(rng, shared, m=m)
    dout = rng.standard_normal(x["q"].shape)
    g = orc.prefill_backward(c, x["q"], x["k"], x["v"], x["zk"], x["zv"], x["bpos_k"], x["bpos_v"], dout, x["sink"],
                             x["gamma_q"], x["gamma_kv"])
    eps = 1e-6
    for name, gname in NAMES.items():
        if x[name] is None:
            continue
        flat = x[name].reshape(-1)
        for idx in rng.choice(flat.size, size=min(12, flat.size), replace=False):
            keep = flat[idx]
            flat[idx] = keep + eps
            up = _loss(c, x, dout)
            flat[idx] = keep - eps
            dn = _loss(c, x, dout)
            flat[idx] = keep
            fd = (up - dn) / (2 * eps)
            an = g[gname].reshape(-1)[idx]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, an)


def test_logit_gradients_sum_to_zero_over_each_block(orc):
    rng = np.random.default_rng(22)
    m, T = 4, 4 * 5 + 3
    c = orc.Config(4, 2, 8, False, m, 5, 8, True)
    x = _inputs(rng, False, T=T, m=m)
    dout = rng.standard_normal(x["q"].shape)
    g = orc.prefill_backward(c, x["q"], x["k"], x["v"], x["zk"], x["zv"], x["bpos_k"], x["bpos_v"], dout, x["sink"])
    for name in ("dzk", "dzv"):
        z = g[name][0]
        blocks = z[:(T // m) * m].reshape(T // m, m, 2, 8).sum(axis=1)
        np.testing.assert_allclose(blocks, 0.0, atol=1e-12)
        np.testing.assert_array_equal(z[(T // m) * m:], 0.0)  # the open block is never pooled
    np.testing.assert_allclose(g["dbk"], g["dzk"][0, :(T // m) * m].reshape(T // m, m, 16).sum(0), atol=1e-12)


def test_identity_pooling_passes_no_gradient_to_the_logits(orc):
    rng = np.random.default_rng(23)
    c = orc.Config(4, 2, 8, False, 1, 3, 8, False)
    x = _inputs(rng, False, m=1)
    x["bpos_k"][:] = 0
    x["bpos_v"][:] = 0
    dout = rng.standard_normal(x["q"].shape)
    g = orc.prefill_backward(c, x["q"], x["k"], x["v"], x["zk"], x["zv"], x["bpos_k"], x["bpos_v"], dout)
    for name in ("dzk", "dzv", "dbk", "dbv"):
        np.testing.assert_allclose(g[name], 0.0, atol=1e-12)
