"""Brute-force NumPy restatement of block-compressed attention, for tiny inputs.

TEST INFRASTRUCTURE ONLY.  It exists to pin the C oracle: it restates the same
definition with different machinery, so that a slip in one (a dropped term, a
wrong index or sign, a transposed operand) shows up as a disagreement.

  * the visible set is found by search, not by a closed form: the largest
    p >= 0 with p*m + w <= L gives the pooled prefix, and the raw region is
    checked to partition the remaining tokens ("mSeek" README, "How LBCA
    works" steps 4-5: completed summaries plus the exact local window;
    incomplete blocks stay raw);
  * pooling uses scipy's softmax over the block axis and an einsum (HCA page,
    "What is implemented": content-dependent softmax weights plus a learnable
    positional bias, Eqs 20-23);
  * RoPE multiplies consecutive-pair complex numbers by exp(i*pos*freq), at
    block-start positions for pooled entries (CSA page, "Deviations from
    paper");
  * the sink is one extra logit with a zero value vector (CSA page, "What is
    implemented", Eq 27); the shared-KV output is rotated back by -t on its
    RoPE dims (same section, "-i rotation of outputs").
"""
from __future__ import annotations

import numpy as np
from scipy.special import softmax


def _rms(x, gamma, eps):
    D = x.shape[-1]
    nrm = np.linalg.norm(x, axis=-1, keepdims=True)
    y = x / np.sqrt(nrm ** 2 / D + eps)
    return y if gamma is None else y * gamma


def _rot(x, pos, rho, theta):
    """Complex-number RoPE of the last rho dims of x [..., D] at pos [...]."""
    if rho == 0:
        return x
    D = x.shape[-1]
    y = np.array(x, dtype=np.float64, copy=True)
    tail = y[..., D - rho:]
    zc = tail[..., 0::2] + 1j * tail[..., 1::2]
    freq = theta ** (-np.arange(rho // 2) * 2.0 / rho)
    ph = np.exp(1j * np.multiply.outer(np.asarray(pos, dtype=np.float64), freq))
    zc = zc * ph
    tail[..., 0::2] = zc.real
    tail[..., 1::2] = zc.imag
    return y


def visible(L, m, w):
    """(P, raw token list) for a query seeing L tokens, by search."""
    p = 0
    while (p + 1) * m + w <= L:
        p += 1
    raw = list(range(p * m, L))
    covered = sorted([s for j in range(p) for s in range(j * m, (j + 1) * m)] + raw)
    assert covered == list(range(L)), "pooled prefix and raw window must partition the history"
    return p, raw


def pool_series(x, z, bpos, m):
    """x, z [T, G, D]; bpos [m, G*D] -> pooled [T//m, G, D] (no finalisation)."""
    T, G, D = x.shape
    nb = T // m
    xb = x[:nb * m].reshape(nb, m, G, D)
    a = z[:nb * m].reshape(nb, m, G, D) + bpos.reshape(1, m, G, D)
    wts = softmax(a, axis=1)
    return np.einsum("jigd,jigd->jgd", wts, xb)


def attention(q, k, v, zk, zv, bpk, bpv, *, m, w, shared_kv, rope_dims=0, theta=10000.0,
              rmsnorm=False, eps=1e-6, sink=None, gamma_q=None, gamma_kv=None, scale=None):
    """Prefill outputs [T, Hq, D] for one sequence (q [T,Hq,D]; k.. [T,G,D])."""
    T, Hq, D = q.shape
    G = k.shape[1]
    r = Hq // G
    scale = 1.0 / np.sqrt(D) if scale is None else scale

    def key_side(e, pos):
        if rmsnorm:
            e = _rms(e, gamma_kv, eps)
        return _rot(e, pos, rope_dims, theta)

    pk = pool_series(k, zk, bpk, m)
    ek = key_side(pk, (np.arange(pk.shape[0]) * m)[:, None] * np.ones((1, G)))
    ev = ek if shared_kv else pool_series(v, zv, bpv, m)
    kr = key_side(k, np.arange(T)[:, None] * np.ones((1, G)))
    vr = kr if shared_kv else v

    qn = _rms(q, gamma_q, eps) if rmsnorm else q
    qr = _rot(qn, np.arange(T)[:, None] * np.ones((1, Hq)), rope_dims, theta)

    out = np.zeros((T, Hq, D))
    for t in range(T):
        p, raw = visible(t + 1, m, w)
        for h in range(Hq):
            g = h // r
            keys = np.concatenate([ek[:p, g], kr[raw, g]], axis=0)
            vals = np.concatenate([ev[:p, g], vr[raw, g]], axis=0)
            logits = keys @ qr[t, h] * scale
            if sink is not None:
                logits = np.append(logits, sink[h])
                vals = np.concatenate([vals, np.zeros((1, D))], axis=0)
            o = softmax(logits) @ vals
            if shared_kv:
                o = _rot(o, -t, rope_dims, theta)
            out[t, h] = o
    return out


# ---- CSA form (CSA page, "What is implemented": Eqs 9-12, 13-17, 18-19, 27) ----
def pool_dual_series(xa, za, xb, zb, bpa, bpb, m):
    """Dual overlapped pooling, one sequence: x*, z* [T, G, D]; bp* [m, G*D] ->
    [T//m, G, D].  Entry i stacks block i of the a-series and block i-1 of the
    b-series along one axis and takes scipy's softmax over all of it (block 0:
    the a-series block alone)."""
    T, G, D = xa.shape
    nb = T // m
    out = np.zeros((nb, G, D))
    for i in range(nb):
        la = za[i * m:(i + 1) * m] + bpa.reshape(m, G, D)
        va = xa[i * m:(i + 1) * m]
        if i > 0:
            lb = zb[(i - 1) * m:i * m] + bpb.reshape(m, G, D)
            logits = np.concatenate([la, lb], axis=0)
            vals = np.concatenate([va, xb[(i - 1) * m:i * m]], axis=0)
        else:
            logits, vals = la, va
        out[i] = (softmax(logits, axis=0) * vals).sum(axis=0)
    return out


def indexer(q, w, kx, nvis):
    """q [HI, DI], w [HI], kx [NB, DI] -> scores of the first nvis blocks."""
    dots = kx[:nvis] @ q.T                      # [nvis, HI]
    return np.maximum(dots, 0.0) @ w


def topk(scores, k):
    """Indices of the k largest scores (ties: lower index first), by sorting."""
    order = sorted(range(len(scores)), key=lambda j: (-scores[j], j))
    return order[:k]


def attention_sparse(q, entries, sel, c_hist, t, *, w, rope_dims=0, theta=10000.0, rmsnorm=False, eps=1e-6,
                     sink=None, gamma_q=None, gamma_kv=None, scale=None):
    """One query q [Hq, D] at position t over entries[sel] ([NB, D] finalised)
    plus the raw window c_hist[max(0, t+1-w) .. t] ([T, D], finalised here)
    and the sink; output rotated back by -t.  [Hq, D]."""
    Hq, D = q.shape
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    win = list(range(max(0, t + 1 - w), t + 1))
    raw = c_hist[win]
    if rmsnorm:
        raw = _rms(raw, gamma_kv, eps)
    raw = _rot(raw, np.asarray(win, dtype=np.float64), rope_dims, theta)
    rows = np.concatenate([entries[[j for j in sel if j >= 0]], raw], axis=0)
    qn = _rms(q, gamma_q, eps) if rmsnorm else q
    qr = _rot(qn, np.full(Hq, float(t)), rope_dims, theta)
    out = np.zeros((Hq, D))
    for h in range(Hq):
        logits = rows @ qr[h] * scale
        vals = rows
        if sink is not None:
            logits = np.append(logits, sink[h])
            vals = np.concatenate([vals, np.zeros((1, D))], axis=0)
        out[h] = _rot(softmax(logits) @ vals, -t, rope_dims, theta)
    return out
