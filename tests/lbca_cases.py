"""Shared helpers for the GPU parity tests: run a workload through the C ABI
and through the fp64 oracle on the same seeded inputs, and compare.

Tolerances (fixed by the method's target): bf16 I/O -> max-abs <= 1e-2 and
mean-abs <= 1e-3; f32 I/O -> max-abs <= 1e-5 * max|oracle| (relative 1e-5).
"""
from __future__ import annotations

import numpy as np
import torch

from block_compressed_long_b200 import synth
from oracle import oracle as orc

f64 = synth.f64


def lib():
    from block_compressed_long_b200 import build
    build.build()
    from block_compressed_long_b200 import lbca
    return lbca


def ocfg(w: synth.Workload) -> orc.Config:
    return orc.Config(w.n_q_heads, w.n_kv_heads, w.head_dim, w.shared_kv, w.block_m, w.n_win,
                      w.rope_dims, w.rmsnorm, w.rope_theta)


def lcfg(L, w: synth.Workload):
    return L.config(w.n_q_heads, w.n_kv_heads, w.head_dim, w.shared_kv, w.block_m, w.n_win, w.rope_dims,
                    w.rmsnorm, w.rope_theta, dtype=w.dtype)


def assert_close(got, want, dtype: str, what: str = ""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    d = np.abs(got - want)
    if dtype == "bf16":
        assert d.max() <= 1e-2, f"{what}: max-abs {d.max():.3e}"
        assert d.mean() <= 1e-3, f"{what}: mean-abs {d.mean():.3e}"
    else:
        scale = max(np.abs(want).max(), 1e-30)
        assert d.max() <= 1e-5 * scale, f"{what}: max-abs {d.max():.3e} vs 1e-5 * {scale:.3e}"
    return float(d.max()), float(d.mean())


def assert_close_stored(got, want, dtype: str, what: str = ""):
    """Check of stored intermediate entries (pooled entries).  The bf16 store of
    an exact value of magnitude |x| is off by up to 2^-9 |x| from rounding
    alone, above 1e-2 once |x| > 5 (RMSNorm'd entries reach that), so each
    element may be off by max(1e-2, 2^-8 |x|): the rounding plus as much again
    for f32 arithmetic.  Likewise the mean: rounding unit-RMS values to bf16
    alone costs ~1.07e-3 mean-abs, so the mean bound is 1e-3 plus the mean
    rounding allowance 2^-9 mean|x|.  f32 keeps relative 1e-5."""
    if dtype != "bf16":
        return assert_close(got, want, dtype, what)
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape and np.all(np.isfinite(got)), what
    d = np.abs(got - want)
    bound = np.maximum(1e-2, np.abs(want) * 2.0 ** -8)
    worst = float((d / bound).max())
    assert worst <= 1.0, f"{what}: error {worst:.2f}x the bf16 storage bound"
    mean_bound = 1e-3 + 2.0 ** -9 * float(np.abs(want).mean())
    assert d.mean() <= mean_bound, f"{what}: mean-abs {d.mean():.3e} > {mean_bound:.3e}"


def visible_entries(w, L):
    """Size of the visible list at length L (block-aligned partition)."""
    P = max(0, (L - w.n_win) // w.block_m)
    return P + (L - P * w.block_m) if L > 0 else 0


def dev(t):
    return None if t is None else t.cuda()


def sub_cache(L, cache, b):
    """The one-sequence view of sequence b of a batched cache (contiguous slices)."""
    per = cache.pool_state.numel() // cache.batch
    sl = slice(b, b + 1)
    return L.Cache(cache.cfg, 1, cache.max_blocks, cache.ring_slots, cache.pooled_k[sl],
                   None if cache.pooled_v is None else cache.pooled_v[sl], cache.ring_k[sl],
                   None if cache.ring_v is None else cache.ring_v[sl],
                   cache.pool_state[b * per:(b + 1) * per], cache.seq_lens[sl])


def gpu_prefill(L, w, inp, cache=None, want_out=True, T=None):
    """Prefill of the first T tokens (all by default) of every sequence."""
    cfg = lcfg(L, w)
    T = inp.k.shape[1] if T is None else T
    B = inp.k.shape[0]
    sl = lambda t: None if t is None else t[:, :T].contiguous().cuda()  # noqa: E731
    q = sl(inp.q) if want_out else None
    out = torch.empty(B, T, w.n_q_heads, w.head_dim, dtype=L.torch_dtype(cfg), device="cuda") if want_out else None
    ws = torch.zeros(max(L.lbca_prefill_workspace_bytes(cfg, B, T, cache is not None), 16), dtype=torch.uint8,
                     device="cuda")
    L.lbca_prefill(cfg, q, sl(inp.k), sl(inp.v), sl(inp.zk), sl(inp.zv), dev(inp.bpos_k), dev(inp.bpos_v),
                   dev(inp.sink), None, None, out, cache, ws, batch=B, T=T)
    return out


def oracle_prefill(w, inp, rows=None, T=None):
    T = inp.k.shape[1] if T is None else T
    sl = lambda t: None if t is None else f64(t[:, :T])  # noqa: E731
    return orc.forward(ocfg(w), sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.zk), sl(inp.zv), f64(inp.bpos_k),
                       f64(inp.bpos_v), f64(inp.sink), rows=rows)


class DecodeRun:
    """Drive a decode workload through the C ABI: prefill every sequence's
    cached context into the cache, then (append, decode) one token per step."""

    def __init__(self, L, w, inp, steps=None, chunked_prefill=True):
        self.L, self.w, self.inp = L, w, inp
        self.cfg = lcfg(L, w)
        self.B = inp.k.shape[0]
        self.steps = w.steps if steps is None else steps
        self.max_ctx = int(inp.lens.max()) + self.steps
        self.cache = L.Cache.allocate(self.cfg, self.B, self.max_ctx)
        self.k, self.v, self.zk, self.zv = (dev(t) for t in (inp.k, inp.v, inp.zk, inp.zv))
        self.bpk, self.bpv, self.sink = dev(inp.bpos_k), dev(inp.bpos_v), dev(inp.sink)
        self.q = dev(inp.q)
        for b in range(self.B):
            Lb = int(inp.lens[b])
            sc = sub_cache(L, self.cache, b)
            s = lambda t: None if t is None else t[b:b + 1, :Lb]  # noqa: E731
            ws = torch.zeros(16, dtype=torch.uint8, device="cuda")
            L.lbca_prefill(self.cfg, None, s(self.k), s(self.v), s(self.zk), s(self.zv), self.bpk, self.bpv,
                           None, None, None, None, sc, ws, batch=1, T=Lb)
        self.ws = torch.zeros(L.lbca_decode_workspace_bytes(self.cfg, self.B, self.max_ctx), dtype=torch.uint8,
                              device="cuda")
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.pos = torch.as_tensor(inp.lens, device="cuda")
        self.ar = torch.arange(self.B, device="cuda")
        self.step_i = 0

    def token(self, t):
        return None if t is None else t[self.ar, self.pos].contiguous()

    def step(self):
        L = self.L
        L.lbca_append(self.cfg, self.token(self.k), self.token(self.v), self.token(self.zk), self.token(self.zv),
                      self.bpk, self.bpv, None, self.cache, self.status)
        out = torch.empty(self.B, self.w.n_q_heads, self.w.head_dim, dtype=L.torch_dtype(self.cfg), device="cuda")
        L.lbca_decode(self.cfg, self.q[self.step_i], self.cache, self.sink, None, None, out, self.ws, self.max_ctx,
                      self.status)
        self.pos += 1
        self.step_i += 1
        return out


def fused_step(run: DecodeRun):
    """The same step as DecodeRun.step through lbca_decode_step (one launch)."""
    L = run.L
    if not hasattr(run, "step_ws"):
        run.step_ws = torch.zeros(max(L.lbca_decode_step_workspace_bytes(run.cfg, run.B, run.max_ctx), 16),
                                  dtype=torch.uint8, device="cuda")
    out = torch.empty(run.B, run.w.n_q_heads, run.w.head_dim, dtype=L.torch_dtype(run.cfg), device="cuda")
    L.lbca_decode_step(run.cfg, run.token(run.k), run.token(run.v), run.token(run.zk), run.token(run.zv), run.bpk,
                       run.bpv, None, run.q[run.step_i], run.cache, run.sink, None, out, run.step_ws, run.max_ctx,
                       run.status)
    run.pos += 1
    run.step_i += 1
    return out


def oracle_decode(w, inp, step, seqs=None):
    """Oracle output of decode step `step` (0-based) for the sequences `seqs`."""
    seqs = range(inp.k.shape[0]) if seqs is None else seqs
    c = ocfg(w)
    outs = []
    for b in seqs:
        Lb = int(inp.lens[b]) + step + 1
        s = lambda t: None if t is None else f64(t[b:b + 1, :Lb])  # noqa: E731
        outs.append(orc.decode(c, f64(inp.q[step, b:b + 1]), s(inp.k), s(inp.v), s(inp.zk), s(inp.zv),
                               f64(inp.bpos_k), f64(inp.bpos_v), [Lb], f64(inp.sink))[0])
    return np.stack(outs)
