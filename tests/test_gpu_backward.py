"""GPU parity of the prefill backward (lbca_prefill_backward) through the C
ABI against the fp64 oracle's gradients (themselves pinned by finite
differences): every gradient -- queries, raw keys and values, pooling
logits, positional biases, sink -- on both forms, with RMSNorm, partial RoPE,
the sink and a ragged last block.  The kernels compute in f32 from the exact
inputs; each gradient must be within 2e-4 of its largest magnitude."""
import numpy as np
import pytest
import torch

from block_compressed_long_b200 import synth
from lbca_cases import f64, lcfg, lib, ocfg
from oracle import oracle as orc

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS
RTOL = 2e-4


@pytest.fixture(scope="module")
def L():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib()


def _run(L, w, inp, dout, gq=None, gkv=None):
    cfg = lcfg(L, w)
    B, T = inp.q.shape[:2]
    G, D, Hq, m = w.n_kv_heads, w.head_dim, w.n_q_heads, w.block_m
    f = lambda *s: torch.full(s, 9.0, dtype=torch.float32, device="cuda")  # noqa: E731
    grads = {"dq": f(B, T, Hq, D), "dk": f(B, T, G, D), "dzk": f(B, T, G, D), "dbk": f(m, G * D)}
    if not w.shared_kv:
        grads.update(dv=f(B, T, G, D), dzv=f(B, T, G, D), dbv=f(m, G * D))
    if inp.sink is not None:
        grads["dsink"] = f(Hq)
    ws = torch.zeros(L.lbca_prefill_backward_workspace_bytes(cfg, B, T), dtype=torch.uint8, device="cuda")
    d = lambda t: None if t is None else t.contiguous().cuda()  # noqa: E731
    L.lbca_prefill_backward(cfg, d(inp.q), d(inp.k), d(inp.v), d(inp.zk), d(inp.zv), d(inp.bpos_k), d(inp.bpos_v),
                            d(inp.sink), d(gq), d(gkv), d(dout), grads, ws)
    torch.cuda.synchronize()
    return {k: v.cpu().double().numpy() for k, v in grads.items()}


@pytest.mark.parametrize("name,kw", [
    ("gqa_prefill_16k", dict(seq_len=16 * 9 + 5, n_win=32)),
    ("gqa_decode_32k", dict(kind="prefill", seq_len=64 * 3 + 11, n_win=64)),
    ("hca_mqa_decode_128k", dict(kind="prefill", seq_len=128 + 70, batch=2, block_m=32, n_win=40)),
    ("hca_mqa_decode_128k", dict(kind="prefill", seq_len=150, head_dim=128, rmsnorm=False, rope_dims=6, block_m=8,
                                 n_win=16, n_q_heads=4)),
    ("tiny_f32_prefill", dict(seq_len=16 * 6 + 9)),
    # more pooled entries than one entry tile and many row tiles, a ragged last row tile
    ("gqa_prefill_16k", dict(seq_len=16 * 40 + 7, n_win=48)),
    # the tiled passes at head dim 64 with bf16 I/O and partial RoPE
    ("gqa_prefill_16k", dict(seq_len=16 * 12 + 3, head_dim=64, rope_dims=32, n_win=40)),
], ids=["gqa-m16", "gqa-m64", "hca", "shared-rope6", "tiny-f32", "gqa-multi-tile", "gqa-d64"])
def test_backward_matches_oracle(L, name, kw):
    w = synth.scaled(W[name], **kw)
    inp = synth.make(w)
    dout = synth.normal(w.seed, "dout", tuple(inp.q.shape), dtype=w.dtype)
    got = _run(L, w, inp, dout)
    want = orc.prefill_backward(ocfg(w), f64(inp.q), f64(inp.k), f64(inp.v), f64(inp.zk), f64(inp.zv),
                                f64(inp.bpos_k), f64(inp.bpos_v), f64(dout), f64(inp.sink))
    for k, v in want.items():
        if k == "dsink" and inp.sink is None:
            continue
        g = got[k].reshape(v.shape)
        assert np.all(np.isfinite(g)), k
        err = np.abs(g - v).max()
        assert err <= RTOL * max(np.abs(v).max(), 1e-30), f"{name} {k}: max-abs {err:.3e} vs {np.abs(v).max():.3e}"


def test_backward_with_gains(L):
    """RMSNorm gains on queries and keys enter the backward through RMSNorm."""
    w = synth.scaled(W["hca_mqa_decode_128k"], kind="prefill", seq_len=130, head_dim=256, block_m=16, n_win=20)
    inp = synth.make(w)
    dout = synth.normal(w.seed, "dout", tuple(inp.q.shape), dtype=w.dtype)
    gq = 1 + 0.1 * synth.normal(w.seed, "gq", (w.head_dim,), dtype=w.dtype).float()
    gkv = 1 + 0.1 * synth.normal(w.seed, "gkv", (w.head_dim,), dtype=w.dtype).float()
    gq, gkv = gq.to(torch.bfloat16), gkv.to(torch.bfloat16)
    got = _run(L, w, inp, dout, gq, gkv)
    want = orc.prefill_backward(ocfg(w), f64(inp.q), f64(inp.k), None, f64(inp.zk), None, f64(inp.bpos_k), None,
                                f64(dout), f64(inp.sink), f64(gq), f64(gkv))
    for k, v in want.items():
        err = np.abs(got[k].reshape(v.shape) - v).max()
        assert err <= RTOL * max(np.abs(v).max(), 1e-30), f"{k}: {err:.3e}"
