"""GPU parity of the one-launch serving step (lbca_decode_step): its outputs
match the oracle step by step across block completions, and the cache it
leaves behind is the one lbca_append + lbca_decode leave."""
import numpy as np
import pytest
import torch

from block_compressed_long_b200 import synth
from lbca_cases import DecodeRun, assert_close, f64, fused_step, lib, oracle_decode

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS


@pytest.fixture(scope="module")
def L():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib()


@pytest.mark.parametrize("name,kw,steps", [
    ("gqa_decode_32k", dict(ctx=(3000, 3000)), 70),
    ("gqa_decode_32k", dict(ctx=(5, 5), n_win=3, block_m=4), 40),
    ("ragged_gqa_decode_append", dict(ctx=(0, 2500), batch=7), 66),
    ("hca_mqa_decode_128k", dict(ctx=(700, 900), batch=2, n_q_heads=4, head_dim=128, rope_dims=32), 130),
    ("tiny_f32_prefill", dict(kind="decode", ctx=(300, 300), n_kv_heads=1, n_q_heads=4), 20),
])
def test_step_matches_oracle(L, name, kw, steps):
    w = synth.scaled(W[name], steps=steps, **kw)
    inp = synth.make(w)
    run = DecodeRun(L, w, inp)
    for s in range(steps):
        got = fused_step(run)
        if s % 5 == 0 or s == steps - 1:
            torch.cuda.synchronize()
            assert_close(f64(got), oracle_decode(w, inp, s), w.dtype, f"{name} step {s}")
    assert int(run.status.item()) == 0


def test_step_leaves_the_same_cache(L):
    """Fused steps and append + decode steps produce identical caches and
    identical outputs (same arithmetic, same rounding)."""
    w = synth.scaled(W["gqa_decode_32k"], ctx=(1000, 1000), steps=140)
    inp = synth.make(w)
    a, b = DecodeRun(L, w, inp), DecodeRun(L, w, inp)
    for _ in range(140):
        oa = a.step()
        ob = fused_step(b)
        torch.cuda.synchronize()
        assert_close(f64(ob), f64(oa), "bf16", "fused vs two-call")
    for name in ("pooled_k", "pooled_v", "ring_k", "ring_v", "pool_state", "seq_lens"):
        assert torch.equal(getattr(a.cache, name), getattr(b.cache, name)), name


def test_step_full_size(L):
    w = synth.scaled(W["gqa_decode_32k"], steps=3)
    inp = synth.make(w)
    run = DecodeRun(L, w, inp)
    for _ in range(3):
        got = fused_step(run)
    torch.cuda.synchronize()
    assert_close(f64(got), oracle_decode(w, inp, 2), "bf16", "step full")


@pytest.mark.parametrize("name,kw", [
    ("gqa_decode_32k", dict(ctx=(1000, 1000))),                                  # cluster step
    ("hca_mqa_decode_128k", dict(ctx=(700, 700), batch=2)),                      # tensor-core shared-entry step
    ("ragged_gqa_decode_append", dict(ctx=(50, 900), batch=16)),                 # persistent step
])
@pytest.mark.parametrize("graph", [False, True], ids=["eager", "graph"])
def test_overlap_flag_changes_nothing_but_timing(L, name, kw, graph):
    """A chain of three layers, each with its own cache, each layer's query the
    previous layer's output (so every step depends on the kernel before it):
    with the caches flagged LBCA_CACHE_OVERLAP_PREV the steps launch with
    programmatic dependence and read their caches while the previous kernel
    drains; outputs and caches must be bit-identical to the unflagged chain."""
    NL, steps = 3, 5
    w = synth.scaled(W[name], steps=steps, **kw)
    inp = synth.make(w)
    runs = {f: [DecodeRun(L, w, inp, steps=steps) for _ in range(NL)] for f in (0, L.LBCA_CACHE_OVERLAP_PREV)}
    outs = {}
    for flags, chain in runs.items():
        for run in chain:
            run.cache.flags = flags
            run.step_ws = torch.zeros(max(L.lbca_decode_step_workspace_bytes(run.cfg, run.B, run.max_ctx), 16),
                                      dtype=torch.uint8, device="cuda")
        o = [[torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.bfloat16, device="cuda") for _ in range(NL)]
             for _ in range(steps)]

        def token(s):
            q = chain[0].q[s]
            for layer, run in enumerate(chain):
                L.lbca_decode_step(run.cfg, run.token(run.k), run.token(run.v), run.token(run.zk),
                                   run.token(run.zv), run.bpk, run.bpv, None, q, run.cache, run.sink, None,
                                   o[s][layer], run.step_ws, run.max_ctx, run.status)
                q = o[s][layer]
            for run in chain:
                run.pos += 1

        if graph and flags:
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                for s in range(steps):
                    token(s)
            gr.replay()
        else:
            for s in range(steps):
                token(s)
        torch.cuda.synchronize()
        outs[flags] = o
    for s in range(steps):
        for layer in range(NL):
            assert torch.equal(outs[0][s][layer], outs[L.LBCA_CACHE_OVERLAP_PREV][s][layer]), (s, layer)
    for a, b in zip(runs[0], runs[L.LBCA_CACHE_OVERLAP_PREV]):
        for f in ("pooled_k", "pooled_v", "ring_k", "ring_v", "pool_state", "seq_lens"):
            x, y = getattr(a.cache, f), getattr(b.cache, f)
            assert (x is None and y is None) or torch.equal(x, y), f
        assert int(a.status.item()) == 0 and int(b.status.item()) == 0
