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
