"""GPU parity of the persistent, evenly split form of lbca_decode_step (many
(sequence, head group) pairs, unequal contexts): outputs match the oracle step
by step across block completions, caches equal those of lbca_append +
lbca_decode, and segments cut between CTAs merge correctly (a long sequence
among short ones, sequences with no cached tokens)."""
import numpy as np
import pytest
import torch

from block_compressed_long_b200 import synth
from lbca_cases import DecodeRun, assert_close, f64, fused_step, lcfg, lib, oracle_decode

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS


@pytest.fixture(scope="module")
def L():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib()


CASES = [
    # GQA, 16 sequences x 8 head groups, contexts 0 .. 2500, blocks of 64: a block completes in 66 steps
    ("ragged_gqa_decode_append", dict(ctx=(0, 2500), batch=16), 66),
    # one long sequence among short ones: its segments are cut between many CTAs
    ("ragged_gqa_decode_append", dict(ctx=(20, 200), batch=13, block_m=16), 20),
    # shared-entry form on CUDA cores (append then decode): RMSNorm, partial RoPE, sink, -t output rotation
    ("hca_mqa_decode_128k", dict(ctx=(100, 900), batch=8, n_q_heads=48, head_dim=128, rope_dims=32, block_m=16),
     20),
    # f32 I/O, 4 query heads on one shared entry, sink logit 0
    ("tiny_f32_prefill", dict(kind="decode", ctx=(0, 300), batch=100, n_kv_heads=1, n_q_heads=4), 18),
    # the other head dims of the persistent kernel (bf16 D = 64 and 256), partial RoPE
    ("ragged_gqa_decode_append", dict(ctx=(10, 1500), batch=16, head_dim=64, rope_dims=32), 20),
    ("ragged_gqa_decode_append", dict(ctx=(10, 1200), batch=16, head_dim=256, rope_dims=64), 20),
]


@pytest.mark.parametrize("name,kw,steps", CASES)
def test_persistent_step_matches_oracle(L, name, kw, steps):
    w = synth.scaled(W[name], steps=steps, **kw)
    lens = synth.contexts(w)
    if name == "ragged_gqa_decode_append" and w.block_m == 16:
        lens[5] = 6000  # the long one
    if name == "tiny_f32_prefill":
        lens[[3, 40]] = 0  # sequences with no cached tokens
    inp = synth.make(w, lens=lens)
    run = DecodeRun(L, w, inp)
    # the CUDA-core fused forms serve the GQA form; the shared form's raw window
    # is finalised by the decode kernels, so its steps run append then decode
    want_form = L.LBCA_STEP_TWO_CALLS if w.shared_kv else L.LBCA_STEP_PERSISTENT
    assert L.lbca_decode_step_form(run.cfg, run.B, run.max_ctx) == want_form
    for s in range(steps):
        got = fused_step(run)
        if s % 6 == 0 or s == steps - 1:
            torch.cuda.synchronize()
            assert_close(f64(got), oracle_decode(w, inp, s), w.dtype, f"{name} step {s}")
    assert int(run.status.item()) == 0


def test_persistent_step_leaves_the_same_cache(L):
    w = synth.scaled(W["ragged_gqa_decode_append"], ctx=(0, 900), batch=16, steps=70)
    inp = synth.make(w)
    a, b = DecodeRun(L, w, inp), DecodeRun(L, w, inp)
    assert L.lbca_decode_step_form(b.cfg, b.B, b.max_ctx) == L.LBCA_STEP_PERSISTENT
    for _ in range(70):
        oa = a.step()
        ob = fused_step(b)
        torch.cuda.synchronize()
        assert_close(f64(ob), f64(oa), "bf16", "persistent vs two-call")
    for nm in ("pooled_k", "pooled_v", "ring_k", "ring_v", "pool_state", "seq_lens"):
        assert torch.equal(getattr(a.cache, nm), getattr(b.cache, nm)), nm
    # the workspace counters are left zero for the next call
    assert int(b.step_ws[:4].view(torch.int32).item()) == 0


def test_persistent_step_full_size_sampled(L):
    """The ragged 32-sequence batch at full size (contexts 4K .. 64K), three
    steps; sampled sequences against the oracle."""
    w = synth.scaled(W["ragged_gqa_decode_append"], steps=3)
    inp = synth.make(w)
    run = DecodeRun(L, w, inp)
    assert L.lbca_decode_step_form(run.cfg, run.B, run.max_ctx) == L.LBCA_STEP_PERSISTENT
    for _ in range(3):
        got = fused_step(run)
    torch.cuda.synchronize()
    seqs = [0, 7, 19, 31]
    want = oracle_decode(w, inp, 2, seqs)
    assert_close(f64(got)[seqs], want, "bf16", "persistent full size")
    assert int(run.status.item()) == 0


def test_persistent_step_reports_contexts_beyond_max_ctx(L):
    """A workspace sized for a smaller max_ctx than a sequence reaches: the
    step reports LBCA_ERR_CAPACITY on the status word instead of writing past
    the partials it was given; other sequences are unaffected in shape."""
    w = synth.scaled(W["ragged_gqa_decode_append"], ctx=(100, 200), batch=16, steps=1)
    lens = synth.contexts(w)
    lens[3] = 60000  # far beyond the max_ctx below: its segments span more CTAs than any grid leaves room for
    inp = synth.make(w, lens=lens)
    run = DecodeRun(L, w, inp)
    small = 300
    assert L.lbca_decode_step_form(run.cfg, run.B, small) == L.LBCA_STEP_PERSISTENT
    run.max_ctx = small
    run.step_ws = torch.zeros(L.lbca_decode_step_workspace_bytes(run.cfg, run.B, small), dtype=torch.uint8,
                              device="cuda")
    got = fused_step(run)
    torch.cuda.synchronize()
    assert int(run.status.item()) == L.LBCA_ERR_CAPACITY
    assert got.shape == (16, w.n_q_heads, w.head_dim)
