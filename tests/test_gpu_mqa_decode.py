"""Decode of the shared-entry (MQA, HCA) form on the tensor-core path.

bf16 shapes with 64 query heads per kv head and head_dim 256 or 512 take the
tcgen05 kernel (entry tiles as the M operand, one cluster per sequence and kv
head, merge in distributed shared memory).  Every case here runs through the
C ABI on seeded inputs and is compared element by element with the fp64
oracle: ragged batches that put 0, 1, 15, 16, 17, 127, 128 ... entries into
a CTA's chunk, the variants of the form (no sink, no RMSNorm, no RoPE, RoPE
dims that split a 16-byte chunk, D = 256, two kv heads, no window), a
sequence whose visible list fills every CTA of a 16-CTA cluster with exactly
128 entries, an empty sequence, and the one-launch step entry point.
"""
import numpy as np
import pytest
import torch

from block_compressed_long_b200 import synth
from lbca_cases import DecodeRun, assert_close, f64, fused_step, lib, oracle_decode

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS["hca_mqa_decode_128k"]


@pytest.fixture(scope="module")
def L():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib()


def _inputs(w, lens, steps):
    """Inputs whose every row is drawn, then the per-sequence cached lengths."""
    top = int(max(lens))
    w = synth.scaled(w, ctx=(top, top), batch=len(lens), steps=steps)
    inp = synth.make(w)
    inp.lens = np.asarray(lens, dtype=np.int64)
    return w, inp


def _check_steps(L, w, lens, steps, what):
    """Every step of every sequence against the oracle, with the plain bf16
    bound whatever the length of its visible list (1 entry up)."""
    w, inp = _inputs(w, lens, steps)
    run = DecodeRun(L, w, inp, steps=steps)
    for s in range(steps):
        got = f64(run.step())
        torch.cuda.synchronize()
        assert_close(got, oracle_decode(w, inp, s), "bf16", f"{what} step {s}")
    assert int(run.status.item()) == 0


def test_ragged_chunk_sizes(L):
    """Visible lists of 1 ... ~2000 entries in one batch: chunks of 0 to 128
    rows, pooled and raw rows in the same chunk, ring wrap-around."""
    lens = [0, 1, 4, 15, 16, 17, 127, 128, 255, 256, 300, 1000, 2900, 131072 // 64]
    _check_steps(L, W, lens, 2, "hca ragged")


@pytest.mark.parametrize("kw", [
    dict(sink="none"),
    dict(rmsnorm=False),
    dict(rope_dims=0),
    dict(rope_dims=6),
    dict(head_dim=256),
    dict(n_kv_heads=2, n_q_heads=128),
    dict(n_win=0, block_m=64),
    dict(sink="zero", rope_dims=512),
], ids=["no-sink", "no-rmsnorm", "no-rope", "rope6", "d256", "two-kv-heads", "no-window", "full-rope"])
def test_form_variants(L, kw):
    _check_steps(L, synth.scaled(W, **kw), [50, 700, 2100], 2, f"hca {kw}")


def test_full_tiles_in_a_16_cta_cluster(L):
    """m = 16, n_win = 16 and 32303 tokens give 2017 pooled + 31 raw = 2048
    visible entries: 16 CTAs with 128 entries each (the largest chunk)."""
    w = synth.scaled(W, block_m=16, n_win=16)
    _check_steps(L, w, [32300], 3, "hca 2048 entries")


def test_empty_sequence_gives_zeros(L):
    """No visible entry: zeros, with or without the sink in the denominator."""
    w, inp = _inputs(W, [0, 0], 1)
    run = DecodeRun(L, w, inp, steps=1)
    run.cache.seq_lens.zero_()
    for sink in (None, run.sink):
        out = torch.full((2, w.n_q_heads, w.head_dim), 3.0, dtype=torch.bfloat16, device="cuda")
        L.lbca_decode(run.cfg, run.q[0], run.cache, sink, None, None, out, run.ws, 1, run.status)
        torch.cuda.synchronize()
        assert torch.all(out == 0)
    assert int(run.status.item()) == 0


def _cache_equal(x, y, what):
    for name in ("pooled_k", "ring_k", "pool_state", "seq_lens"):
        assert torch.equal(getattr(x.cache, name), getattr(y.cache, name)), f"{what}: {name}"


@pytest.mark.parametrize("kw", [dict(), dict(head_dim=256, rmsnorm=False, sink="none")], ids=["hca", "d256"])
def test_step_entry_point_equals_append_then_decode(L, kw):
    """lbca_decode_step on this form is one launch, the append done by the CTA
    that holds the newest visible row: output, ring, pooled entries, running
    pool state and lengths bit-identical to lbca_append then lbca_decode.  The
    lengths put steps on a block's last token (an entry finishes), on a block's
    first token (the running state restarts), in a one-CTA list and in lists
    split over the cluster."""
    w = synth.scaled(W, **kw)
    assert L.lbca_decode_step_launches(L.config(**_cfg_kw(w)), 5, 3000) == 1
    assert L.lbca_decode_step_form(L.config(**_cfg_kw(w)), 5, 3000) == L.LBCA_STEP_SHARED_TC
    w, inp = _inputs(w, [383, 1500, 40, 255, 2900], 3)
    a = DecodeRun(L, w, inp, steps=3)
    b = DecodeRun(L, w, inp, steps=3)
    for s in range(3):
        x = a.step()
        y = fused_step(b)
        torch.cuda.synchronize()
        assert torch.equal(x, y), f"step {s}"
        _cache_equal(a, b, f"step {s}")
        assert_close(f64(y), oracle_decode(w, inp, s), "bf16", f"step {s}")
    assert int(a.status.item()) == 0 and int(b.status.item()) == 0


def _cfg_kw(w):
    return dict(n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, shared_kv=w.shared_kv,
                block_m=w.block_m, n_win=w.n_win, rope_dims=w.rope_dims, rmsnorm=w.rmsnorm)


def test_step_with_two_kv_heads_takes_two_calls(L):
    """Two kv heads of the shared form: the step runs append then decode and
    still matches the oracle."""
    w = synth.scaled(W, n_kv_heads=2, n_q_heads=128)
    assert L.lbca_decode_step_launches(L.config(**_cfg_kw(w)), 2, 3000) == 2
    w, inp = _inputs(w, [383, 700], 2)
    run = DecodeRun(L, w, inp, steps=2)
    for s in range(2):
        y = fused_step(run)
        torch.cuda.synchronize()
        assert_close(f64(y), oracle_decode(w, inp, s), "bf16", f"step {s}")
    assert int(run.status.item()) == 0


def test_entry_beyond_fp16_range_sets_status(L):
    """Without RMSNorm a shared entry keeps its input's magnitude; a window
    entry beyond the fp16 range of the tensor-core operands sets the status
    word to LBCA_ERR_UNSUPPORTED instead of silently becoming inf."""
    w, inp = _inputs(synth.scaled(W, rmsnorm=False), [300, 300], 1)
    inp.k[1, 290, 0, 33] = 70000.0  # inside the raw window of the query at 300
    run = DecodeRun(L, w, inp, steps=1)
    run.step()
    torch.cuda.synchronize()
    assert int(run.status.item()) == L.LBCA_ERR_UNSUPPORTED


def test_step_full_size_sampled(L):
    """lbca_decode_step in its fused tensor-core form (the launch the HCA bench
    times) at the full 8 x 128K size: two steps, outputs of sampled sequences
    against the oracle."""
    w = synth.scaled(W, steps=2)
    inp = synth.make(w)
    run = DecodeRun(L, w, inp, steps=2)
    assert L.lbca_decode_step_form(run.cfg, run.B, run.max_ctx) == L.LBCA_STEP_SHARED_TC
    for s in range(2):
        got = fused_step(run)
    torch.cuda.synchronize()
    assert_close(f64(got)[[0, 3, 7]], oracle_decode(w, inp, 1, [0, 3, 7]), "bf16", "hca step full size")
    assert int(run.status.item()) == 0
