"""Checkpoint and resume of a decode cache: the cache is plain device memory
the caller owns (pooled entries, raw window, open-block pooling state,
lengths), so copying it out between steps and back into fresh memory resumes
the stream exactly.  Steps run after a restore must be bit-identical to the
same steps run without the interruption, in every step form."""
import pytest
import torch

from block_compressed_long_b200 import synth
from lbca_cases import DecodeRun, f64, assert_close, fused_step, lib, oracle_decode

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS
FIELDS = ("pooled_k", "pooled_v", "ring_k", "ring_v", "pool_state", "seq_lens")


@pytest.fixture(scope="module")
def L():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib()


def _snapshot(cache):
    return {f: None if getattr(cache, f) is None else getattr(cache, f).cpu().clone() for f in FIELDS}


def _restore(cache, snap):
    for f in FIELDS:
        t = getattr(cache, f)
        if t is not None:
            t.copy_(snap[f].to(t.device))


@pytest.mark.parametrize("name,kw", [
    ("gqa_decode_32k", dict(ctx=(1000, 1000))),                       # cluster step
    ("ragged_gqa_decode_append", dict(ctx=(50, 900), batch=16)),      # persistent step
    ("hca_mqa_decode_128k", dict(ctx=(300, 700), batch=3)),           # tensor-core shared-entry step
])
def test_resume_from_a_cache_snapshot_is_bit_exact(L, name, kw):
    steps, cut = 70, 33   # the blocks of m = 64 / 128 complete on both sides of the cut
    w = synth.scaled(W[name], steps=steps, **kw)
    inp = synth.make(w)
    a = DecodeRun(L, w, inp)
    outs_a = [fused_step(a) for _ in range(steps)]
    b = DecodeRun(L, w, inp)
    for _ in range(cut):
        fused_step(b)
    torch.cuda.synchronize()
    snap = _snapshot(b.cache)
    for f in FIELDS:  # wipe the live cache: the resumed run must need nothing but the snapshot
        t = getattr(b.cache, f)
        if t is not None:
            t.fill_(0)
    _restore(b.cache, snap)
    for s in range(cut, steps):
        got = fused_step(b)
        assert torch.equal(got, outs_a[s]), f"{name}: step {s} after the restore differs"
    torch.cuda.synchronize()
    for f in FIELDS:
        x, y = getattr(a.cache, f), getattr(b.cache, f)
        assert (x is None and y is None) or torch.equal(x, y), f
    assert_close(f64(outs_a[-1]), oracle_decode(w, inp, steps - 1), w.dtype, f"{name} last step")
    assert int(a.status.item()) == 0 and int(b.status.item()) == 0
