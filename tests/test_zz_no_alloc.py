"""lbca_decode_noalloc: decode for callers that may not allocate device memory.

Such callers (a host framework that owns every device allocation, a serving
loop that must not allocate once running) cannot hand lbca_decode a workspace;
this entry point keeps its split partials in the library's own static device
scratch instead (the shared-entry tensor-core form needs none).  Checked here
through the C ABI against the fp64 oracle and against lbca_decode on the same
cache (the same kernels and plan: bit-identical), on two calls in a row (the
second finds the scratch holding the first call's contents), for the
shared-entry form at its full size (a batch whose CUDA-core split plan would
not fit the scratch), and for the clear error on a request larger than the
scratch.  This file is collected last on purpose.
"""
import pytest
import torch

from block_compressed_long_b200 import synth
from lbca_cases import DecodeRun, assert_close, f64, lib, oracle_decode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib()


def _two_calls_per_step(L, name, w, seqs=None):
    inp = synth.make(w)
    run = DecodeRun(L, w, inp, steps=w.steps)
    for step in range(w.steps):
        L.lbca_append(run.cfg, run.token(run.k), run.token(run.v), run.token(run.zk), run.token(run.zv),
                      run.bpk, run.bpv, None, run.cache, run.status)
        run.pos += 1
        want = torch.empty(run.B, w.n_q_heads, w.head_dim, dtype=torch.bfloat16, device="cuda")
        L.lbca_decode(run.cfg, run.q[step], run.cache, run.sink, None, None, want, run.ws, run.max_ctx, run.status)
        outs = []
        for _ in range(2):  # two calls in a row on the shared scratch
            got = torch.full_like(want, 5.0)
            L.lbca_decode_noalloc(run.cfg, run.q[step], run.cache, run.sink, None, None, got, run.max_ctx,
                                  run.status)
            outs.append(got)
        torch.cuda.synchronize()
        pick = list(range(run.B)) if seqs is None else seqs
        oracle = oracle_decode(w, inp, step, pick)
        for i, got in enumerate(outs):
            assert torch.equal(got, want), f"{name} step {step} call {i}: differs from lbca_decode"
            assert_close(f64(got)[pick], oracle, "bf16", f"{name} step {step} call {i}")
    assert int(run.status.item()) == 0


@pytest.mark.parametrize("name,kw", [
    ("gqa_decode_32k", dict(ctx=(3000, 3000))),
    ("ragged_gqa_decode_append", dict(ctx=(100, 2500), batch=6)),
])
def test_noalloc_matches_oracle_and_workspace_decode_twice(L, name, kw):
    _two_calls_per_step(L, name, synth.scaled(synth.WORKLOADS[name], steps=2, **kw))


def test_noalloc_shared_entry_full_size(L):
    """The HCA form at full size (8 x 128K, 64 heads on one 512-dim entry):
    the tensor-core kernel, which needs no scratch, runs although the CUDA-core
    split plan for this batch would need more than the static scratch holds."""
    w = synth.scaled(synth.WORKLOADS["hca_mqa_decode_128k"], steps=2)
    cfg = L.config(w.n_q_heads, w.n_kv_heads, w.head_dim, w.shared_kv, w.block_m, w.n_win, w.rope_dims,
                   w.rmsnorm, w.rope_theta, dtype=w.dtype)
    assert L.lbca_decode_workspace_bytes(cfg, w.batch, w.ctx[1] + w.steps) > 8 << 20
    _two_calls_per_step(L, "hca full", w, seqs=[0, 7])


def test_noalloc_rejects_requests_beyond_its_scratch(L):
    """A batch whose split partials exceed the static scratch is refused with
    LBCA_ERR_CAPACITY before anything is launched."""
    w = synth.scaled(synth.WORKLOADS["ragged_gqa_decode_append"], ctx=(10, 20), batch=2, steps=1)
    cfg = L.config(w.n_q_heads, w.n_kv_heads, w.head_dim, w.shared_kv, w.block_m, w.n_win, w.rope_dims,
                   dtype=w.dtype)
    big = 8
    cache = L.Cache.allocate(cfg, big, 64)
    q = torch.zeros(big, w.n_q_heads, w.head_dim, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    need = L.lbca_decode_workspace_bytes(cfg, big, 1 << 20)
    assert need > 8 << 20
    with pytest.raises(L.LbcaError) as e:
        L.lbca_decode_noalloc(cfg, q, cache, None, None, None, out, 1 << 20)
    assert e.value.status == L.LBCA_ERR_CAPACITY
