"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the
same seeded inputs.  Small cases span several tiles, blocks and a ragged
tail; the workloads' full sizes are checked on sampled outputs."""
import numpy as np
import pytest
import torch

from block_compressed_long_b200 import synth
from lbca_cases import (DecodeRun, assert_close, assert_close_stored, f64, gpu_prefill, lcfg, lib, ocfg, oracle_decode,
                        oracle_prefill)
from oracle import oracle as orc

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS


@pytest.fixture(scope="module")
def L():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib()


# ---------------------------------------------------------------- pool ----
POOL_CASES = [
    ("tiny_f32_prefill", dict(seq_len=16 * 7 + 5)),
    ("gqa_decode_32k", dict(seq_len=64 * 5 + 17)),
    ("gqa_prefill_16k", dict(seq_len=16 * 9 + 3)),
    ("hca_mqa_decode_128k", dict(seq_len=128 * 4 + 100, batch=3)),
    ("ragged_gqa_decode_append", dict(seq_len=64 * 3, batch=2)),
    # more blocks than the GPU holds CTAs at once, and a ragged tail
    ("gqa_prefill_16k", dict(seq_len=16 * 1100 + 5, batch=1)),
]


@pytest.mark.parametrize("name,kw", POOL_CASES)
@pytest.mark.parametrize("pos0_blocks", [0, 3])
def test_pool_matches_oracle(L, name, kw, pos0_blocks):
    w = synth.scaled(W[name], kind="prefill", **kw)
    inp = synth.make(w)
    cfg = lcfg(L, w)
    m = w.block_m
    B, T = inp.k.shape[:2]
    nb = T // m
    ob = pos0_blocks + nb + 2
    series = [(0, inp.k, inp.zk, inp.bpos_k)] + ([] if w.shared_kv else [(1, inp.v, inp.zv, inp.bpos_v)])
    outs = []
    for s, x, z, bp in series:
        out = torch.full((B, w.n_kv_heads, ob, w.head_dim), 7.0, dtype=L.torch_dtype(cfg), device="cuda")
        outs.append(out)
        L.lbca_pool(cfg, s, x.cuda(), z.cuda(), bp.cuda(), None, out, pos0=pos0_blocks * m)
        torch.cuda.synchronize()
        want = orc.pool(ocfg(w), s, f64(x), f64(z), f64(bp), None, pos0=pos0_blocks * m)  # [B, nb, G, D]
        got = f64(out[:, :, pos0_blocks:pos0_blocks + nb]).transpose(0, 2, 1, 3)
        assert_close_stored(got, want, w.dtype, f"{name} series {s}")
        untouched = f64(out[:, :, :pos0_blocks]), f64(out[:, :, pos0_blocks + nb:])
        assert all(np.all(u == 7.0) for u in untouched), "pool wrote outside its blocks"
        # the f32 form: the same entries before their one rounding to the I/O dtype
        o32 = torch.full((B, w.n_kv_heads, ob, w.head_dim), 7.0, dtype=torch.float32, device="cuda")
        L.lbca_pool_f32(cfg, s, x.cuda(), z.cuda(), bp.cuda(), None, o32, pos0=pos0_blocks * m)
        torch.cuda.synchronize()
        assert torch.equal(o32.to(out.dtype), out), f"{name} series {s}: f32 entries round to other values"
        g32 = f64(o32[:, :, pos0_blocks:pos0_blocks + nb]).transpose(0, 2, 1, 3)
        scale = max(float(np.abs(want).max()), 1e-30)
        assert np.abs(g32 - want).max() <= 1e-5 * scale, f"{name} series {s}: f32 entries"
        assert np.all(f64(o32[:, :, pos0_blocks + nb:]) == 7.0) and np.all(f64(o32[:, :, :pos0_blocks]) == 7.0)
    if not w.shared_kv:  # both series in one launch: the same entries, bit for bit, and nothing else written
        pk, pv = torch.full_like(outs[0], 7.0), torch.full_like(outs[1], 7.0)
        L.lbca_pool_kv(cfg, inp.k.cuda(), inp.v.cuda(), inp.zk.cuda(), inp.zv.cuda(), inp.bpos_k.cuda(),
                       inp.bpos_v.cuda(), None, pk, pv, pos0=pos0_blocks * m)
        torch.cuda.synchronize()
        assert torch.equal(pk, outs[0]) and torch.equal(pv, outs[1]), f"{name}: lbca_pool_kv"


# ------------------------------------------------------------- prefill ----
def test_prefill_tiny_f32_full(L):
    """The tiny f32 workload at full size, every row, relative 1e-5."""
    w = W["tiny_f32_prefill"]
    inp = synth.make(w)
    got = gpu_prefill(L, w, inp)
    torch.cuda.synchronize()
    assert_close(f64(got), oracle_prefill(w, inp), "f32", "tiny f32 prefill")


@pytest.mark.parametrize("name,kw", [
    ("gqa_prefill_16k", dict(seq_len=700)),
    ("gqa_prefill_16k", dict(seq_len=700, n_win=0)),
    ("gqa_prefill_16k", dict(seq_len=333, block_m=1, n_win=5)),
    ("gqa_prefill_16k", dict(seq_len=300, block_m=64, n_win=3)),
    ("hca_mqa_decode_128k", dict(kind="prefill", seq_len=600, batch=2)),
    ("tiny_f32_prefill", dict(seq_len=200, n_win=7, block_m=5)),
    ("tiny_f32_prefill", dict(seq_len=130, rope_dims=16, rmsnorm=True, sink="normal", n_kv_heads=2,
                              shared_kv=False)),
])
def test_prefill_small_all_rows(L, name, kw):
    w = synth.scaled(W[name], **kw)
    inp = synth.make(w)
    got = gpu_prefill(L, w, inp)
    torch.cuda.synchronize()
    assert_close(f64(got), oracle_prefill(w, inp), w.dtype, f"{name} {kw}")


def test_prefill_gqa_full_sampled_rows(L):
    """The 16K-token GQA prefill in its own launch configuration; rows sampled
    at the start, around block and window edges, and at the end."""
    w = W["gqa_prefill_16k"]
    inp = synth.make(w)
    got = gpu_prefill(L, w, inp)
    torch.cuda.synchronize()
    T = w.seq_len
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 143, 144, 145, 4095, 8191, T - 17, T - 1],
                                     rng.integers(0, T, 24)]))
    want = oracle_prefill(w, inp, rows=rows)
    assert_close(f64(got)[:, rows], want, "bf16", "gqa prefill 16k sampled")


# -------------------------------------------------------------- decode ----
@pytest.mark.parametrize("name,kw,steps", [
    ("gqa_decode_32k", dict(ctx=(3000, 3000)), 70),
    ("gqa_decode_32k", dict(ctx=(500, 500), n_win=0), 66),
    ("hca_mqa_decode_128k", dict(ctx=(1000, 1000), batch=2), 130),
    ("ragged_gqa_decode_append", dict(ctx=(100, 2500), batch=6), 70),
    ("ragged_gqa_decode_append", dict(ctx=(0, 40), batch=5, n_win=16, block_m=8), 20),
])
def test_decode_steps_match_oracle(L, name, kw, steps):
    """Append + decode for enough steps that every sequence completes a block;
    every step is checked against the oracle."""
    w = synth.scaled(W[name], steps=steps, **kw)
    inp = synth.make(w)
    run = DecodeRun(L, w, inp)
    for s in range(steps):
        got = run.step()
        if s % 7 == 0 or s == steps - 1:
            torch.cuda.synchronize()
            assert_close(f64(got), oracle_decode(w, inp, s), w.dtype, f"{name} step {s}")
    assert int(run.status.item()) == 0


@pytest.mark.parametrize("name,steps,seqs", [
    ("gqa_decode_32k", 2, None),
    ("hca_mqa_decode_128k", 2, [0, 7]),
    ("ragged_gqa_decode_append", 1, [0, 5, 31]),
])
def test_decode_full_size_sampled(L, name, steps, seqs):
    """The decode workloads at full size in their own launch configuration;
    outputs checked for sampled sequences."""
    w = synth.scaled(W[name], steps=steps)
    inp = synth.make(w)
    run = DecodeRun(L, w, inp)
    for s in range(steps):
        got = run.step()
    torch.cuda.synchronize()
    pick = list(range(inp.k.shape[0])) if seqs is None else seqs
    assert_close(f64(got)[pick], oracle_decode(w, inp, steps - 1, pick), "bf16", f"{name} full")
    assert int(run.status.item()) == 0


def test_stream_equals_prefill_rows(L):
    """prefill(T) into the cache, then k (append, decode) steps, reproduces
    rows T..T+k-1 of prefill(T+k) (and both match the oracle)."""
    w = synth.scaled(W["gqa_decode_32k"], kind="prefill", seq_len=1000 + 90, ctx=(1000, 1000), steps=90)
    inp = synth.make(w)
    full = f64(gpu_prefill(L, w, inp))
    wd = synth.scaled(w, kind="decode")
    dinp = synth.Inputs(inp.q[0, 1000:].unsqueeze(1).contiguous(), inp.k, inp.v, inp.zk, inp.zv, inp.bpos_k,
                        inp.bpos_v, inp.sink, np.array([1000]))
    run = DecodeRun(L, wd, dinp, steps=90)
    outs = np.stack([f64(run.step())[0] for _ in range(90)])
    torch.cuda.synchronize()
    assert_close(outs, full[0, 1000:1090], "bf16", "stream vs prefill")
    want = oracle_prefill(w, inp, rows=np.arange(1000, 1090))[0]
    assert_close(outs, want, "bf16", "stream vs oracle")


def test_decode_empty_sequence_gives_zeros(L):
    w = synth.scaled(W["ragged_gqa_decode_append"], batch=2, ctx=(0, 0), steps=1)
    inp = synth.make(w)
    run = DecodeRun(L, w, inp, steps=1)
    run.cache.seq_lens.zero_()
    out = torch.full((2, w.n_q_heads, w.head_dim), 3.0, dtype=torch.bfloat16, device="cuda")
    L.lbca_decode(run.cfg, run.q[0], run.cache, None, None, None, out, run.ws, 1, run.status)
    torch.cuda.synchronize()
    assert torch.all(out == 0)


def test_append_beyond_capacity_sets_status(L):
    w = synth.scaled(W["ragged_gqa_decode_append"], batch=1, ctx=(60, 60), steps=10, block_m=16, n_win=4)
    inp = synth.make(w)
    run = DecodeRun(L, w, inp, steps=10)
    run.cache.max_blocks = 3      # 60 tokens already hold 3 complete blocks; the 4th cannot be stored
    for _ in range(5):
        L.lbca_append(run.cfg, run.token(run.k), run.token(run.v), run.token(run.zk), run.token(run.zv),
                      run.bpk, run.bpv, None, run.cache, run.status)
        run.pos += 1
    torch.cuda.synchronize()
    assert int(run.status.item()) == L.LBCA_ERR_CAPACITY


# ----------------------------------------------------- fp16 operand range ----
@pytest.mark.parametrize("where", ["none", "query", "key_in_block", "value_in_tail"])
def test_prefill_fp16_range_sets_status(L, where):
    """The tensor-core prefill multiplies in fp16: a bf16 input beyond the fp16
    range (|x| > 65504) would silently become inf, so it sets the status word
    to LBCA_ERR_UNSUPPORTED -- a query (widened in the kernel), a key of a
    complete block (fp16 copy made by the pool pass), a value past the last
    complete block (fp16 copy of the tail).  In-range inputs leave it zero."""
    w = synth.scaled(W["gqa_prefill_16k"], seq_len=16 * 18 + 7)
    inp = synth.make(w)
    big = 1.0e5  # after any rotation one of its pair's components stays above 65504
    if where == "query":
        inp.q[0, 100, 5, 17] = big
    elif where == "key_in_block":
        inp.k[0, 40, 3, 120] = -big
    elif where == "value_in_tail":
        inp.v[0, 16 * 18 + 3, 6, 2] = big
    cfg = lcfg(L, w)
    B, T = 1, w.seq_len
    out = torch.empty(B, T, w.n_q_heads, w.head_dim, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(L.lbca_prefill_workspace_bytes(cfg, B, T, False), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    d = lambda t: None if t is None else t.cuda()  # noqa: E731
    L.lbca_prefill(cfg, d(inp.q), d(inp.k), d(inp.v), d(inp.zk), d(inp.zv), d(inp.bpos_k), d(inp.bpos_v), None,
                   None, None, out, None, ws, d_status=st)
    torch.cuda.synchronize()
    want = 0 if where == "none" else L.LBCA_ERR_UNSUPPORTED
    assert int(st.item()) == want
    if where == "none":
        assert_close(f64(out), oracle_prefill(w, inp), "bf16", "in-range prefill")


# ---------------------------------------------------------- context parallel ----
@pytest.mark.parametrize("name,kw,world", [
    ("gqa_prefill_16k", dict(seq_len=16 * 40 + 7, n_win=48), 3),
    ("hca_mqa_decode_128k", dict(kind="prefill", seq_len=128 * 5 + 30, block_m=32, n_win=40, batch=2), 2),
    ("tiny_f32_prefill", dict(seq_len=16 * 20 + 5, n_win=24), 3),
])
def test_context_parallel_rows_equal_the_whole_prefill(L, name, kw, world):
    """The ranks' compute of a context-parallel prefill, run one after another
    on this GPU: each pools its own blocks into their slots of one pooled
    buffer (the union is what the all-gather delivers), attends its own rows
    from the pooled prefix and the raw tokens from its halo on
    (lbca_prefill_rows); the rows together match the oracle, and the
    whole-sequence call of the same kernel (whose groups of rows per CTA
    start elsewhere, so the rounding order may differ)."""
    from block_compressed_long_b200 import context_parallel as cp
    w = synth.scaled(W[name], **kw)
    inp = synth.make(w)
    cfg = lcfg(L, w)
    B, T = inp.q.shape[:2]
    p = cp.plan(T, w.block_m, w.n_win, world)
    d = lambda t: None if t is None else t.contiguous().cuda()  # noqa: E731
    pk = torch.zeros(B, w.n_kv_heads, p.blocks, w.head_dim, dtype=torch.float32, device="cuda")
    pv = None if w.shared_kv else torch.zeros_like(pk)
    for r in range(world):
        t0, t1 = p.ranges[r]
        L.lbca_pool_f32(cfg, L.LBCA_KEY, d(inp.k[:, t0:t1]), d(inp.zk[:, t0:t1]), d(inp.bpos_k), None, pk, pos0=t0)
        if not w.shared_kv:
            L.lbca_pool_f32(cfg, L.LBCA_VALUE, d(inp.v[:, t0:t1]), d(inp.zv[:, t0:t1]), d(inp.bpos_v), None, pv,
                            pos0=t0)
    outs = []
    for r in range(world):
        t0, t1 = p.ranges[r]
        lo, _ = p.halo_range(r)
        outs.append(cp.attend_rows(L, cfg, d(inp.q[:, t0:t1]), t0, d(inp.k[:, lo:t1]),
                                   None if w.shared_kv else d(inp.v[:, lo:t1]), lo, pk, pv, d(inp.sink)))
    torch.cuda.synchronize()
    got = f64(torch.cat(outs, dim=1))
    assert_close(got, oracle_prefill(w, inp), w.dtype, f"context parallel {name}")
    # the same rows from one whole-sequence call of the same CUDA-core kernel
    whole = torch.empty_like(d(inp.q))
    L.lbca_prefill_rows(cfg, d(inp.q), 0, d(inp.k), d(inp.v), 0, pk, pv, d(inp.sink), None, None, whole)
    torch.cuda.synchronize()
    assert_close(got, f64(whole), w.dtype, f"context parallel {name} vs one call")


def test_prefill_rows_rejects_a_window_that_starts_too_late(L):
    w = synth.scaled(W["gqa_prefill_16k"], seq_len=16 * 10, n_win=32)
    cfg = lcfg(L, w)
    q = torch.zeros(1, 16, w.n_q_heads, w.head_dim, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(1, 16, w.n_kv_heads, w.head_dim, dtype=torch.bfloat16, device="cuda")
    pk = torch.zeros(1, w.n_kv_heads, 10, w.head_dim, dtype=torch.float32, device="cuda")
    with pytest.raises(L.LbcaError) as e:  # rows 96..111 need raw tokens from 64 on; these start at 96
        L.lbca_prefill_rows(cfg, q, 96, kv, kv, 96, pk, pk, None, None, None, torch.empty_like(q))
    assert e.value.status == L.LBCA_ERR_ARG
