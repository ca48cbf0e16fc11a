"""GPU parity of the CSA path (CSA page, "What is implemented") through the C
ABI against the fp64 oracle on the same seeded inputs: dual overlapped pooling
(Eqs 9-12) of the shared entries and of the indexer keys."""
import numpy as np
import pytest
import torch

from block_compressed_long_b200 import synth
from lbca_cases import assert_close, assert_close_stored, f64, lcfg, lib, ocfg
from oracle import oracle as orc

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS["csa_sparse_decode_64k"]


@pytest.fixture(scope="module")
def L():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib()


def _pool_dual_gpu(L, cfg, series, xa, za, xb, zb, bpa, bpb, ob):
    B, T, G, D = xa.shape
    out = torch.full((B, G, ob, D), 7.0, dtype=xa.dtype, device="cuda")
    d = lambda t: t.contiguous().cuda()  # noqa: E731
    L.lbca_pool_dual(cfg, series, d(xa), d(za), d(xb), d(zb), d(bpa), d(bpb), None, out)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("kw", [
    dict(ctx=(4 * 300 + 3, 4 * 300 + 3), batch=2),                   # the CSA shapes, a ragged tail
    dict(ctx=(64 * 9, 64 * 9), batch=1, block_m=64),                  # long blocks
    dict(ctx=(16 * 40 + 5, 16 * 40 + 5), batch=3, rmsnorm=False, rope_dims=6, n_kv_heads=2, n_q_heads=128,
         head_dim=128),                                               # two heads, RoPE dims inside a vector
    dict(ctx=(4 * 70, 4 * 70), batch=2, dtype="f32", head_dim=64, n_q_heads=64),   # f32 I/O
    dict(ctx=(3, 3), batch=1),                                        # no complete block
], ids=["csa", "m64", "gqa2", "f32", "empty"])
@pytest.mark.parametrize("series", [0, 1], ids=["key", "value"])
def test_pool_dual_matches_oracle(L, kw, series):
    w = synth.scaled(W, steps=0, index_heads=0, **kw)
    inp = synth.make(w)
    T = int(inp.lens.max())
    cfg = lcfg(L, w)
    xa, za = inp.k[:, :T], inp.zk[:, :T]
    xb, zb = inp.csa["kb"][:, :T], inp.csa["zkb"][:, :T]
    nb = T // w.block_m
    out = _pool_dual_gpu(L, cfg, series, xa, za, xb, zb, inp.bpos_k, inp.csa["bpos_kb"], nb + 2)
    got = f64(out[:, :, :nb]).transpose(0, 2, 1, 3)
    want = orc.pool_dual(ocfg(w), series, f64(xa), f64(za), f64(xb), f64(zb), f64(inp.bpos_k),
                         f64(inp.csa["bpos_kb"]))
    if nb:
        assert_close_stored(got, want, w.dtype, f"dual pool {kw} series {series}")
    assert np.all(f64(out[:, :, nb:]) == 7.0), "pool wrote outside its entries"


def test_pool_dual_indexer_keys_full_size_sampled(L):
    """The indexer key series of the full workload (4 x 64K tokens, 128 dims),
    pooled as values; sampled entries against the oracle."""
    w = synth.scaled(W, steps=1)
    inp = synth.make(w)
    T = int(inp.lens.max())
    c = inp.csa
    cfg = L.config(1, 1, w.index_dim, True, w.block_m, w.n_win, 0, False, dtype=w.dtype)
    nb = T // w.block_m
    out = _pool_dual_gpu(L, cfg, 1, c["ika"][:, :T], c["izka"][:, :T], c["ikb"][:, :T], c["izkb"][:, :T],
                         c["ibpa"], c["ibpb"], nb)
    oc = orc.Config(1, 1, w.index_dim, True, w.block_m, w.n_win)
    for b in range(w.batch):
        for j0 in (0, 7, nb // 2, nb - 3):
            sl = slice(max(0, (j0 - 1) * w.block_m), (j0 + 3) * w.block_m)
            want = orc.pool_dual(oc, 1, f64(c["ika"][b:b + 1, sl]), f64(c["izka"][b:b + 1, sl]),
                                 f64(c["ikb"][b:b + 1, sl]), f64(c["izkb"][b:b + 1, sl]), f64(c["ibpa"]),
                                 f64(c["ibpb"]))[0, :, 0]
            first = 0 if j0 == 0 else 1  # a window starting one block early re-creates entry j0's preceding block
            got = f64(out[b, 0, j0:j0 + 3])
            assert_close_stored(got, want[first:first + 3], w.dtype, f"indexer keys b{b} j{j0}")


# ------------------------------------------------ indexer top-k and sparse decode ----
class CsaRun:
    """A CSA cache on the GPU built through the C ABI from the seeded inputs:
    dual-pooled finalised entries (pooled_k), dual-pooled indexer keys, the raw
    window (the a-series raw entries of the last ring_slots tokens, token s in
    slot s % ring_slots) and the lengths."""

    def __init__(self, L, w, inp):
        self.L, self.w, self.inp = L, w, inp
        self.cfg = lcfg(L, w)
        self.B = w.batch
        self.lens = np.asarray(inp.lens, dtype=np.int64)
        Lmax = int(self.lens.max())
        self.cache = L.Cache.allocate(self.cfg, self.B, Lmax + 1)
        nb = self.cache.max_blocks
        c = inp.csa
        d = lambda t: t.contiguous().cuda()  # noqa: E731
        icfg = L.config(1, 1, w.index_dim, True, w.block_m, w.n_win, 0, False, dtype=w.dtype)
        self.k_idx = torch.zeros(self.B, 1, nb, w.index_dim, dtype=torch.bfloat16, device="cuda")
        for b in range(self.B):
            n = int(self.lens[b])
            sl = lambda t: d(t[b:b + 1, :n])  # noqa: E731
            L.lbca_pool_dual(self.cfg, L.LBCA_KEY, sl(inp.k), sl(inp.zk), sl(c["kb"]), sl(c["zkb"]), d(inp.bpos_k),
                             d(c["bpos_kb"]), None, self.cache.pooled_k[b:b + 1], nb)
            L.lbca_pool_dual(icfg, L.LBCA_VALUE, sl(c["ika"]), sl(c["izka"]), sl(c["ikb"]), sl(c["izkb"]),
                             d(c["ibpa"]), d(c["ibpb"]), None, self.k_idx[b:b + 1], nb)
            R = self.cache.ring_slots
            for s in range(max(0, n - R), n):
                self.cache.ring_k[b, 0, s % R] = inp.k[b, s, 0].cuda()
        self.cache.seq_lens.copy_(torch.as_tensor(self.lens, dtype=torch.int32))
        self.k_idx = self.k_idx[:, 0].contiguous()
        self.ws = torch.zeros(L.lbca_indexer_workspace_bytes(self.B, nb), dtype=torch.uint8, device="cuda")
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def topk(self, step):
        c = self.inp.csa
        sel = torch.full((self.B, self.w.top_k), -7, dtype=torch.int32, device="cuda")
        val = torch.zeros(self.B, self.w.top_k, dtype=torch.float32, device="cuda")
        self.L.lbca_indexer_topk(c["iq"][step].cuda(), c["iw"][step].cuda(), self.k_idx, self.cache.seq_lens,
                                 self.w.block_m, sel, val, self.ws, self.status)
        return sel, val

    def decode(self, step, sel):
        out = torch.empty(self.B, self.w.n_q_heads, self.w.head_dim, dtype=torch.bfloat16, device="cuda")
        self.L.lbca_decode_sparse(self.cfg, self.inp.q[step].cuda(), self.cache, sel, dev(self.inp.sink), None, None,
                                  out, self.status)
        return out


def dev(t):
    return None if t is None else t.cuda()


def _oracle_indexer(w, inp, step, b):
    """fp64 relevance of sequence b's visible blocks from the raw inputs, and the
    per-block bound of the error that storing the pooled keys in bf16 allows:
    sum_h |w_h| 2^-8 sum_d |q_hd| |k_jd| (ReLU is 1-Lipschitz; a bf16 rounding
    moves each key element by at most 2^-9 of it, doubled for the f32
    accumulation and the rounding of k itself near a power of two)."""
    c = inp.csa
    n = int(inp.lens[b])
    oc = orc.Config(1, 1, w.index_dim, True, w.block_m, w.n_win)
    kx = orc.pool_dual(oc, orc.VALUE, *(f64(c[t][b:b + 1, :n]) for t in ("ika", "izka", "ikb", "izkb")),
                       f64(c["ibpa"]), f64(c["ibpb"]))[0, :, 0]
    q, wt = f64(c["iq"][step, b]), f64(c["iw"][step, b])
    nvis = kx.shape[0]
    scores = orc.indexer_scores(q[None], wt[None], kx[None], [nvis])[0]
    bound = (np.abs(kx) @ np.abs(q).T) @ np.abs(wt) * 2.0 ** -8 + 1e-4
    return scores, bound, kx


def _index_order(sel):
    """A selection in increasing block order, padding (-1) last: the layout
    lbca_indexer_topk writes, so equal selections give equal inputs."""
    valid = np.sort(sel[sel >= 0])
    return np.concatenate([valid, np.full(len(sel) - len(valid), -1)]).astype(np.int64)


def _check_selection(sel, val, scores, bound, k, what):
    nvis = len(scores)
    take = min(k, nvis)
    got = [int(j) for j in sel[:take]]
    assert all(int(j) == -1 for j in sel[take:]), f"{what}: padding"
    assert len(set(got)) == take and all(0 <= j < nvis for j in got), f"{what}: not {take} distinct visible blocks"
    assert got == sorted(got), f"{what}: not in increasing index order"
    np.testing.assert_array_less(np.abs(val[:take] - scores[got]), bound[got] + 1e-6, err_msg=f"{what}: relevance")
    if take < nvis:
        kth = np.sort(scores)[::-1][take - 1]
        chosen = np.zeros(nvis, bool)
        chosen[got] = True
        eps = 2 * bound.max()
        assert np.all(scores[chosen] >= kth - eps), f"{what}: a block far below the k-th relevance was chosen"
        assert np.all(chosen[scores > kth + eps]), f"{what}: a block far above the k-th relevance was left out"


@pytest.mark.parametrize("lens,top_k", [([37, 1200, 4099], 64), ([5, 600, 2000], 700), ([3, 4, 130], 16)],
                         ids=["ragged", "k-above-visible", "tiny"])
def test_indexer_topk_and_sparse_decode_match_oracle(L, lens, top_k):
    w = synth.scaled(W, batch=len(lens), ctx=(max(lens), max(lens)), steps=2, top_k=top_k)
    inp = synth.make(w, lens=np.asarray(lens))
    run = CsaRun(L, w, inp)
    oc = ocfg(w)
    for step in range(2):
        sel, val = run.topk(step)
        torch.cuda.synchronize()
        sel_h, val_h = sel.cpu().numpy(), val.cpu().numpy()
        osel = np.full((w.batch, top_k), -1, dtype=np.int32)
        for b in range(w.batch):
            scores, bound, _ = _oracle_indexer(w, inp, step, b)
            _check_selection(sel_h[b], val_h[b], scores, bound, top_k, f"step {step} seq {b}")
            osel[b] = _index_order(orc.topk_blocks(scores[None], [len(scores)], top_k)[0])
        # the attention step on the oracle's selection, both sides
        out = run.decode(step, torch.as_tensor(osel, device="cuda"))
        torch.cuda.synchronize()
        for b in range(w.batch):
            n = int(inp.lens[b])
            ek = orc.pool_dual(oc, orc.KEY, f64(inp.k[b:b + 1, :n]), f64(inp.zk[b:b + 1, :n]),
                               f64(inp.csa["kb"][b:b + 1, :n]), f64(inp.csa["zkb"][b:b + 1, :n]), f64(inp.bpos_k),
                               f64(inp.csa["bpos_kb"]))
            want = orc.attend_sparse(oc, f64(inp.q[step, b:b + 1]), ek, osel[b:b + 1].astype(np.int64),
                                     f64(inp.k[b:b + 1, :n]), [n], f64(inp.sink))
            assert_close(f64(out[b:b + 1]), want, "bf16", f"sparse decode step {step} seq {b}")
    assert int(run.status.item()) == 0


def test_csa_full_size_sampled(L):
    """The CSA workload at full size (4 x 64K tokens, 16384 blocks per
    sequence, top-512): selection validity and the sparse attention of sampled
    sequences against the oracle."""
    w = synth.scaled(W, steps=1)
    inp = synth.make(w)
    run = CsaRun(L, w, inp)
    sel, val = run.topk(0)
    out = run.decode(0, sel)
    torch.cuda.synchronize()
    oc = ocfg(w)
    for b in (0, 3):
        scores, bound, _ = _oracle_indexer(w, inp, 0, b)
        _check_selection(sel[b].cpu().numpy(), val[b].cpu().numpy(), scores, bound, w.top_k, f"full seq {b}")
        # the attention of the GPU's (validated) selection against the oracle, on the oracle's selection too
        osel = _index_order(orc.topk_blocks(scores[None], [len(scores)], w.top_k)[0])[None]
        n = int(inp.lens[b])
        ek = orc.pool_dual(oc, orc.KEY, f64(inp.k[b:b + 1, :n]), f64(inp.zk[b:b + 1, :n]),
                           f64(inp.csa["kb"][b:b + 1, :n]), f64(inp.csa["zkb"][b:b + 1, :n]), f64(inp.bpos_k),
                           f64(inp.csa["bpos_kb"]))
        out_o = run.decode(0, torch.as_tensor(np.repeat(osel, w.batch, 0).astype(np.int32), device="cuda"))
        torch.cuda.synchronize()
        want = orc.attend_sparse(oc, f64(inp.q[0, b:b + 1]), ek, osel, f64(inp.k[b:b + 1, :n]), [n], f64(inp.sink))
        assert_close(f64(out_o[b:b + 1]), want, "bf16", f"full sparse decode seq {b}")
        if np.array_equal(np.sort(sel[b].cpu().numpy()), np.sort(osel[0])):
            assert torch.equal(out[b], out_o[b])
    assert int(run.status.item()) == 0


def test_sparse_decode_rejects_shapes_off_the_tensor_cores(L):
    w = synth.scaled(W, batch=1, ctx=(64, 64), steps=1, n_q_heads=32)
    cfg = lcfg(L, w)
    cache = L.Cache.allocate(cfg, 1, 65)
    q = torch.zeros(1, 32, w.head_dim, dtype=torch.bfloat16, device="cuda")
    sel = torch.zeros(1, 8, dtype=torch.int32, device="cuda")
    with pytest.raises(L.LbcaError) as e:
        L.lbca_decode_sparse(cfg, q, cache, sel, None, None, None, torch.empty_like(q))
    assert e.value.status == L.LBCA_ERR_UNSUPPORTED
