"""Thin ctypes binding of liblbca.so (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
arithmetic of its own: tensors become raw device pointers, the current torch
CUDA stream becomes the ``cudaStream_t``, and a non-OK status raises
``LbcaError``.  PyTorch is used for device memory and streams only.  Importing
this module fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

# LBCA_CHECKED=1 selects the bounds-checked build of the same library
_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                         "liblbca_checked.so" if os.environ.get("LBCA_CHECKED") == "1" else "liblbca.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is not built; run `python -m block_compressed_long_b200.build` "
                      "(needs nvcc) -- there is no CPU fallback")
_lib = ctypes.CDLL(_LIB_PATH)

LBCA_OK, LBCA_ERR_ARG, LBCA_ERR_UNSUPPORTED, LBCA_ERR_CAPACITY, LBCA_ERR_CUDA, LBCA_ERR_TIMEOUT, \
    LBCA_ERR_ALIGN = range(7)
LBCA_F32, LBCA_BF16 = 0, 1
LBCA_KEY, LBCA_VALUE = 0, 1

ENTRY_POINTS = ("lbca_ring_slots", "lbca_pool_state_elems", "lbca_decode_workspace_bytes",
                "lbca_prefill_workspace_bytes", "lbca_pool", "lbca_append", "lbca_decode",
                "lbca_prefill", "lbca_status_string", "lbca_decode_noalloc",
                "lbca_decode_step_workspace_bytes", "lbca_decode_step", "lbca_decode_step_launches",
                "lbca_decode_step_form", "lbca_selftest_bounded_wait", "lbca_pool_dual", "lbca_decode_sparse",
                "lbca_indexer_workspace_bytes", "lbca_indexer_topk", "lbca_prefill_backward_workspace_bytes",
                "lbca_prefill_backward", "lbca_prefill_rows", "lbca_pool_f32", "lbca_pool_kv")


class lbca_config(ctypes.Structure):
    _fields_ = [("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("shared_kv", ctypes.c_int32),
                ("block_m", ctypes.c_int32), ("n_win", ctypes.c_int32),
                ("rope_dims", ctypes.c_int32), ("rmsnorm", ctypes.c_int32),
                ("rope_theta", ctypes.c_double), ("rms_eps", ctypes.c_float),
                ("softmax_scale", ctypes.c_float), ("dtype", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class lbca_cache(ctypes.Structure):
    _fields_ = [("pooled_k", ctypes.c_void_p), ("pooled_v", ctypes.c_void_p),
                ("ring_k", ctypes.c_void_p), ("ring_v", ctypes.c_void_p),
                ("pool_state", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
                ("batch", ctypes.c_int32), ("max_blocks", ctypes.c_int32),
                ("ring_slots", ctypes.c_int32), ("flags", ctypes.c_int32)]

LBCA_CACHE_OVERLAP_PREV = 1


_vp, _i32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
_CP, _KP = ctypes.POINTER(lbca_config), ctypes.POINTER(lbca_cache)
_lib.lbca_ring_slots.argtypes = [_CP]
_lib.lbca_ring_slots.restype = _i32
_lib.lbca_pool_state_elems.argtypes = [_CP, _i32]
_lib.lbca_pool_state_elems.restype = _sz
_lib.lbca_decode_workspace_bytes.argtypes = [_CP, _i32, _i32]
_lib.lbca_decode_workspace_bytes.restype = _sz
_lib.lbca_prefill_workspace_bytes.argtypes = [_CP, _i32, _i32, _i32]
_lib.lbca_prefill_workspace_bytes.restype = _sz
_lib.lbca_pool.argtypes = [_CP, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp, _i32, _vp]
_lib.lbca_pool.restype = ctypes.c_int
_lib.lbca_pool_f32.argtypes = [_CP, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp, _i32, _vp]
_lib.lbca_pool_f32.restype = ctypes.c_int
_lib.lbca_pool_kv.argtypes = [_CP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _i32, _vp]
_lib.lbca_pool_kv.restype = ctypes.c_int
_lib.lbca_pool_dual.argtypes = [_CP, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _i32, _vp]
_lib.lbca_pool_dual.restype = ctypes.c_int
_lib.lbca_append.argtypes = [_CP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _KP, _vp, _vp]
_lib.lbca_append.restype = ctypes.c_int
_lib.lbca_decode.argtypes = [_CP, _vp, _KP, _vp, _vp, _vp, _i32, _vp, _vp, _sz, _vp, _vp]
_lib.lbca_decode.restype = ctypes.c_int
_lib.lbca_prefill.argtypes = [_CP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _vp,
                              _KP, _vp, _sz, _vp, _vp]
_lib.lbca_prefill.restype = ctypes.c_int
_lib.lbca_decode_step_workspace_bytes.argtypes = [_CP, _i32, _i32]
_lib.lbca_decode_step_workspace_bytes.restype = _sz
_lib.lbca_decode_step.argtypes = [_CP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _KP, _vp, _vp, _i32, _vp, _vp, _sz,
                                  _vp, _vp]
_lib.lbca_decode_step.restype = ctypes.c_int
_lib.lbca_decode_step_launches.argtypes = [_CP, _i32, _i32]
_lib.lbca_decode_step_launches.restype = _i32
_lib.lbca_decode_step_form.argtypes = [_CP, _i32, _i32]
_lib.lbca_decode_step_form.restype = _i32
_lib.lbca_decode_noalloc.argtypes = [_CP, _vp, _KP, _vp, _vp, _vp, _i32, _vp, _vp, _vp]
_lib.lbca_decode_noalloc.restype = ctypes.c_int
_lib.lbca_selftest_bounded_wait.argtypes = [_i32, ctypes.c_uint64, _vp, _vp]
_lib.lbca_selftest_bounded_wait.restype = ctypes.c_int
_lib.lbca_decode_sparse.argtypes = [_CP, _vp, _KP, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.lbca_decode_sparse.restype = ctypes.c_int
_lib.lbca_indexer_workspace_bytes.argtypes = [_i32, _i32]
_lib.lbca_indexer_workspace_bytes.restype = _sz
_lib.lbca_indexer_topk.argtypes = [_i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _sz, _vp,
                                   _vp]
_lib.lbca_indexer_topk.restype = ctypes.c_int
_lib.lbca_prefill_backward_workspace_bytes.argtypes = [_CP, _i32, _i32]
_lib.lbca_prefill_backward_workspace_bytes.restype = _sz
_lib.lbca_prefill_backward.argtypes = [_CP] + [_vp] * 11 + [_i32, _i32] + [_vp] * 9 + [_sz, _vp]
_lib.lbca_prefill_backward.restype = ctypes.c_int
_lib.lbca_prefill_rows.argtypes = [_CP, _vp, _i32, _i32, _vp, _vp, _i32, _i32, _vp, _vp, _i32, _vp, _vp, _vp, _i32, _vp,
                                   _vp]
_lib.lbca_prefill_rows.restype = ctypes.c_int
_lib.lbca_status_string.argtypes = [ctypes.c_int]
_lib.lbca_status_string.restype = ctypes.c_char_p


class LbcaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {lbca_status_string(status)} (status {status})")
        self.status = status


def lbca_status_string(status: int) -> str:
    return _lib.lbca_status_string(int(status)).decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(fn: str, st: int):
    if st != LBCA_OK:
        raise LbcaError(fn, st)


def config(n_q_heads, n_kv_heads, head_dim, shared_kv, block_m, n_win, rope_dims=0, rmsnorm=False,
           rope_theta=10000.0, rms_eps=1e-6, softmax_scale=0.0, dtype="bf16") -> lbca_config:
    """Build an ``lbca_config`` (dtype "bf16" or "f32")."""
    return lbca_config(n_q_heads, n_kv_heads, head_dim, int(shared_kv), block_m, n_win, rope_dims,
                       int(rmsnorm), float(rope_theta), float(rms_eps), float(softmax_scale),
                       LBCA_BF16 if dtype == "bf16" else LBCA_F32, 0)


def torch_dtype(cfg: lbca_config):
    return torch.bfloat16 if cfg.dtype == LBCA_BF16 else torch.float32


def lbca_ring_slots(cfg: lbca_config) -> int:
    return int(_lib.lbca_ring_slots(ctypes.byref(cfg)))


def lbca_pool_state_elems(cfg: lbca_config, batch: int) -> int:
    return int(_lib.lbca_pool_state_elems(ctypes.byref(cfg), batch))


def lbca_decode_workspace_bytes(cfg: lbca_config, batch: int, max_ctx: int) -> int:
    return int(_lib.lbca_decode_workspace_bytes(ctypes.byref(cfg), batch, max_ctx))


def lbca_prefill_workspace_bytes(cfg: lbca_config, batch: int, T: int, has_cache: bool) -> int:
    return int(_lib.lbca_prefill_workspace_bytes(ctypes.byref(cfg), batch, T, int(has_cache)))


@dataclass
class Cache:
    """Device tensors of an ``lbca_cache`` (allocated with torch, zero-filled)."""
    cfg: lbca_config
    batch: int
    max_blocks: int
    ring_slots: int
    pooled_k: torch.Tensor
    pooled_v: torch.Tensor | None
    ring_k: torch.Tensor
    ring_v: torch.Tensor | None
    pool_state: torch.Tensor
    seq_lens: torch.Tensor
    flags: int = 0  # LBCA_CACHE_OVERLAP_PREV: steps may read this cache while the preceding kernel drains

    @staticmethod
    def allocate(cfg: lbca_config, batch: int, max_ctx: int, device="cuda") -> "Cache":
        G, D = cfg.n_kv_heads, cfg.head_dim
        dt = torch_dtype(cfg)
        nb = max(1, max_ctx // cfg.block_m)
        R = lbca_ring_slots(cfg)
        shared = bool(cfg.shared_kv)
        z = lambda *s, dtype=dt: torch.zeros(*s, dtype=dtype, device=device)  # noqa: E731
        return Cache(cfg, batch, nb, R, z(batch, G, nb, D), None if shared else z(batch, G, nb, D),
                     z(batch, G, R, D), None if shared else z(batch, G, R, D),
                     z(lbca_pool_state_elems(cfg, batch), dtype=torch.float32),
                     z(batch, dtype=torch.int32))

    def __setattr__(self, name, value):
        object.__setattr__(self, name, value)
        if name != "_c":
            object.__setattr__(self, "_c", None)  # any field change rebuilds the C struct

    def c(self) -> lbca_cache:
        """The C struct (built once, rebuilt after any field change: a decode loop
        pays the marshalling of its cache once)."""
        cc = self.__dict__.get("_c")
        if cc is None:
            cc = lbca_cache(_ptr(self.pooled_k), _ptr(self.pooled_v), _ptr(self.ring_k), _ptr(self.ring_v),
                            _ptr(self.pool_state), _ptr(self.seq_lens), self.batch, self.max_blocks,
                            self.ring_slots, self.flags)
            object.__setattr__(self, "_c", cc)
        return cc


def lbca_pool(cfg, series, x, z, b_pos, gamma, out, pos0=0, out_blocks=None, stream=None):
    """x, z [B, T, G, D]; out [B, G, out_blocks, D]."""
    B, T = x.shape[0], x.shape[1]
    ob = out.shape[2] if out_blocks is None else out_blocks
    _check("lbca_pool", _lib.lbca_pool(ctypes.byref(cfg), series, _ptr(x), _ptr(z), _ptr(b_pos), _ptr(gamma),
                                       B, T, pos0, _ptr(out), ob, _stream(stream)))


def lbca_pool_f32(cfg, series, x, z, b_pos, gamma, out, pos0=0, out_blocks=None, stream=None):
    """lbca_pool with f32 entries: out float32 [B, G, out_blocks, D]."""
    if out.dtype != torch.float32:
        raise TypeError("lbca_pool_f32 writes float32 entries")
    B, T = x.shape[0], x.shape[1]
    ob = out.shape[2] if out_blocks is None else out_blocks
    _check("lbca_pool_f32", _lib.lbca_pool_f32(ctypes.byref(cfg), series, _ptr(x), _ptr(z), _ptr(b_pos), _ptr(gamma),
                                               B, T, pos0, _ptr(out), ob, _stream(stream)))


def lbca_pool_kv(cfg, k, v, zk, zv, b_pos_k, b_pos_v, gamma_kv, pooled_k, pooled_v, pos0=0, out_blocks=None,
                 stream=None):
    """Both series of the GQA form in one launch: k, v, zk, zv [B, T, G, D];
    pooled_k, pooled_v [B, G, out_blocks, D]."""
    B, T = k.shape[0], k.shape[1]
    ob = pooled_k.shape[2] if out_blocks is None else out_blocks
    _check("lbca_pool_kv", _lib.lbca_pool_kv(ctypes.byref(cfg), _ptr(k), _ptr(v), _ptr(zk), _ptr(zv), _ptr(b_pos_k),
                                             _ptr(b_pos_v), _ptr(gamma_kv), B, T, pos0, _ptr(pooled_k),
                                             _ptr(pooled_v), ob, _stream(stream)))


def lbca_pool_dual(cfg, series, xa, za, xb, zb, b_pos_a, b_pos_b, gamma, out, out_blocks=None, stream=None):
    """x*, z* [B, T, G, D]; out [B, G, out_blocks, D] (entry j pools block j of
    the a-series and block j - 1 of the b-series under one softmax)."""
    B, T = xa.shape[0], xa.shape[1]
    ob = out.shape[2] if out_blocks is None else out_blocks
    _check("lbca_pool_dual", _lib.lbca_pool_dual(ctypes.byref(cfg), series, _ptr(xa), _ptr(za), _ptr(xb), _ptr(zb),
                                                 _ptr(b_pos_a), _ptr(b_pos_b), _ptr(gamma), B, T, _ptr(out), ob,
                                                 _stream(stream)))


def lbca_append(cfg, k, v, zk, zv, b_pos_k, b_pos_v, gamma_kv, cache: Cache, d_status=None, stream=None):
    """k, v, zk, zv [B, G, D]: one token per sequence."""
    cc = cache.c()
    _check("lbca_append", _lib.lbca_append(ctypes.byref(cfg), _ptr(k), _ptr(v), _ptr(zk), _ptr(zv),
                                           _ptr(b_pos_k), _ptr(b_pos_v), _ptr(gamma_kv), ctypes.byref(cc),
                                           _ptr(d_status), _stream(stream)))


def lbca_decode(cfg, q, cache: Cache, sink, gamma_q, gamma_kv, out, workspace, max_ctx=0, d_status=None,
                stream=None):
    """q, out [B, Hq, D]; workspace a zero-filled uint8 tensor."""
    cc = cache.c()
    _check("lbca_decode", _lib.lbca_decode(ctypes.byref(cfg), _ptr(q), ctypes.byref(cc), _ptr(sink),
                                           _ptr(gamma_q), _ptr(gamma_kv), max_ctx, _ptr(out), _ptr(workspace),
                                           workspace.numel() * workspace.element_size(), _ptr(d_status),
                                           _stream(stream)))


def lbca_decode_step_workspace_bytes(cfg: lbca_config, batch: int, max_ctx: int) -> int:
    return int(_lib.lbca_decode_step_workspace_bytes(ctypes.byref(cfg), batch, max_ctx))


def lbca_decode_step_launches(cfg: lbca_config, batch: int, max_ctx: int) -> int:
    return int(_lib.lbca_decode_step_launches(ctypes.byref(cfg), batch, max_ctx))


LBCA_STEP_TWO_CALLS, LBCA_STEP_CLUSTER, LBCA_STEP_PERSISTENT, LBCA_STEP_SHARED_TC = range(4)


def lbca_decode_step_form(cfg: lbca_config, batch: int, max_ctx: int) -> int:
    return int(_lib.lbca_decode_step_form(ctypes.byref(cfg), batch, max_ctx))


def lbca_decode_step(cfg, k, v, zk, zv, b_pos_k, b_pos_v, gamma_kv, q, cache: Cache, sink, gamma_q, out,
                     workspace, max_ctx=0, d_status=None, stream=None):
    """Append the token (k, v, zk, zv [B, G, D]) and decode q [B, Hq, D] in one step."""
    cc = cache.c()
    _check("lbca_decode_step", _lib.lbca_decode_step(
        ctypes.byref(cfg), _ptr(k), _ptr(v), _ptr(zk), _ptr(zv), _ptr(b_pos_k), _ptr(b_pos_v), _ptr(gamma_kv),
        _ptr(q), ctypes.byref(cc), _ptr(sink), _ptr(gamma_q), max_ctx, _ptr(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(d_status), _stream(stream)))


def lbca_prefill(cfg, q, k, v, zk, zv, b_pos_k, b_pos_v, sink, gamma_q, gamma_kv, out,
                 cache_out: Cache | None = None, workspace=None, batch=None, T=None, d_status=None, stream=None):
    """q, out [B, T, Hq, D]; k, v, zk, zv [B, T, G, D]."""
    B = k.shape[0] if batch is None else batch
    TT = k.shape[1] if T is None else T
    cc = cache_out.c() if cache_out is not None else None
    wb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("lbca_prefill", _lib.lbca_prefill(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(zk), _ptr(zv),
                                             _ptr(b_pos_k), _ptr(b_pos_v), _ptr(sink), _ptr(gamma_q),
                                             _ptr(gamma_kv), B, TT, _ptr(out),
                                             ctypes.byref(cc) if cc is not None else None,
                                             _ptr(workspace), wb, _ptr(d_status), _stream(stream)))


def lbca_decode_noalloc(cfg, q, cache: Cache, sink, gamma_q, gamma_kv, out, max_ctx=0, d_status=None,
                        stream=None):
    """lbca_decode without a workspace, for callers that may not allocate device
    memory: the library's own static scratch holds the split partials.  Calls
    that overlap on the GPU race on that scratch."""
    cc = cache.c()
    _check("lbca_decode_noalloc", _lib.lbca_decode_noalloc(ctypes.byref(cfg), _ptr(q), ctypes.byref(cc), _ptr(sink),
                                                           _ptr(gamma_q), _ptr(gamma_kv), max_ctx, _ptr(out),
                                                           _ptr(d_status),
                                                           _stream(stream)))


def lbca_selftest_bounded_wait(arrive: bool, limit_ns: int, d_status, stream=None):
    """One CTA waits on an mbarrier nothing arrives at (arrive=False) or that it
    completes itself (arrive=True); a wait that runs out writes
    LBCA_ERR_TIMEOUT to d_status (an int32 device tensor)."""
    _check("lbca_selftest_bounded_wait", _lib.lbca_selftest_bounded_wait(int(arrive), int(limit_ns), _ptr(d_status),
                                                                         _stream(stream)))


def lbca_decode_sparse(cfg, q, cache: Cache, sel, sink, gamma_q, gamma_kv, out, d_status=None, stream=None):
    """q, out [B, Hq, D]; sel [B, top_k] int32 selected block indices."""
    cc = cache.c()
    _check("lbca_decode_sparse", _lib.lbca_decode_sparse(ctypes.byref(cfg), _ptr(q), ctypes.byref(cc), _ptr(sel),
                                                         sel.shape[1], _ptr(sink), _ptr(gamma_q), _ptr(gamma_kv),
                                                         _ptr(out), _ptr(d_status), _stream(stream)))


def lbca_indexer_workspace_bytes(batch: int, max_blocks: int) -> int:
    return int(_lib.lbca_indexer_workspace_bytes(batch, max_blocks))


def lbca_indexer_topk(q_idx, w_idx, k_idx, seq_lens, block_m, sel, sel_scores, workspace, d_status=None,
                      stream=None):
    """q_idx [B, HI, DI] bf16, w_idx [B, HI] f32, k_idx [B, max_blocks, DI] bf16,
    seq_lens [B] int32; sel [B, top_k] int32 (and sel_scores [B, top_k] f32 or None) out."""
    B, HI, DI = q_idx.shape
    _check("lbca_indexer_topk", _lib.lbca_indexer_topk(
        B, HI, DI, block_m, sel.shape[1], _ptr(q_idx), _ptr(w_idx), _ptr(k_idx), k_idx.shape[1], _ptr(seq_lens),
        _ptr(sel), _ptr(sel_scores), _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(d_status),
        _stream(stream)))


def lbca_prefill_backward_workspace_bytes(cfg: lbca_config, batch: int, T: int) -> int:
    return int(_lib.lbca_prefill_backward_workspace_bytes(ctypes.byref(cfg), batch, T))


def lbca_prefill_backward(cfg, q, k, v, zk, zv, b_pos_k, b_pos_v, sink, gamma_q, gamma_kv, dout, grads: dict,
                          workspace, stream=None):
    """Gradients into the f32 tensors of ``grads`` (dq, dk, dzk, dbk and, GQA,
    dv, dzv, dbv; dsink with a sink)."""
    B, T = q.shape[0], q.shape[1]
    g = lambda n: _ptr(grads.get(n))  # noqa: E731
    _check("lbca_prefill_backward", _lib.lbca_prefill_backward(
        ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(zk), _ptr(zv), _ptr(b_pos_k), _ptr(b_pos_v), _ptr(sink),
        _ptr(gamma_q), _ptr(gamma_kv), _ptr(dout), B, T, g("dq"), g("dk"), g("dv"), g("dzk"), g("dzv"), g("dbk"),
        g("dbv"), g("dsink"), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def lbca_prefill_rows(cfg, q, row0, k, v, raw0, pooled_k, pooled_v, sink, gamma_q, gamma_kv, out, stream=None):
    """q, out [B, n_rows, Hq, D] at absolute rows row0..; k, v [B, n_raw, G, D]
    from absolute position raw0; pooled_k/v float32 [B, G, pool_stride, D]
    (lbca_pool_f32)."""
    for p in (pooled_k, pooled_v):
        if p is not None and p.dtype != torch.float32:
            raise TypeError("lbca_prefill_rows reads float32 pooled entries")
    B, n = q.shape[0], q.shape[1]
    stride = 0 if pooled_k is None else pooled_k.shape[2]
    _check("lbca_prefill_rows", _lib.lbca_prefill_rows(
        ctypes.byref(cfg), _ptr(q), row0, n, _ptr(k), _ptr(v), raw0, k.shape[1], _ptr(pooled_k), _ptr(pooled_v),
        stride, _ptr(sink), _ptr(gamma_q), _ptr(gamma_kv), B, _ptr(out), _stream(stream)))
