"""Python front of the fp64 CPU oracle for block-compressed attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg use it; the CUDA library never does, and the two
share no code.  The arithmetic lives in ``lbca_oracle.c`` (fp64, plain loops,
OpenMP over independent rows); this module only marshals numpy arrays.

Functions and the passages they follow:
  * ``pool``      -- block pooling + entry finalisation ("mSeek" README,
                     "How LBCA works" steps 2-3; HCA page, "What is
                     implemented", Eqs 20-23; CSA page, "Deviations from
                     paper": RoPE at block-start positions).
  * ``attend``    -- attention over visible pooled entries + raw window + sink
                     ("mSeek" README, "How LBCA works" steps 4-5; CSA page,
                     "What is implemented": Eqs 18-19, Eq 27, -i rotation).
  * ``forward``   -- prefill: pool, then attend every row.
  * ``decode``    -- one query per sequence at position len-1 (ragged lens).
  * ``Stream``    -- the same definition driven token by token, pooling each
                     block when it completes ("mSeek" README, repository
                     layout: generation through the LBCA cache).
  * ``pool_dual``  -- CSA dual overlapped pooling: entry i combines block i of
                     the a-series with block i - 1 of the b-series, all 2m
                     tokens weighted by a single softmax (CSA page, "What is
                     implemented", Eqs 9-12).
  * ``indexer_scores`` / ``topk_blocks`` -- lightning-indexer relevance
                     sum_h w_h ReLU(q_h . k_j) over the complete blocks, and
                     the top-k of them (CSA page, "What is implemented",
                     Eqs 13-17).
  * ``attend_sparse`` -- shared-KV core attention over the selected entries
                     plus the overlapping window of the last n_win raw tokens
                     and the sink (CSA page, "What is implemented", Eqs 18-19,
                     Eq 27, -i rotation).
  * ``prefill_backward`` -- gradients of sum(dout * prefill output) with
                     respect to the queries, raw keys and values, the pooling
                     logits, the positional biases and the sink: reverse-mode
                     differentiation of ``pool`` + ``attend`` ("mSeek" README,
                     "Experiment at a glance": the LBCA layers are trained).
  * ``visible_blocks`` -- P(L) of the block-aligned visibility reading.
  * ``cache_entries`` / ``kv_cache_bytes`` -- analytic cache accounting
                     ("mSeek" README, "Results").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lbca_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liblbca_oracle.so")
_lib = None

KEY, VALUE = 0, 1


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, -O2, OpenMP, no fast-math) in place."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared",
                               "-fno-fast-math", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Cfg(ctypes.Structure):
    _fields_ = [("n_q_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("shared_kv", ctypes.c_int),
                ("block_m", ctypes.c_int), ("n_win", ctypes.c_int),
                ("rope_dims", ctypes.c_int), ("rmsnorm", ctypes.c_int),
                ("rope_theta", ctypes.c_double), ("rms_eps", ctypes.c_double),
                ("softmax_scale", ctypes.c_double)]


@dataclass(frozen=True)
class Config:
    """Layer shape and method parameters (same meaning as the C struct)."""
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    shared_kv: bool
    block_m: int
    n_win: int
    rope_dims: int = 0
    rmsnorm: bool = False
    rope_theta: float = 10000.0
    rms_eps: float = 1e-6
    softmax_scale: float = 0.0

    def c(self) -> _Cfg:
        return _Cfg(self.n_q_heads, self.n_kv_heads, self.head_dim, int(self.shared_kv),
                    self.block_m, self.n_win, self.rope_dims, int(self.rmsnorm),
                    float(self.rope_theta), float(self.rms_eps), float(self.softmax_scale))


def _load():
    global _lib
    if _lib is None:
        # LBCA_ORACLE_LIB: another build of lbca_oracle.c (the pin-strength
        # test loads copies with one planted mistake each)
        lib = ctypes.CDLL(os.environ.get("LBCA_ORACLE_LIB") or build())
        dp = ctypes.POINTER(ctypes.c_double)
        lp = ctypes.POINTER(ctypes.c_long)
        lib.orc_visible_blocks.argtypes = [ctypes.c_long, ctypes.c_int, ctypes.c_int]
        lib.orc_visible_blocks.restype = ctypes.c_long
        lib.orc_pool.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int, ctypes.c_int, ctypes.c_long,
                                 ctypes.c_long, dp, dp, dp, dp, dp]
        lib.orc_pool.restype = ctypes.c_int
        lib.orc_attend.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int, ctypes.c_int, lp, dp, dp, dp,
                                   ctypes.c_long, dp, dp, ctypes.c_long, lp, dp, dp, dp, dp]
        lib.orc_attend.restype = ctypes.c_int
        lib.orc_pool_dual.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int, ctypes.c_int, ctypes.c_long,
                                      dp, dp, dp, dp, dp, dp, dp, dp]
        lib.orc_pool_dual.restype = ctypes.c_int
        lib.orc_indexer_scores.argtypes = [ctypes.c_int, ctypes.c_long, ctypes.c_int, ctypes.c_int, dp, dp, dp,
                                           lp, dp]
        lib.orc_indexer_scores.restype = ctypes.c_int
        lib.orc_attend_sparse.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int, dp, dp, ctypes.c_long, lp,
                                          ctypes.c_int, dp, ctypes.c_long, lp, dp, dp, dp, dp]
        lib.orc_attend_sparse.restype = ctypes.c_int
        lib.orc_prefill_backward.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int, ctypes.c_long] + [dp] * 19
        lib.orc_prefill_backward.restype = ctypes.c_int
        _lib = lib
    return _lib


def _d(a):
    """fp64 C-contiguous view (or None -> NULL)."""
    if a is None:
        return None, None
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def visible_blocks(L: int, m: int, w: int) -> int:
    """P(L): pooled entries visible to a query that sees L tokens."""
    return int(_load().orc_visible_blocks(int(L), int(m), int(w)))


def pool(cfg: Config, series: int, x, z, b_pos, gamma=None, pos0: int = 0):
    """Pooled + finalised entries of one series: [B, T//m, G, D] fp64."""
    x, xp = _d(x)
    z, zp = _d(z)
    b_pos, bp = _d(b_pos)
    gamma, gp = _d(gamma)
    B, T, G, D = x.shape
    assert z.shape == x.shape and G == cfg.n_kv_heads and D == cfg.head_dim
    assert b_pos.shape == (cfg.block_m, G * D)
    out = np.zeros((B, T // cfg.block_m, G, D))
    rc = _load().orc_pool(ctypes.byref(cfg.c()), series, B, T, pos0, xp, zp, bp, gp,
                          out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc:
        raise ValueError("orc_pool rejected its arguments")
    return out


def attend(cfg: Config, q, qpos, ek, ev, k, v, lens, sink=None, gamma_q=None, gamma_kv=None):
    """Attention of query rows q [B, nq, Hq, D] at positions qpos [B, nq]."""
    q, qp = _d(q)
    B, nq, Hq, D = q.shape
    qpos = np.ascontiguousarray(qpos, dtype=np.int64).reshape(B, nq)
    lens = np.ascontiguousarray(lens, dtype=np.int64).reshape(B)
    k, kp = _d(k)
    v, vp = _d(v)
    if ek is None:
        ek = np.zeros((B, 0, cfg.n_kv_heads, D))
    ek, ekp = _d(ek)
    ev, evp = _d(ev)
    sink, sp = _d(sink)
    gamma_q, gqp = _d(gamma_q)
    gamma_kv, gkp = _d(gamma_kv)
    out = np.zeros((B, nq, Hq, D))
    lp = ctypes.POINTER(ctypes.c_long)
    rc = _load().orc_attend(ctypes.byref(cfg.c()), B, nq, qpos.ctypes.data_as(lp), qp, ekp, evp,
                            ek.shape[1], kp, vp, k.shape[1], lens.ctypes.data_as(lp), sp, gqp, gkp,
                            out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc:
        raise ValueError("orc_attend rejected its arguments")
    return out


def forward(cfg: Config, q, k, v, zk, zv, bpos_k, bpos_v=None, sink=None,
            gamma_q=None, gamma_kv=None, rows=None):
    """Prefill: outputs [B, len(rows), Hq, D] for query rows (all by default).

    Pools the blocks that any requested row can see, then attends.
    In the shared form pass k=C, zk=Z and leave v, zv, bpos_v as None.
    """
    q = np.asarray(q)
    B, T = q.shape[:2]
    rows = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    need = visible_blocks(int(rows.max()) + 1, cfg.block_m, cfg.n_win) if len(rows) else 0
    kk = np.asarray(k)[:, :need * cfg.block_m]
    ek = pool(cfg, KEY, kk, np.asarray(zk)[:, :need * cfg.block_m], bpos_k, gamma_kv)
    ev = None
    if not cfg.shared_kv:
        ev = pool(cfg, VALUE, np.asarray(v)[:, :need * cfg.block_m],
                  np.asarray(zv)[:, :need * cfg.block_m], bpos_v)
    qpos = np.broadcast_to(rows, (B, len(rows)))
    return attend(cfg, q[:, rows], qpos, ek, ev, k, v, np.full(B, T), sink, gamma_q, gamma_kv)


def decode(cfg: Config, q, k, v, zk, zv, bpos_k, bpos_v, lens, sink=None,
           gamma_q=None, gamma_kv=None):
    """One query per sequence: q [B, Hq, D] at position lens[b]-1 over history
    k, v, zk, zv [B, Tmax, G, D] of which lens[b] tokens are valid."""
    q = np.asarray(q)
    B = q.shape[0]
    lens = np.asarray(lens, dtype=np.int64).reshape(B)
    out = np.zeros(q.shape)
    for b in range(B):  # sequences have different visible block counts
        L = int(lens[b])
        need = visible_blocks(L, cfg.block_m, cfg.n_win) * cfg.block_m
        sl = slice(b, b + 1)
        ek = pool(cfg, KEY, np.asarray(k)[sl, :need], np.asarray(zk)[sl, :need], bpos_k, gamma_kv)
        ev = None if cfg.shared_kv else pool(cfg, VALUE, np.asarray(v)[sl, :need],
                                             np.asarray(zv)[sl, :need], bpos_v)
        vv = None if cfg.shared_kv else np.asarray(v)[sl, :L]
        out[b] = attend(cfg, q[sl, None], np.array([[L - 1]]), ek, ev, np.asarray(k)[sl, :L], vv,
                        np.array([L]), sink, gamma_q, gamma_kv)[0, 0]
    return out


class Stream:
    """Token-by-token form of the same definition for one sequence.

    ``extend`` adds raw tokens; each block they complete is pooled and
    finalised once and kept.  ``query`` attends one query at the position of
    the last appended token.  The arithmetic is the C oracle's; the buffers
    grow by doubling so that a step does not copy the history.
    """

    def __init__(self, cfg: Config, bpos_k, bpos_v=None, gamma_kv=None):
        self.cfg = cfg
        self.bpos_k, self.bpos_v, self.gamma_kv = bpos_k, bpos_v, gamma_kv
        self.n = 0
        self.nb = 0
        self._buf = {}

    def _grow(self, name, need, row):
        b = self._buf.get(name)
        if b is None or b.shape[0] < need:
            nb = np.zeros((max(need, 2 * (0 if b is None else b.shape[0]), 64),) + row)
            if b is not None:
                nb[:b.shape[0]] = b
            self._buf[name] = nb
        return self._buf[name]

    def _arr(self, name, n):
        b = self._buf.get(name)
        return None if b is None else b[:n]

    def extend(self, k, zk, v=None, zv=None):
        """Append a run of raw tokens [n, G, D] (pools every block it completes)."""
        m = self.cfg.block_m
        row = (self.cfg.n_kv_heads, self.cfg.head_dim)
        new = np.asarray(k).shape[0]
        names = [("k", k), ("zk", zk)] + ([] if self.cfg.shared_kv else [("v", v), ("zv", zv)])
        for name, a in names:
            self._grow(name, self.n + new, row)[self.n:self.n + new] = a
        self.n += new
        done = self.n // m
        if done > self.nb:
            sl = slice(self.nb * m, done * m)
            ek = pool(self.cfg, KEY, self._buf["k"][None, sl], self._buf["zk"][None, sl], self.bpos_k,
                      self.gamma_kv, pos0=self.nb * m)[0]
            self._grow("ek", done, row)[self.nb:done] = ek
            if not self.cfg.shared_kv:
                ev = pool(self.cfg, VALUE, self._buf["v"][None, sl], self._buf["zv"][None, sl], self.bpos_v)[0]
                self._grow("ev", done, row)[self.nb:done] = ev
            self.nb = done

    def query(self, q, sink=None, gamma_q=None):
        """Output [Hq, D] for query q [Hq, D] at the last appended position."""
        L = self.n
        shared = self.cfg.shared_kv
        ek = self._arr("ek", self.nb)
        ev = None if shared else self._arr("ev", self.nb)
        return attend(self.cfg, np.asarray(q)[None, None], np.array([[L - 1]]),
                      None if ek is None else ek[None], None if ev is None else ev[None],
                      self._arr("k", L)[None], None if shared else self._arr("v", L)[None],
                      np.array([L]), sink, gamma_q, self.gamma_kv)[0, 0]


def pool_dual(cfg: Config, series: int, xa, za, xb, zb, bpos_a, bpos_b, gamma=None):
    """Dual overlapped pooling of the T//m complete blocks: [B, T//m, G, D] fp64.
    Entry i: one softmax over block i's a-series logits and block i-1's
    b-series logits (block 0: its a-series alone); ORC KEY entries then take
    RMSNorm (when on) and RoPE at i*m."""
    xa, xap = _d(xa)
    za, zap = _d(za)
    xb, xbp = _d(xb)
    zb, zbp = _d(zb)
    bpos_a, bap = _d(bpos_a)
    bpos_b, bbp = _d(bpos_b)
    gamma, gp = _d(gamma)
    B, T, G, D = xa.shape
    assert za.shape == xb.shape == zb.shape == xa.shape and G == cfg.n_kv_heads and D == cfg.head_dim
    assert bpos_a.shape == bpos_b.shape == (cfg.block_m, G * D)
    out = np.zeros((B, T // cfg.block_m, G, D))
    rc = _load().orc_pool_dual(ctypes.byref(cfg.c()), series, B, T, xap, zap, xbp, zbp, bap, bbp, gp,
                               out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc:
        raise ValueError("orc_pool_dual rejected its arguments")
    return out


def complete_blocks(L: int, m: int) -> int:
    """Blocks of m tokens complete within the first L tokens: the compressed
    entries a query that sees L tokens may select (the CSA form's entries are
    visible once complete; its raw window overlaps them)."""
    return int(L) // int(m)


def indexer_scores(q, w, kx, nvis):
    """I[b, j] = sum_h w[b, h] ReLU(q[b, h] . kx[b, j]) for j < nvis[b], -inf after.
    q [B, HI, DI], w [B, HI], kx [B, NB, DI]."""
    q, qp = _d(q)
    w, wp = _d(w)
    kx, kp = _d(kx)
    B, HI, DI = q.shape
    NB = kx.shape[1]
    assert w.shape == (B, HI) and kx.shape == (B, NB, DI)
    nvis = np.ascontiguousarray(nvis, dtype=np.int64).reshape(B)
    out = np.zeros((B, NB))
    rc = _load().orc_indexer_scores(B, NB, HI, DI, qp, wp, kp,
                                    nvis.ctypes.data_as(ctypes.POINTER(ctypes.c_long)),
                                    out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc:
        raise ValueError("orc_indexer_scores rejected its arguments")
    return out


def topk_blocks(scores, nvis, k: int):
    """The k highest-scoring visible blocks per row, highest first (equal
    scores: lower index first), padded with -1 when fewer than k are visible:
    [B, k] int64."""
    scores = np.asarray(scores, dtype=np.float64)
    B, NB = scores.shape
    out = np.full((B, k), -1, dtype=np.int64)
    for b in range(B):
        n = int(nvis[b])
        idx = np.arange(n)
        order = np.lexsort((idx, -scores[b, :n]))  # by score descending, then index
        take = order[:k]
        out[b, :len(take)] = take
    return out


def attend_sparse(cfg: Config, q, ek, sel, k, lens, sink=None, gamma_q=None, gamma_kv=None):
    """Shared-KV attention of one query per sequence (at lens[b] - 1) over the
    selected entries ek[b, sel[b, i]] (sel -1: unused) plus the raw window of
    the last n_win tokens and the sink: [B, Hq, D]."""
    q, qp = _d(q)
    B, Hq, D = q.shape
    ek, ekp = _d(ek)
    sel = np.ascontiguousarray(sel, dtype=np.int64)
    K = sel.shape[1] if sel.ndim == 2 else 0
    k, kp = _d(k)
    lens = np.ascontiguousarray(lens, dtype=np.int64).reshape(B)
    sink, sp = _d(sink)
    gamma_q, gqp = _d(gamma_q)
    gamma_kv, gkp = _d(gamma_kv)
    out = np.zeros((B, Hq, D))
    lp = ctypes.POINTER(ctypes.c_long)
    rc = _load().orc_attend_sparse(ctypes.byref(cfg.c()), B, qp, ekp, 0 if ek is None else ek.shape[1],
                                   sel.ctypes.data_as(lp) if K else None, K, kp, k.shape[1],
                                   lens.ctypes.data_as(lp), sp, gqp, gkp,
                                   out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc:
        raise ValueError("orc_attend_sparse rejected its arguments")
    return out


def prefill_backward(cfg: Config, q, k, v, zk, zv, bpos_k, bpos_v, dout, sink=None, gamma_q=None, gamma_kv=None):
    """Gradients of sum(dout * forward(...)) over every row: a dict with dq,
    dk, dzk, dbk, dsink and (GQA) dv, dzv, dbv, fp64 in the inputs' shapes."""
    q, qp = _d(q)
    k, kp = _d(k)
    v, vp = _d(v)
    zk, zkp = _d(zk)
    zv, zvp = _d(zv)
    bpos_k, bkp = _d(bpos_k)
    bpos_v, bvp = _d(bpos_v)
    dout, dop = _d(dout)
    sink, sp = _d(sink)
    gamma_q, gqp = _d(gamma_q)
    gamma_kv, gkp = _d(gamma_kv)
    B, T = q.shape[:2]
    out = {"dq": np.zeros(q.shape), "dk": np.zeros(k.shape), "dzk": np.zeros(k.shape),
           "dbk": np.zeros(bpos_k.shape), "dsink": np.zeros(cfg.n_q_heads)}
    if not cfg.shared_kv:
        out.update(dv=np.zeros(k.shape), dzv=np.zeros(k.shape), dbv=np.zeros(bpos_k.shape))
    ptr = lambda name: out[name].ctypes.data_as(ctypes.POINTER(ctypes.c_double)) if name in out else None  # noqa
    rc = _load().orc_prefill_backward(ctypes.byref(cfg.c()), B, T, qp, kp, vp, zkp, zvp, bkp, bvp, sp, gqp, gkp,
                                      dop, ptr("dq"), ptr("dk"), ptr("dv"), ptr("dzk"), ptr("dzv"), ptr("dbk"),
                                      ptr("dbv"), ptr("dsink"))
    if rc:
        raise ValueError("orc_prefill_backward rejected its arguments")
    return out


def cache_entries(T: int, m: int, w: int) -> int:
    """Entries one LBCA layer stores per kv head for a T-token context:
    P(T) pooled entries plus the raw tokens from P(T)*m on."""
    P = visible_blocks(T, m, w)
    return P + (T - P * m)


def kv_cache_bytes(T: int, n_layers: int, n_lbca_layers: int, m: int, w: int,
                   n_kv_heads: int, head_dim: int, elt_bytes: int = 2) -> int:
    """Analytic K+V bytes for a model whose LBCA layers store ``cache_entries``
    per head and whose other layers store every token."""
    per_entry = 2 * n_kv_heads * head_dim * elt_bytes
    dense_layers = n_layers - n_lbca_layers
    return (dense_layers * T + n_lbca_layers * cache_entries(T, m, w)) * per_entry
