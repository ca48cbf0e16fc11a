"""Seeded synthetic inputs for block-compressed attention.

This module holds the workload table and the random draws only -- none of the
method's arithmetic -- so that the CUDA path and the CPU oracle can be fed the
very same values.  Every tensor is drawn as N(0, std^2) from a counter-seeded
numpy generator, rounded (round-to-nearest-even) to the I/O dtype, and returned
as a CPU torch tensor; callers move it to the GPU or widen it to fp64 for the
oracle.  Each array has its own stream, keyed by (seed, name, sequence), so a
single sequence of a large batch can be regenerated alone.

The workloads follow the shapes of the pages: a Llama-3.2-3B-shaped GQA layer
(24 query heads, 8 kv heads, head_dim 128; "mSeek" README, "Experiment at a
glance": window 128, blocks of 16 then 64) and the HCA form (64 query heads
sharing one 512-dim K=V entry, partial RoPE on the last 64 dims, m' = 128;
HCA page and the CSA page's "What is implemented").
"""
from __future__ import annotations

import os
import zlib
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "prefill" or "decode"
    dtype: str           # "f32" or "bf16" (I/O dtype; accumulation is f32 on the GPU)
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    shared_kv: bool
    block_m: int
    n_win: int
    rope_dims: int = 0
    rmsnorm: bool = False
    sink: str = "none"   # "none", "zero" (present, logit 0) or "normal" (N(0,1) per head)
    seq_len: int = 0     # prefill tokens
    ctx: tuple = (0, 0)  # decode: cached context, drawn uniformly in [lo, hi] per sequence
    steps: int = 1       # decode: tokens appended (one per step)
    bpos_std: float = 0.02
    seed: int = 0
    rope_theta: float = 10000.0
    # CSA form: dual overlapped pooling (a second raw series and bias), a
    # lightning indexer of index_heads x index_dim over its own dual-pooled
    # keys, and top_k selected entries per query
    dual: bool = False
    index_heads: int = 0
    index_dim: int = 0
    top_k: int = 0


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_f32_prefill", "prefill", "f32", 1, 4, 1, 64, True, 16, 128,
                 rope_dims=0, sink="zero", seq_len=512, seed=1001),
        Workload("gqa_decode_32k", "decode", "bf16", 1, 24, 8, 128, False, 64, 128,
                 rope_dims=128, ctx=(32768, 32768), steps=64, seed=1002),
        Workload("gqa_prefill_16k", "prefill", "bf16", 1, 24, 8, 128, False, 16, 128,
                 rope_dims=128, seq_len=16384, seed=1003),
        Workload("hca_mqa_decode_128k", "decode", "bf16", 8, 64, 1, 512, True, 128, 128,
                 rope_dims=64, rmsnorm=True, sink="normal", ctx=(131072, 131072), steps=16,
                 seed=1004),
        Workload("ragged_gqa_decode_append", "decode", "bf16", 32, 24, 8, 128, False, 64, 128,
                 rope_dims=128, ctx=(4096, 65536), steps=64, seed=1005),
        Workload("csa_sparse_decode_64k", "decode", "bf16", 4, 64, 1, 512, True, 4, 128,
                 rope_dims=64, rmsnorm=True, sink="normal", ctx=(65536, 65536), steps=8, seed=1006,
                 dual=True, index_heads=64, index_dim=128, top_k=512),
    ]
}


def scaled(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (smaller parity cases)."""
    return replace(w, **kw)


def _rng(seed: int, tag: str, idx: int = 0) -> np.random.Generator:
    return np.random.default_rng([seed, zlib.crc32(tag.encode()), idx])


def _round(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16) if dtype == "bf16" else t


CHUNK = 4096  # tokens per random stream along the sequence axis


def normal(seed: int, tag: str, shape, std: float = 1.0, dtype: str = "bf16", row_len=None) -> torch.Tensor:
    """N(0, std^2) tensor of ``shape`` rounded to ``dtype``.  Streams are keyed
    by (index along axis 0, chunk of CHUNK entries along axis 1), so any
    sequence or span can be regenerated alone.  With ``row_len``, row i holds
    draws only in its first row_len[i] entries of axis 1 and zeros after
    (ragged sequences)."""
    shape = tuple(int(s) for s in shape)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = torch.zeros(shape, dtype=tdt)
    if len(shape) == 0 or shape[0] == 0:
        return out
    if len(shape) == 1:
        out[:] = _round(_rng(seed, tag, 0).standard_normal(shape, dtype=np.float32) * np.float32(std), dtype)
        return out
    jobs = []
    for i in range(shape[0]):
        n = shape[1] if row_len is None else min(int(row_len[i]), shape[1])
        for c0 in range(0, n, CHUNK):
            jobs.append((i, c0, min(n, c0 + CHUNK)))

    def fill(job):
        i, c0, c1 = job
        a = _rng(seed, tag, i * 1_000_003 + c0 // CHUNK).standard_normal((c1 - c0,) + shape[2:], dtype=np.float32)
        if std != 1.0:
            a *= np.float32(std)
        out[i, c0:c1] = _round(a, dtype)

    with ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
        list(ex.map(fill, jobs))
    return out


def contexts(w: Workload) -> np.ndarray:
    """Per-sequence cached context length for a decode workload."""
    lo, hi = w.ctx
    if lo == hi:
        return np.full(w.batch, lo, dtype=np.int64)
    return _rng(w.seed, "ctx").integers(lo, hi + 1, size=w.batch).astype(np.int64)


@dataclass
class Inputs:
    """Raw inputs of one workload (CPU tensors in the I/O dtype; sink f32)."""
    q: torch.Tensor                   # prefill [B,T,Hq,D]; decode [steps,B,Hq,D]
    k: torch.Tensor                   # [B,T,G,D] (shared form: C)
    v: torch.Tensor | None            # [B,T,G,D] or None (shared form)
    zk: torch.Tensor                  # [B,T,G,D] (shared form: Z)
    zv: torch.Tensor | None
    bpos_k: torch.Tensor              # [m, G*D]
    bpos_v: torch.Tensor | None
    sink: torch.Tensor | None         # [Hq] f32
    lens: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))  # decode: context per sequence
    # CSA form: b-series kb, zkb [B,T,G,D] and bias bpos_kb [m, G*D]; indexer
    # queries iq [steps,B,HI,DI] and head weights iw [steps,B,HI] (f32), its
    # key series ika, izka, ikb, izkb [B,T,1,DI] and biases ibpa, ibpb [m, DI]
    csa: dict = field(default_factory=dict)


def make(w: Workload, lens: np.ndarray | None = None) -> Inputs:
    """Draw a workload's inputs.  Order of draws: Q, K (or C), V, Z_K (or Z),
    Z_V, B_pos_K, B_pos_V, sink; each from its own keyed stream.  A decode
    workload's cached contexts come from `contexts(w)` unless given."""
    B, Hq, G, D, m = w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block_m
    if w.kind == "prefill":
        T = w.seq_len
        q = normal(w.seed, "q", (B, T, Hq, D), dtype=w.dtype)
        lens = np.full(B, T, dtype=np.int64)
    else:
        lens = contexts(w) if lens is None else np.asarray(lens, dtype=np.int64)
        T = int(lens.max()) + w.steps
        q = normal(w.seed, "q", (w.steps, B, Hq, D), dtype=w.dtype)
    rl = None if w.kind == "prefill" else lens + w.steps  # history each sequence reaches
    k = normal(w.seed, "k", (B, T, G, D), dtype=w.dtype, row_len=rl)
    v = None if w.shared_kv else normal(w.seed, "v", (B, T, G, D), dtype=w.dtype, row_len=rl)
    zk = normal(w.seed, "zk", (B, T, G, D), dtype=w.dtype, row_len=rl)
    zv = None if w.shared_kv else normal(w.seed, "zv", (B, T, G, D), dtype=w.dtype, row_len=rl)
    bpk = normal(w.seed, "bpos_k", (m, G * D), std=w.bpos_std, dtype=w.dtype)
    bpv = None if w.shared_kv else normal(w.seed, "bpos_v", (m, G * D), std=w.bpos_std, dtype=w.dtype)
    if w.sink == "none":
        sink = None
    elif w.sink == "zero":
        sink = torch.zeros(Hq, dtype=torch.float32)
    else:
        sink = normal(w.seed, "sink", (Hq,), dtype="f32")
    csa = {}
    if w.dual:
        csa["kb"] = normal(w.seed, "kb", (B, T, G, D), dtype=w.dtype, row_len=rl)
        csa["zkb"] = normal(w.seed, "zkb", (B, T, G, D), dtype=w.dtype, row_len=rl)
        csa["bpos_kb"] = normal(w.seed, "bpos_kb", (m, G * D), std=w.bpos_std, dtype=w.dtype)
        if w.index_heads:
            HI, DI = w.index_heads, w.index_dim
            lead = (B, T, HI, DI) if w.kind == "prefill" else (w.steps, B, HI, DI)
            csa["iq"] = normal(w.seed, "iq", lead, dtype=w.dtype)
            csa["iw"] = normal(w.seed, "iw", lead[:-1], dtype="f32")
            for tag in ("ika", "izka", "ikb", "izkb"):
                csa[tag] = normal(w.seed, tag, (B, T, 1, DI), dtype=w.dtype, row_len=rl)
            csa["ibpa"] = normal(w.seed, "ibpa", (m, DI), std=w.bpos_std, dtype=w.dtype)
            csa["ibpb"] = normal(w.seed, "ibpb", (m, DI), std=w.bpos_std, dtype=w.dtype)
    return Inputs(q, k, v, zk, zv, bpk, bpv, sink, lens, csa)


def f64(t):
    """fp64 numpy copy of a CPU tensor (None passes through)."""
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()
