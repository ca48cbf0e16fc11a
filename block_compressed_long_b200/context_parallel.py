"""Context-parallel prefill of one long sequence over the ranks of a process
group, with one exchange step.

Each rank owns a contiguous, block-aligned range of the sequence's tokens
(the last rank also takes the tokens past the last complete block).  The
attention of a query at position t reads the pooled entries of blocks
j < P(t+1) and the raw tokens [P(t+1) m, t] (mSeek README, "How LBCA works",
steps 4-5); so a rank needs, besides its own tokens, every earlier rank's
pooled entries (1/m of their K/V) and at most the last n_win + m - 1 raw
tokens before its range.  The step is:

  1. pool the rank's own complete blocks (lbca_pool_f32 at the range's first
     position) into their slots of a full-length f32 pooled buffer;
  2. all-gather the pooled entries (every rank's slice of blocks; f32, the
     precision the single-GPU prefill keeps them at, for 1/m of the raw
     K/V bytes);
  3. all-gather the ranks' last n_win + m - 1 raw keys (and values), from
     which each rank takes the halo that precedes its range;
  4. attend the rank's own query rows (lbca_prefill_rows).

The collectives are torch.distributed calls (NCCL over NVLink between GPUs;
the tests run them as gloo ranks on the CPU).  Received data lands in local
memory before any kernel reads it.  The arithmetic is the library's.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class CpPlan:
    T: int            # tokens of the sequence
    m: int            # block size
    n_win: int        # raw window
    world: int
    ranges: tuple     # per rank (t0, t1)

    @property
    def halo(self) -> int:
        """Raw tokens before a range that its first rows can see."""
        return self.n_win + self.m - 1

    @property
    def blocks(self) -> int:
        return self.T // self.m

    def block_range(self, rank: int) -> tuple[int, int]:
        t0, t1 = self.ranges[rank]
        return t0 // self.m, t1 // self.m

    def halo_range(self, rank: int) -> tuple[int, int]:
        """Absolute token positions [lo, t0) of the halo this rank receives."""
        t0 = self.ranges[rank][0]
        return max(0, t0 - self.halo), t0


def plan(T: int, m: int, n_win: int, world: int) -> CpPlan:
    """Block-aligned contiguous ranges: the complete blocks split as evenly as
    possible (sizes differ by at most one block), the tail tokens to the last
    rank."""
    if world < 1:
        raise ValueError("world must be >= 1")
    nb = T // m
    ranges = []
    for r in range(world):
        b0, b1 = r * nb // world, (r + 1) * nb // world
        t1 = T if r == world - 1 else b1 * m
        ranges.append((b0 * m, t1))
    return CpPlan(T, m, n_win, world, tuple(ranges))


def gather_pooled(p: CpPlan, pooled: torch.Tensor, rank: int, group=None) -> torch.Tensor:
    """All-gather: every rank's own blocks of `pooled` ([B, G, NB, D], this
    rank's slice filled) into all slots, in place; returns `pooled`."""
    j0, j1 = p.block_range(rank)
    sizes = [p.block_range(r)[1] - p.block_range(r)[0] for r in range(p.world)]
    width = max(max(sizes), 1)
    B, G, _, D = pooled.shape
    mine = torch.zeros(B, G, width, D, dtype=pooled.dtype, device=pooled.device)
    mine[:, :, :j1 - j0] = pooled[:, :, j0:j1]
    parts = [torch.empty_like(mine) for _ in range(p.world)]
    dist.all_gather(parts, mine, group=group)
    for r, part in enumerate(parts):
        a, b = p.block_range(r)
        pooled[:, :, a:b] = part[:, :, :b - a]
    return pooled


def exchange_halo(p: CpPlan, raw: torch.Tensor, rank: int, group=None) -> torch.Tensor:
    """All-gather every rank's last `halo` raw tokens (raw: the rank's own
    tokens [B, n, G, D]) and return the tokens [lo, t0) that precede this
    rank's range ([B, t0 - lo, G, D]).  Every rank's tail is a suffix that
    ends where the next range starts, so the last t0 - lo tokens of the
    earlier ranks' tails, in order, are exactly the halo."""
    H = p.halo
    B, n, G, D = raw.shape
    tail = torch.zeros(B, H, G, D, dtype=raw.dtype, device=raw.device)
    k = min(H, n)
    if k:
        tail[:, H - k:] = raw[:, n - k:]
    parts = [torch.empty_like(tail) for _ in range(p.world)]
    dist.all_gather(parts, tail, group=group)
    lo, t0 = p.halo_range(rank)
    need = t0 - lo
    pieces, have = [], 0
    for r in range(rank - 1, -1, -1):
        if have >= need:
            break
        a, b = p.ranges[r]
        take = min(need - have, b - a, H)
        pieces.append(parts[r][:, H - take:])
        have += take
    if not pieces:
        return raw[:, :0]
    return torch.cat(pieces[::-1], dim=1)


def attend_rows(L, cfg, q_local, t0, raw_k, raw_v, raw0, pooled_k, pooled_v, sink=None, gamma_q=None,
                gamma_kv=None, out=None):
    """The rank's own rows (lbca_prefill_rows over the assembled inputs)."""
    if out is None:
        out = torch.empty_like(q_local)
    L.lbca_prefill_rows(cfg, q_local, t0, raw_k, raw_v, raw0, pooled_k, pooled_v, sink, gamma_q, gamma_kv, out)
    return out


def cp_prefill(L, cfg, p: CpPlan, rank: int, q, k, v, zk, zv, bpos_k, bpos_v, sink=None, gamma_q=None,
               gamma_kv=None, group=None) -> torch.Tensor:
    """The rank's output rows [B, n, Hq, D] of the context-parallel prefill;
    q, k, v, zk, zv hold the rank's own tokens (device tensors)."""
    t0, t1 = p.ranges[rank]
    B, _, G, D = k.shape
    shared = v is None
    pooled_k = torch.zeros(B, G, max(p.blocks, 1), D, dtype=torch.float32, device=k.device)
    pooled_v = None if shared else torch.zeros_like(pooled_k)
    L.lbca_pool_f32(cfg, L.LBCA_KEY, k, zk, bpos_k, gamma_kv, pooled_k, pos0=t0)
    if not shared:
        L.lbca_pool_f32(cfg, L.LBCA_VALUE, v, zv, bpos_v, None, pooled_v, pos0=t0)
    gather_pooled(p, pooled_k, rank, group)
    if not shared:
        gather_pooled(p, pooled_v, rank, group)
    hk = exchange_halo(p, k, rank, group)
    raw_k = torch.cat([hk, k], dim=1).contiguous()
    raw_v = None
    if not shared:
        raw_v = torch.cat([exchange_halo(p, v, rank, group), v], dim=1).contiguous()
    return attend_rows(L, cfg, q, t0, raw_k, raw_v, t0 - hk.shape[1], pooled_k, pooled_v, sink, gamma_q, gamma_kv)
