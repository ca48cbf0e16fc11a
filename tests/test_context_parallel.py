"""Context-parallel prefill, host side, on the CPU: world-size 2 and 3 gloo
ranks run the one exchange step (all-gather of the pooled entries, all-gather
of the raw-token tails), and every rank must then hold exactly the full
sequence's pooled prefix (the oracle's pooling of the whole sequence) and the
raw tokens that precede its range -- the inputs its own rows need (mSeek
README, "How LBCA works", steps 4-5)."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_compressed_long_b200 import context_parallel as cp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_plan_ranges_are_block_aligned_and_cover_the_sequence():
    for T, m, world in [(1000, 16, 3), (64, 64, 2), (4097, 64, 4), (10, 4, 1), (7, 4, 2)]:
        p = cp.plan(T, m, 8, world)
        assert p.ranges[0][0] == 0 and p.ranges[-1][1] == T
        for (a0, a1), (b0, _) in zip(p.ranges, p.ranges[1:]):
            assert a1 == b0 and a0 % m == 0 and a1 % m == 0
        sizes = [p.block_range(r)[1] - p.block_range(r)[0] for r in range(world)]
        assert max(sizes) - min(sizes) <= 1 and sum(sizes) == T // m
        assert p.halo == 8 + m - 1


def _rank_main(rank, world, port, T, m, w, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import sys
        sys.path.insert(0, ROOT)
        from oracle import oracle as orc
        rng = np.random.default_rng(5)  # every rank draws the same full sequence, then keeps its part
        B, G, D = 2, 2, 16
        x, z = rng.standard_normal((B, T, G, D)), rng.standard_normal((B, T, G, D))
        bp = 0.3 * rng.standard_normal((m, G * D))
        c = orc.Config(4, G, D, False, m, w)
        p = cp.plan(T, m, w, world)
        t0, t1 = p.ranges[rank]
        # 1. this rank pools its own complete blocks into their slots (fp64 oracle as the local pooling)
        pooled = torch.zeros(B, G, p.blocks, D, dtype=torch.float64)
        j0, j1 = p.block_range(rank)
        if j1 > j0:
            mine = orc.pool(c, orc.VALUE, x[:, j0 * m:j1 * m], z[:, j0 * m:j1 * m], bp)  # [B, nb, G, D]
            pooled[:, :, j0:j1] = torch.from_numpy(mine).permute(0, 2, 1, 3)
        # 2-3. the exchange step
        cp.gather_pooled(p, pooled, rank)
        halo = cp.exchange_halo(p, torch.from_numpy(x[:, t0:t1].copy()), rank)
        want_pooled = torch.from_numpy(orc.pool(c, orc.VALUE, x, z, bp)).permute(0, 2, 1, 3)
        lo, hi = p.halo_range(rank)
        ok = torch.allclose(pooled, want_pooled, rtol=0, atol=1e-12) and halo.shape[1] == hi - lo and \
            torch.equal(halo, torch.from_numpy(x[:, lo:hi].copy()))
        np.save(os.path.join(out_dir, f"ok{rank}.npy"), np.array([ok]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("T,m,w,world", [(16 * 9 + 5, 16, 20, 2), (8 * 12, 8, 30, 3)])
def test_exchange_gives_each_rank_its_prefix_and_halo(tmp_path, T, m, w, world):
    mp.start_processes(_rank_main, args=(world, _free_port(), T, m, w, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        assert bool(np.load(tmp_path / f"ok{r}.npy")[0]), f"rank {r}"


def _rank_rows(rank, world, port, T, m, w, out_dir):
    """Every rank's own output rows, from nothing but its own tokens and what
    the exchange step hands it, equal the whole-sequence oracle's rows."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import sys
        sys.path.insert(0, ROOT)
        from oracle import oracle as orc
        rng = np.random.default_rng(11)
        B, Hq, G, D, rho = 1, 4, 2, 16, 8
        q = rng.standard_normal((B, T, Hq, D))
        k, v = rng.standard_normal((B, T, G, D)), rng.standard_normal((B, T, G, D))
        zk, zv = rng.standard_normal((B, T, G, D)), rng.standard_normal((B, T, G, D))
        bk, bv = 0.3 * rng.standard_normal((m, G * D)), 0.3 * rng.standard_normal((m, G * D))
        sink = rng.standard_normal(Hq)
        c = orc.Config(Hq, G, D, False, m, w, rho)
        p = cp.plan(T, m, w, world)
        t0, t1 = p.ranges[rank]
        j0, j1 = p.block_range(rank)
        pk = torch.zeros(B, G, max(p.blocks, 1), D, dtype=torch.float64)
        pv = torch.zeros_like(pk)
        if j1 > j0:  # this rank's own blocks, pooled at their absolute positions
            pk[:, :, j0:j1] = torch.from_numpy(orc.pool(c, orc.KEY, k[:, t0:j1 * m], zk[:, t0:j1 * m], bk,
                                                        pos0=t0)).permute(0, 2, 1, 3)
            pv[:, :, j0:j1] = torch.from_numpy(orc.pool(c, orc.VALUE, v[:, t0:j1 * m], zv[:, t0:j1 * m], bv,
                                                        pos0=t0)).permute(0, 2, 1, 3)
        cp.gather_pooled(p, pk, rank)
        cp.gather_pooled(p, pv, rank)
        hk = cp.exchange_halo(p, torch.from_numpy(k[:, t0:t1].copy()), rank)
        hv = cp.exchange_halo(p, torch.from_numpy(v[:, t0:t1].copy()), rank)
        lo = t0 - hk.shape[1]
        # raw tokens this rank holds: its halo and its own; nothing else is filled in
        kr, vr = np.zeros_like(k), np.zeros_like(v)
        kr[:, lo:t1] = np.concatenate([hk.numpy(), k[:, t0:t1]], axis=1)
        vr[:, lo:t1] = np.concatenate([hv.numpy(), v[:, t0:t1]], axis=1)
        ek = pk[:, :, :p.blocks].permute(0, 2, 1, 3).numpy()
        ev = pv[:, :, :p.blocks].permute(0, 2, 1, 3).numpy()
        rows = np.arange(t0, t1)
        got = orc.attend(c, q[:, t0:t1], np.broadcast_to(rows, (B, len(rows))), ek, ev, kr, vr, np.full(B, T), sink)
        want = orc.forward(c, q, k, v, zk, zv, bk, bv, sink, rows=rows)
        np.save(os.path.join(out_dir, f"err{rank}.npy"), np.array([np.abs(got - want).max()]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("T,m,w,world", [(16 * 9 + 5, 16, 20, 2), (8 * 12 + 3, 8, 30, 3), (4 * 20, 4, 5, 4)])
def test_each_rank_computes_its_rows_from_the_exchange_alone(tmp_path, T, m, w, world):
    mp.start_processes(_rank_rows, args=(world, _free_port(), T, m, w, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        err = float(np.load(tmp_path / f"err{r}.npy")[0])
        assert err <= 1e-12, f"rank {r}: max-abs {err:.3e}"
