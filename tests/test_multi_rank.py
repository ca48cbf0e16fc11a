"""The N > 1 path on CPU: world-size-2 gloo process groups.

Decode shards by sequence with no data-path collective; what a multi-GPU run
adds is host logic (per-rank workloads, the max over ranks of the device
timings, the whole-job per-token figure) and the launch of one process per
rank.  These tests run that logic in two gloo ranks, and run bench.py's
reference arm under torch.distributed.run with two ranks (rank 0 alone works
and prints; the other rank exits 0 without work).
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_compressed_long_b200 import ranks, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = ranks.rank_workload(synth.scaled(synth.WORKLOADS["ragged_gqa_decode_append"], ctx=(40, 90), batch=3,
                                             steps=2), rank)
        inp = synth.make(w)
        # a rank-dependent "device time" per quantity; the job's is the slowest rank's
        mine = [1.0 + rank, 5.0 - rank, 2.5]
        red = ranks.max_over_ranks(mine)
        lo, hi = ranks.shard_range(7, world, rank)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), q=inp.q.float().numpy(), lens=inp.lens, red=np.array(red),
                 shard=np.array([lo, hi]), seed=w.seed)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_and_own_their_sequences(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r = [np.load(tmp_path / f"r{i}.npz") for i in range(world)]
    for x in r:  # every rank holds the same reduced values: the element-wise max
        assert x["red"].tolist() == [2.0, 5.0, 2.5]
    assert int(r[0]["seed"]) != int(r[1]["seed"])
    assert not np.array_equal(r[0]["q"], r[1]["q"])  # disjoint (independently drawn) sequences
    shards = [tuple(x["shard"].tolist()) for x in r]
    assert shards == [(0, 4), (4, 7)]


def test_max_over_ranks_without_a_group_is_identity():
    assert ranks.max_over_ranks([3.0, 1.5]) == [3.0, 1.5]


@pytest.mark.parametrize("n,world", [(0, 3), (5, 1), (7, 2), (32, 8), (3, 8)])
def test_shard_range_covers_each_unit_once(n, world):
    owned = []
    for rank in range(world):
        lo, hi = ranks.shard_range(n, world, rank)
        assert 0 <= lo <= hi <= n
        owned += list(range(lo, hi))
    assert owned == list(range(n))
    sizes = [ranks.shard_range(n, world, k)[1] - ranks.shard_range(n, world, k)[0] for k in range(world)]
    assert max(sizes) - min(sizes) <= 1


def test_job_us_per_token_counts_all_ranks_tokens():
    # 32 sequences per rank, 4 ranks, a 1 ms step: 128 tokens per ms
    assert ranks.job_us_per_token(1.0, 32, 4) == pytest.approx(1000.0 / 128)


def test_reference_arm_under_two_ranks_prints_one_line():
    env = dict(os.environ, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0
