"""The N>1 path on CPU: 2 gloo ranks, each with its own shard of sequences.

Decode shards need no collective on the data path; what the ranks share is the
barrier and the max-reduce of the timed region.  These tests run that logic
with the gloo backend (world size 2) and the oracle as the per-rank compute.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_long_uocr_b200 import dist as udist


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import oracle
    import workloads
    r, _, w = udist.env_rank_world()
    assert (r, w) == (rank, world)
    # each rank decodes its own shard of 6 sequences
    lo, hi = udist.shard_range(6, rank, world)
    lens = [32 * (20 + 3 * i) + i for i in range(lo, hi)]
    case = workloads.make_case(lens, heads=2, shuffle=True, seed=udist.shard_seed(0, rank))
    res = oracle.run(case.q, case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool, case.block_table,
                     case.q_seq, case.q_pos)
    np.save(os.path.join(outdir, f"out{rank}.npy"), res["out"])
    # per-rank "elapsed time" and the reductions the bench uses
    mx = udist.max_over_ranks(1.5 + rank)
    sm = udist.sum_over_ranks(hi - lo)
    dist.barrier()
    with open(os.path.join(outdir, f"red{rank}.txt"), "w") as f:
        f.write(f"{mx} {sm}")
    dist.destroy_process_group()


def test_shard_range_partitions_units():
    for n in [0, 1, 5, 16, 17, 64]:
        for world in [1, 2, 3, 8]:
            parts = [udist.shard_range(n, r, world) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            assert all(parts[i][1] == parts[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in parts]
            assert max(sizes) - min(sizes) <= 1


def test_shard_seeds_differ_per_rank():
    assert len({udist.shard_seed(0, r) for r in range(8)}) == 8
    assert udist.shard_seed(0, 0) == 0


def test_reductions_without_a_process_group():
    assert udist.max_over_ranks(3.25) == 3.25
    assert udist.sum_over_ranks(2) == 2.0


@pytest.mark.timeout(300)
def test_two_gloo_ranks_shard_and_reduce(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    import oracle
    import workloads
    for rank in range(world):
        mx, sm = open(tmp_path / f"red{rank}.txt").read().split()
        assert float(mx) == 2.5 and float(sm) == 6.0
        # a rank's shard is exactly what one process computes for the same sequences and seed
        lo, hi = udist.shard_range(6, rank, world)
        lens = [32 * (20 + 3 * i) + i for i in range(lo, hi)]
        case = workloads.make_case(lens, heads=2, shuffle=True, seed=udist.shard_seed(0, rank))
        ref = oracle.run(case.q, case.idx_q, case.k_pool, case.v_pool, case.idx_k_pool, case.block_table,
                         case.q_seq, case.q_pos)["out"]
        assert np.array_equal(np.load(tmp_path / f"out{rank}.npy"), ref)
