"""Host logic of multi-rank benchmarking on CPU (gloo, world size 2).

Every rank runs its own batch (weak scaling, no collective on the data path);
the ranks only agree on the slowest rank's time. This checks the per-rank
seeds, the max-over-ranks reduction, the barrier and the whole-job value.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w = W.WORKLOADS["qwen2.5-1.5b"]
    rng = np.random.default_rng(W.shard_seed(0, rank))
    lens = W.draw_context_lens(w, rng)
    elapsed = 10.0 + 5.0 * rank                      # rank 1 is the slow one
    bench.barrier(world)
    mx = bench.reduce_max(elapsed, world)
    np.save(os.path.join(out_dir, f"rank{rank}.npy"), np.array([mx, lens.sum()], dtype=np.float64))
    dist.destroy_process_group()


def test_two_ranks_gloo(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r0 = np.load(tmp_path / "rank0.npy")
    r1 = np.load(tmp_path / "rank1.npy")
    assert r0[0] == r1[0] == 15.0                    # both ranks see the slowest time
    assert r0[1] != r1[1]                            # each rank drew its own batch


def test_whole_job_value_is_weak_scaling():
    import bench
    one = bench.whole_job_gbs(1, 10 ** 9, 100, 50.0)
    eight = bench.whole_job_gbs(8, 10 ** 9, 100, 50.0)
    assert eight == pytest.approx(8 * one)
    assert one == pytest.approx(2000.0)             # 100 GB in 50 ms
