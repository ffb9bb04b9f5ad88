"""Host logic of the multi-rank bench path, on CPU with two gloo ranks.

Under torchrun every rank runs its own batch of independent sequences (weak scaling, no
data-path collective); the only collectives are the barrier and the max over ranks of the
device timings.  These tests run that logic with the gloo backend: each rank draws a
different batch, the timing reduction returns the slowest rank's time on every rank, and
the whole-job rate counts the units of all ranks over that time.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import csa_inputs as CI
        # each rank its own batch: a different seed and different data
        seed = bench.rank_seed(1, rank)
        wl = CI.make_workload(0, seed=seed)
        checksum = float(np.abs(np.asarray(wl.tensors["q"], np.float64)).sum())
        sums = [None] * world
        dist.all_gather_object(sums, (seed, checksum))
        # the slowest rank's time on every rank
        my_ms = 1.0 + 2.0 * rank
        slowest = bench.max_over_ranks(my_ms, world, "cpu")
        rate = bench.job_rate(16, world, slowest)
        dist.barrier()
        np.save(os.path.join(out_dir, f"rank{rank}.npy"),
                np.array([slowest, rate] + [s for s, _ in sums] + [c for _, c in sums], np.float64))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_weak_scaling(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [np.load(tmp_path / f"rank{r}.npy") for r in range(world)]
    for r in res:
        slowest, rate = r[0], r[1]
        assert slowest == pytest.approx(3.0)                    # max of 1 ms and 3 ms
        assert rate == pytest.approx(16 * world / 3e-3)         # all ranks' tokens over the slowest time
        seeds, sums = r[2:2 + world], r[2 + world:]
        assert len(set(seeds.tolist())) == world                # distinct batches
        assert sums[0] != sums[1]
    # every rank sees the same reduced values
    assert res[0][0] == res[1][0] and res[0][1] == res[1][1]


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(2.5, 1, "cpu") == 2.5
    assert bench.job_rate(16, 1, 0.5) == pytest.approx(32000.0)
    assert bench.rank_seed(3, 0) != bench.rank_seed(3, 1)
