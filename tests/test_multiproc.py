"""The N > 1 bench path on CPU: two gloo ranks (no GPU).

Sequences are independent, so each rank runs its own replica of the batch and
no collective touches the data path; the only cross-rank step is the timing
reduction (slowest rank) and the whole-job aggregation.  These tests run that
host logic on two processes with the gloo backend.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        slowest = bench._max_over_ranks(times[rank], world, "cpu")
        rate = bench.whole_job_rate(268435456 / 1e9, 100, slowest, world)
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(f"{slowest} {rate}")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("times", [[5.0, 7.5], [9.0, 3.0]])
def test_two_gloo_ranks_agree_on_the_slowest_time(tmp_path, times):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), times,
                                      str(tmp_path)),
                       nprocs=world, start_method="spawn", join=True)
    got = [open(tmp_path / f"r{r}.txt").read().split() for r in range(world)]
    slowest = max(times)
    for s, rate in got:
        assert float(s) == slowest
        # two replicas of 268 MB of K/V per step, 100 steps
        assert float(rate) == pytest.approx(
            2 * 0.268435456 * 100 / (slowest / 1e3))


def test_single_rank_needs_no_process_group():
    assert bench._max_over_ranks(4.2, 1, "cpu") == 4.2
    assert bench.whole_job_rate(2.0, 10, 20.0, 1) == pytest.approx(1000.0)
