"""The multi-GPU host logic of bench.py on CPU: two gloo ranks (world size 2).

Under torchrun every rank runs its own independently seeded call (weak scaling: no
collective on the data path); the whole-job numbers take the max over ranks of each
time and the sum over ranks of the work.  These tests run that reduction, the seeding
and the reference arm's rank handling without a GPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from inputs import WORKLOADS


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        times = [10.0 + 2.0 * rank, 1.0 + rank]        # step time, e2e time
        work = [100.0, 50.0][rank]
        (t_max, e_max), total = bench.combine_over_ranks(dist, torch.device("cpu"), times, work)
        out[rank] = (t_max, e_max, total)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_combine_over_ranks_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for r in range(world):
        t_max, e_max, total = res[r]
        assert t_max == 12.0 and e_max == 2.0 and total == 150.0


def test_rank_seeds_differ():
    wl = WORKLOADS["tiny"]
    seeds = {bench.rank_seed(wl, r) for r in range(8)}
    assert len(seeds) == 8
    assert bench.rank_seed(wl, 0) == wl.seed


def test_reference_arm_other_ranks_do_nothing(monkeypatch):
    monkeypatch.setenv("RANK", "1")

    class A:
        steps, warmup, gpus, ref_budget = 3, 3, 2, 10.0

    assert bench.run_reference(A(), WORKLOADS["tiny"]) is None


@pytest.mark.parametrize("steps,warmup", [(100, 5), (10, 3), (1, 3), (1000, 10)])
def test_reference_budget_bounded(steps, warmup):
    b = bench.reference_step_budget(steps, warmup)
    assert 0.2 <= b <= 10.0
    assert b * (steps + warmup) <= max(150.0, 0.2 * (steps + warmup)) + 1e-9
