"""Host-side logic of multi-GPU runs, on CPU with the gloo backend (world size 2):
every rank runs an independent problem (distinct seeds), the step time is the max
over ranks, and the whole-job value counts every rank's tokens."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, wsz, lr = bench.dist_env()
    bench.dist_setup(wsz, "gloo")
    bench.barrier()
    t = bench.max_over_ranks(1.5 + rank)             # per-rank "step time" in ms
    seeds = [None] * wsz
    torch.distributed.all_gather_object(seeds, bench.rank_seed(1002, r))
    value = wsz * 65536 / (t / 1e3)
    out[rank] = (t, tuple(seeds), value)
    torch.distributed.destroy_process_group()


def test_two_gloo_ranks_max_time_and_distinct_problems():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()          # no fork of this (threaded) process
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == pytest.approx(2.5)
    assert len(set(out[0][1])) == world
    assert out[0][2] == pytest.approx(2 * 65536 / 2.5e-3)


def test_single_process_identity():
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.rank_seed(5, 0) == 5
