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


# --------------------------------------------------------------------------------------
# Data-parallel prefill of a packed batch: ranks take whole sequences (shard.py). Each
# rank computes its shard on its own (here the FP64 oracle stands in for the GPU call,
# which needs a B200); the gathered shards must equal the whole batch computed at once.
def test_shard_sequences_balances_and_covers():
    from mamba_ssd_state_02_b200 import shard
    lens = [8192, 512, 3000, 7000, 100, 2500, 6000, 0, 1]
    for world in (1, 2, 3, 4, 8, 16):
        parts = shard.shard_sequences(lens, world)
        assert len(parts) == world
        assert sorted(i for p in parts for i in p) == list(range(len(lens)))
        loads = [sum(lens[i] for i in p) for p in parts]
        # LPT bound: no rank exceeds the average by more than the longest sequence
        assert max(loads) <= sum(lens) / world + max(lens)
        assert all(p == sorted(p) for p in parts)
    spans, cu = shard.local_batch([0, 5, 5, 12, 20], [0, 2, 3])
    assert spans == [(0, 5), (5, 12), (12, 20)] and cu == [0, 5, 12, 20]
    t = torch.arange(20).view(20, 1)
    assert shard.take_rows(t, [(2, 4), (10, 11)]).view(-1).tolist() == [2, 3, 10]


def _dp_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    from mamba_ssd_state_02_b200 import shard, workloads as W
    from oracle import oracle as O
    w = W.Workload("dp", nheads=2, headdim=8, ngroups=1, dstate=8, chunk=64, dtype=torch.float32,
                   seqlens=[300, 17, 129, 0, 211, 64], varlen=True, init="normal", seed=123)
    d = W.make_all(w)
    cu = d["cu_seqlens"].tolist()
    mine = shard.shard_sequences(w.seqlens, world)[rank]
    spans, cu_local = shard.local_batch(cu, mine)
    take = lambda k: shard.take_rows(d[k], spans)
    y, fin = O.ssd_scan(take("x"), take("dt_raw"), d["dt_bias"], d["A"], take("B"), take("C"), d["D"],
                        init_state=d["init_state"][mine], cu_seqlens=torch.tensor(cu_local, dtype=torch.int32))
    got = [None] * world
    torch.distributed.all_gather_object(got, (mine, spans, y, fin))
    out[rank] = got
    torch.distributed.destroy_process_group()


def test_two_gloo_ranks_data_parallel_prefill_equals_whole_batch():
    from mamba_ssd_state_02_b200 import workloads as W
    from oracle import oracle as O
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_dp_worker, args=(world, port, out), nprocs=world, join=True)
    w = W.Workload("dp", nheads=2, headdim=8, ngroups=1, dstate=8, chunk=64, dtype=torch.float32,
                   seqlens=[300, 17, 129, 0, 211, 64], varlen=True, init="normal", seed=123)
    d = W.make_all(w)
    y_all, fin_all = O.ssd_scan(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                                init_state=d["init_state"], cu_seqlens=d["cu_seqlens"])
    y = torch.full_like(y_all, float("nan"))
    fin = torch.full_like(fin_all, float("nan"))
    seen = []
    for mine, spans, y_r, fin_r in out[0]:                # rank 0's gather holds every shard
        row = 0
        for k, (i, (a, b)) in enumerate(zip(mine, spans)):
            y[a:b] = torch.as_tensor(y_r)[row:row + (b - a)]
            fin[i] = torch.as_tensor(fin_r)[k]
            row += b - a
        seen += mine
    assert sorted(seen) == list(range(len(w.seqlens)))
    assert torch.equal(y, y_all)                          # each sequence's result is independent
    assert torch.equal(fin, fin_all)
