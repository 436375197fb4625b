"""The multi-GPU benchmark path on the CPU: two gloo ranks, no GPU.

Each rank runs an independent replica (its own seed); the job's rate is all ranks' query
tokens over the slowest rank's time, and every rank must see the same aggregate."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from workloads import CONFIGS, generate, small


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, ms, queries, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = bench.aggregate(ms[rank], queries[rank], world)
        seed = bench.replica_seed(CONFIGS["prefill64k"].seed, rank)
        out[rank] = (res[0], res[1], seed)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ms", [(2.0, 3.0), (5.0, 1.0)])
def test_two_rank_aggregate(ms):
    world, port = 2, _free_port()
    queries = (65536, 65536)
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank, args=(world, port, ms, queries, out), nprocs=world,
                           start_method="spawn")
        res = dict(out)
    mx = max(ms)
    for r in range(world):
        assert res[r][0] == pytest.approx(mx)
        assert res[r][1] == pytest.approx(sum(queries) / (mx * 1e-3))
    assert res[0][2] != res[1][2]                      # independent replicas


def test_replicas_draw_different_inputs():
    wl = small("rep", Nq=256, Nk=256, d=8, s=8, w=32)
    a = generate(wl.with_(seed=bench.replica_seed(wl.seed, 0)))
    b = generate(wl.with_(seed=bench.replica_seed(wl.seed, 1)))
    assert not (a.Q == b.Q).all()


def test_single_rank_needs_no_process_group():
    ms, value = bench.aggregate(4.0, 1000, 1)
    assert ms == 4.0 and value == pytest.approx(1000 / 4e-3)
