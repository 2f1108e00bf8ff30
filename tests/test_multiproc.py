"""The N > 1 path of bench.py on CPU: two gloo ranks, each its own batch (no
collective on the data path); timing is the max over ranks and the units are
summed."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank)})
    import bench
    import torch.distributed as dist
    ws, r, local, _ = bench.dist_setup()
    try:
        assert (ws, r) == (world, rank)
        bench.barrier(ws)
        # rank r "ran" for 1+r seconds over 10*(r+1) units
        t, u = bench.aggregate(1.0 + r, 10.0 * (r + 1), ws)
        seed = bench.rank_seed(2, r)
        seeds = [None] * ws
        dist.all_gather_object(seeds, seed)
        # each rank's batch: same shape, its own values
        import workloads
        wl = workloads.long_context(seed=seed, steps=1, batch=1, seq_len=64, num_blocks=8)
        st = next(iter(wl.steps))
        sums = [None] * ws
        dist.all_gather_object(sums, float(st.k_new.float().sum()))
        out[rank] = (t, u, seeds, sums)
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_and_sharding():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:  # no fork of this threaded process
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        t, u, seeds, sums = res[r]
        assert t == 2.0                      # max over ranks
        assert u == 30.0                     # units of all ranks
        assert len(set(seeds)) == world      # distinct batches
        assert sums[0] != sums[1]
