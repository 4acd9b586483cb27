"""Multi-rank host logic of the benchmark, as 2 gloo ranks on the CPU.

The layer shards by tokens with no data-path collective: every rank runs its
own replica on its own seeded batch, and the job's time is the slowest rank's.
These tests run the two pieces of rank-dependent host code (batch generation
and the max-over-ranks reduction) under torch.distributed with world size 2.
"""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import bench
    import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = synth.custom_workload(64, 512, 256, 16, "nvfp4", "bf16", n_out=5, factor=50.0, seed=0)
        x = bench.replica_batch(wl, rank)
        # rank-dependent "step time"; every rank must see the largest one
        t = bench.max_over_ranks(1.5 + rank, dist, torch.device("cpu"))
        out[rank] = (t, int(np.frombuffer(x.tobytes(), np.uint8).astype(np.uint64).sum()), x.shape)
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_distinct_batches():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert set(res) == {0, 1}
    assert res[0][0] == res[1][0] == 2.5            # max over ranks
    assert res[0][2] == res[1][2]                   # same shape
    assert res[0][1] != res[1][1]                   # own batch per replica


def test_single_process_reduction_is_identity():
    import bench
    assert bench.max_over_ranks(3.25, None, None) == 3.25
