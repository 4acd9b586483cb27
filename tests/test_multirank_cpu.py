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


def _column_worker(rank, world, port, out):
    """Column-parallel layer on gloo ranks: each rank takes its 256-aligned
    column shard of the prepared layer, computes its slice of Y (with the
    CPU oracle standing in for the GPU kernels) and all-gathers the slices."""
    import rank_gemm_svdq_b200 as sv
    import synth
    from oracle import svdquant as sq
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = synth.custom_workload(24, 256, 1280, 16, "nvfp4", "bf16", n_out=3, factor=30.0, seed=8)
        p = sv.params(wl.K, wl.N, 16, "nvfp4", "bf16")
        blob, _ = sv.prepare(p, wl.Wt, wl.bias, wl.X)
        bounds = sv.shard_bounds(wl.N, world)
        n0, n1 = bounds[rank]
        q, shard = sv.shard_columns(p, blob, n0, n1)
        c = sv.blob_export(q, shard)
        L1, L2 = synth.bf16_bits_to_f64(c.L1), synth.bf16_bits_to_f64(c.L2)
        x64 = wl.x_f64()
        # the shard as a layer of its own: its weight rows, the layer's lambda and factors
        ref = sq.shard_columns(sq.prepare(x64, wl.Wt, wl.bias, 16, "nvfp4", "bf16", factors=(
            c.inv_lambda, synth.bf16_bits_to_f64(sv.blob_export(p, blob).L1),
            synth.bf16_bits_to_f64(sv.blob_export(p, blob).L2))), n0, n1)
        assert np.array_equal(L2, ref.L2) and np.array_equal(L1, ref.L1)
        y_local = torch.from_numpy(sq.forward(x64, ref))
        y = sv.all_gather_columns(y_local, bounds)
        out[rank] = (bounds, y.numpy())
    finally:
        dist.destroy_process_group()


def test_column_parallel_shards_gather_to_the_full_layer():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_column_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    import rank_gemm_svdq_b200 as sv
    import synth
    from oracle import svdquant as sq
    assert res[0][0] == [(0, 768), (768, 1280)]      # 5 tiles: 3 + 2
    wl = synth.custom_workload(24, 256, 1280, 16, "nvfp4", "bf16", n_out=3, factor=30.0, seed=8)
    p = sv.params(wl.K, wl.N, 16, "nvfp4", "bf16")
    blob, _ = sv.prepare(p, wl.Wt, wl.bias, wl.X)
    c = sv.blob_export(p, blob)
    x64 = wl.x_f64()
    full = sq.forward(x64, sq.prepare(x64, wl.Wt, wl.bias, 16, "nvfp4", "bf16", factors=(
        c.inv_lambda, synth.bf16_bits_to_f64(c.L1), synth.bf16_bits_to_f64(c.L2))))
    assert np.array_equal(res[0][1], full) and np.array_equal(res[1][1], full)


def test_shard_bounds():
    import rank_gemm_svdq_b200 as sv
    assert sv.shard_bounds(3072, 4) == [(0, 768), (768, 1536), (1536, 2304), (2304, 3072)]
    assert sv.shard_bounds(1280, 3) == [(0, 512), (512, 1024), (1024, 1280)]
    assert sv.shard_bounds(256, 1) == [(0, 256)]
