"""Column shards of a prepared layer (output features [n0, n1), for
column-parallel use on several GPUs): the oracle's shard against the full
layer's columns, and the host library's svdq_shard_columns against slices of
the full blob.  No GPU."""
import numpy as np
import pytest

import rank_gemm_svdq_b200 as sv
import synth
from oracle import svdquant as sq


@pytest.mark.parametrize("fmt,dtype", [("int4", "fp16"), ("nvfp4", "bf16")])
def test_oracle_shard_is_the_full_layers_columns(fmt, dtype):
    wl = synth.custom_workload(20, 256, 768, 16, fmt, dtype, n_out=3, factor=30.0, seed=21)
    x64 = wl.x_f64()
    ref = sq.prepare(x64, wl.Wt, wl.bias, 16, fmt, dtype)
    full = sq.forward(x64, ref)
    for n0, n1 in ((0, 256), (256, 768), (512, 768)):
        assert np.array_equal(sq.forward(x64, sq.shard_columns(ref, n0, n1)), full[:, n0:n1])


@pytest.mark.parametrize("fmt,dtype,rank", [("int4", "bf16", 32), ("nvfp4", "fp16", 16), ("nvfp4", "bf16", 0)])
def test_shard_columns_slices_the_blob(fmt, dtype, rank):
    wl = synth.custom_workload(16, 512, 1024, rank, fmt, dtype, n_out=3, factor=30.0, seed=22)
    p = sv.params(wl.K, wl.N, rank, fmt, dtype)
    blob, _ = sv.prepare(p, wl.Wt, wl.bias, wl.X)
    c = sv.blob_export(p, blob)
    for n0, n1 in ((0, 256), (256, 1024), (768, 1024)):
        q, b = sv.shard_columns(p, blob, n0, n1)
        assert q.N == n1 - n0 and (q.K, q.rank, q.fmt) == (p.K, p.rank, p.fmt)
        assert sv.blob_check(q, b) == sv.OK
        s = sv.blob_export(q, b)
        assert np.array_equal(s.inv_lambda.view(np.uint32), c.inv_lambda.view(np.uint32))
        assert np.array_equal(s.L1, c.L1) and np.array_equal(s.L2, c.L2[:, n0:n1])
        assert np.array_equal(s.wcodes, c.wcodes[n0:n1])
        assert np.array_equal(s.wscales.view(np.uint8), c.wscales[n0:n1].view(np.uint8))
        assert (s.s_gx, s.s_gw) == (c.s_gx, c.s_gw)
        assert np.array_equal(s.bias, c.bias[n0:n1])


def test_shard_columns_rejects_bad_ranges():
    wl = synth.custom_workload(8, 256, 512, 16, "nvfp4", "bf16", n_out=2, factor=20.0, seed=23)
    p = sv.params(wl.K, wl.N, 16, "nvfp4", "bf16")
    blob, _ = sv.prepare(p, wl.Wt, wl.bias, wl.X)
    for n0, n1 in ((128, 512), (0, 384), (256, 256), (0, 768), (-256, 256)):
        with pytest.raises(sv.SVDQError) as e:
            sv.shard_columns(p, blob, n0, n1)
        assert e.value.status == sv.ERR_INVALID_ARG
