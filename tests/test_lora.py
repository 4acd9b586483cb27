"""LoRA adapters added to a prepared layer without re-quantisation
("SVDQuant是什么？…" 概述简介 and 功能特色, LoRA集成): the oracle's construction
pinned against plain matrix products, and the host library's svdq_append_lora
against the oracle (bit-exact factors, untouched 4-bit residual).  No GPU."""
import numpy as np
import pytest

import rank_gemm_svdq_b200 as sv
import synth
from oracle import formats, svdquant as sq


def _layer(fmt, dtype, smooth, M=24, K=256, N=128, rank=16, seed=3):
    wl = synth.custom_workload(M, K, N, rank, fmt, dtype, n_out=3, factor=30.0, seed=seed, smooth=smooth)
    x64 = wl.x_f64()
    ref = sq.prepare(x64, wl.Wt, wl.bias, rank, fmt, dtype, wl.alpha, smooth)
    return wl, x64, ref


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_oracle_lora_adds_exactly_xab_without_smoothing(fmt):
    """lambda = 1 and adapter entries exact in the dtype: the layer output grows
    by exactly X A B (a plain product of the inputs), up to f64 summation."""
    wl, x64, ref = _layer(fmt, "bf16", smooth=False)
    rng = np.random.default_rng(0)
    A = rng.integers(-4, 5, size=(wl.K, 16)) / 8.0
    B = rng.integers(-4, 5, size=(16, wl.N)) / 16.0
    ref2 = sq.append_lora(ref, A, B)
    assert ref2.rank == ref.rank + 16 and ref2.wq is ref.wq and ref2.R is ref.R
    dY = sq.forward(x64, ref2) - sq.forward(x64, ref)
    xab = (x64 @ A) @ B
    assert np.max(np.abs(dY - xab)) <= 1e-9 * max(1.0, np.max(np.abs(xab)))


@pytest.mark.parametrize("fmt,dtype", [("int4", "fp16"), ("nvfp4", "bf16")])
def test_oracle_lora_with_smoothing_matches_xab_to_the_dtype(fmt, dtype):
    """With smoothing the adapter rides on X^ = X diag(lambda)^-1, so its L1
    columns are diag(lambda) A: the increase is X A B up to the 16-bit rounding
    of lambda A, of B and of X^ (a few 2^-9 relative)."""
    wl, x64, ref = _layer(fmt, dtype, smooth=True)
    A, B = synth.make_lora(7, wl.K, wl.N, 32)
    ref2 = sq.append_lora(ref, A, B)
    dY = sq.forward(x64, ref2) - sq.forward(x64, ref)
    xab = (x64 @ A.astype(np.float64)) @ B.astype(np.float64)
    assert sq.rel_fro(dY, xab) <= 2.0 ** -6
    # dropping the lambda factor is far off: the pin sees a missing diag(lambda)
    bad = sq.Prepared(ref.fmt, ref.dtype, ref.rank + 32, ref.inv_lambda, ref.lam_eff,
                      np.hstack([ref.L1, formats.to_dtype(A.astype(np.float64), dtype)]),
                      np.vstack([ref.L2, formats.to_dtype(B.astype(np.float64), dtype)]),
                      ref.sigma, ref.R, ref.wq, ref.s_gx, ref.bias)
    assert sq.rel_fro(sq.forward(x64, bad) - sq.forward(x64, ref), xab) > 0.1


def _factors_f64(p, c):
    if p.act_dtype == sv.F16:
        return c.L1.view(np.float16).astype(np.float64), c.L2.view(np.float16).astype(np.float64)
    return synth.bf16_bits_to_f64(c.L1), synth.bf16_bits_to_f64(c.L2)


@pytest.mark.parametrize("fmt,dtype,rank,r_lora", [("int4", "fp16", 16, 16), ("nvfp4", "bf16", 32, 32),
                                                    ("nvfp4", "fp16", 0, 48), ("int4", "bf16", 96, 32)])
def test_append_lora_matches_oracle(fmt, dtype, rank, r_lora):
    wl = synth.custom_workload(16, 512, 256, rank, fmt, dtype, n_out=3, factor=30.0, seed=11)
    p = sv.params(wl.K, wl.N, rank, fmt, dtype, wl.alpha, wl.smooth)
    blob, _ = sv.prepare(p, wl.Wt, wl.bias, wl.X)
    A, B = synth.make_lora(5, wl.K, wl.N, r_lora)
    q, blob2 = sv.append_lora(p, blob, A, B)
    assert q.rank == rank + r_lora and sv.blob_check(q, blob2) == sv.OK
    c, c2 = sv.blob_export(p, blob), sv.blob_export(q, blob2)
    # the 4-bit residual, its scales, lambda, tensor scales and bias are untouched
    assert np.array_equal(c.wcodes, c2.wcodes)
    assert np.array_equal(c.wscales.view(np.uint8), c2.wscales.view(np.uint8))
    assert np.array_equal(c.inv_lambda.view(np.uint32), c2.inv_lambda.view(np.uint32))
    assert (c.s_gx, c.s_gw) == (c2.s_gx, c2.s_gw) and np.array_equal(c.bias, c2.bias)
    # the factors are the oracle's appended ones, bit for bit
    L1, L2 = _factors_f64(p, c)
    ref = sq.prepare(wl.x_f64(), wl.Wt, wl.bias, rank, fmt, dtype, wl.alpha, wl.smooth,
                     factors=(c.inv_lambda, L1, L2))
    ref2 = sq.append_lora(ref, A, B)
    L1b, L2b = _factors_f64(q, c2)
    assert np.array_equal(L1b, ref2.L1) and np.array_equal(L2b, ref2.L2)


def test_append_lora_stacks():
    """Two adapters appended one after the other give the same blob as the two
    appended at once."""
    wl = synth.custom_workload(8, 256, 256, 16, "nvfp4", "bf16", n_out=2, factor=20.0, seed=2)
    p = sv.params(wl.K, wl.N, 16, "nvfp4", "bf16")
    blob, _ = sv.prepare(p, wl.Wt, wl.bias, wl.X)
    A1, B1 = synth.make_lora(1, wl.K, wl.N, 16)
    A2, B2 = synth.make_lora(2, wl.K, wl.N, 32)
    q1, b1 = sv.append_lora(p, blob, A1, B1)
    q2, b2 = sv.append_lora(q1, b1, A2, B2)
    q3, b3 = sv.append_lora(p, blob, np.hstack([A1, A2]), np.vstack([B1, B2]))
    assert q2.rank == q3.rank == 64 and np.array_equal(b2, b3)


def test_append_lora_rejects_bad_arguments():
    wl = synth.custom_workload(8, 256, 256, 112, "int4", "bf16", n_out=2, factor=20.0, seed=4)
    p = sv.params(wl.K, wl.N, 112, "int4", "bf16")
    blob, _ = sv.prepare(p, wl.Wt, wl.bias, wl.X)
    for r_lora in (8, 32):          # not a multiple of 16 / rank above 128
        A, B = synth.make_lora(1, wl.K, wl.N, r_lora)
        with pytest.raises(sv.SVDQError) as e:
            sv.append_lora(p, blob, A, B)
        assert e.value.status == sv.ERR_INVALID_ARG
    A, B = synth.make_lora(1, wl.K, wl.N, 16)
    bad = blob.copy()
    bad[-1] ^= 1
    with pytest.raises(sv.SVDQError) as e:
        sv.append_lora(p, bad, A, B)
    assert e.value.status == sv.ERR_BLOB
