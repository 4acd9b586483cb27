"""svdq_linear on the GPU against the CPU oracle, through the C ABI.

Bit-exact: activation codes and scales (and, via the host prepare, weight
codes and scales).  Y: relative Frobenius error <= 1e-3 against the oracle's
output rounded to bf16.  Guard rows around Y and a guard tail behind the
workspace catch out-of-bounds writes.
"""
import numpy as np
import pytest

import rank_gemm_svdq_b200 as sv
import synth
from oracle import formats
from tests import gpu_cases as G

pytestmark = pytest.mark.gpu


def test_probe_cvt_matches_oracle_encoders(gpu):
    """The GPU's cvt.rn.satfinite to E2M1 / E4M3 equals the oracle's
    round-to-nearest-even encoders (ties, saturation, signed zero)."""
    import torch
    rng = np.random.default_rng(1)
    e2 = formats.E2M1_VALUES[:8]; e4 = formats.E4M3_VALUES[:0x7F]
    mids = np.concatenate([0.5 * (e2[:-1] + e2[1:]), 0.5 * (e4[:-1] + e4[1:])]).astype(np.float32)
    x = np.concatenate([mids, np.nextafter(mids, np.float32(np.inf)), np.nextafter(mids, np.float32(0)),
                        e2.astype(np.float32), e4.astype(np.float32),
                        rng.uniform(0, 8, 20000).astype(np.float32),
                        np.exp(rng.uniform(-14, 7, 20000)).astype(np.float32),
                        np.array([1e-30, 1e30, 500.0, 464.0, 6.5, 7.0, 0.0], np.float32)])
    x = np.concatenate([x, -x])
    xd = torch.from_numpy(x).cuda()
    o2 = torch.zeros(len(x), dtype=torch.uint8, device="cuda")
    o4 = torch.zeros(len(x), dtype=torch.uint8, device="cuda")
    sv.probe_cvt(xd, o2, o4)
    torch.cuda.synchronize()
    g2, g4 = o2.cpu().numpy(), o4.cpu().numpy()
    r2 = formats.e2m1_encode(x.astype(np.float64)); r4 = formats.e4m3_encode(x.astype(np.float64))
    bad2 = np.flatnonzero(g2 != r2); bad4 = np.flatnonzero(g4 != r4)
    assert len(bad2) == 0, (x[bad2[:8]], g2[bad2[:8]], r2[bad2[:8]])
    assert len(bad4) == 0, (x[bad4[:8]], g4[bad4[:8]], r4[bad4[:8]])


def test_probe_division_matches_ieee(gpu):
    """The activation kernel's quotient (reciprocal + FMA correction) equals
    the IEEE round-to-nearest division on random operands and on operands
    placed at and around the code decision points (E2M1 midpoints, INT4
    half-integers) times the divisor."""
    import torch
    rng = np.random.default_rng(2)
    n = 1 << 20
    d = np.exp(rng.uniform(np.log(1e-37), np.log(1e30), n)).astype(np.float32)
    t = rng.uniform(-8, 8, n)
    marks = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1.5, 2.5, 3.5, 4.5, 5.5, 6.5, 7.0])
    t[: n // 2] = rng.choice(marks, n // 2) * rng.choice([-1.0, 1.0], n // 2)
    v = (t * d).astype(np.float32)
    k = n // 4
    v[:k] = np.nextafter(v[:k], np.float32(np.inf))
    v[k:2 * k] = np.nextafter(v[k:2 * k], np.float32(-np.inf))
    v[-64:] = 0.0
    vd, dd = torch.from_numpy(v).cuda(), torch.from_numpy(d).cuda()
    q = torch.empty_like(vd); qi = torch.empty_like(vd)
    sv.probe_div(vd, dd, q, qi)
    torch.cuda.synchronize()
    a, b = q.cpu().numpy(), qi.cpu().numpy()
    bad = np.flatnonzero(a.view(np.uint32) != b.view(np.uint32))
    assert len(bad) == 0, (v[bad[:5]], d[bad[:5]], a[bad[:5]], b[bad[:5]])
    # and the IEEE quotient equals the host's fp32 division
    assert np.array_equal(b.view(np.uint32), (v / d).astype(np.float32).view(np.uint32))


def test_tiny_int4_config(gpu):
    """The tiny INT4 layer (M=256, K=512, N=512, fp16, rank 16, 4 outlier
    channels x100): every output and every code against the oracle."""
    pp = G.prepared_preset("tiny_int4")
    run = G.run_gpu(pp, pp.wl.X)
    G.compare(pp, pp.wl.X, run)


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("M,rank", [(1, 16), (127, 32), (129, 0), (300, 16), (384, 48)])
def test_small_shapes(gpu, fmt, dtype, M, rank):
    """Ragged token counts (1, 127, 129, 300: partial 128-row tiles), several
    tiles along N and K, rank 0 (no low-rank branch) and rank 48 (two
    low-rank K-steps for fp16)."""
    wl = synth.custom_workload(M, 512, 768, rank, fmt, dtype, n_out=5, factor=80.0, seed=M + rank)
    pp = G.prepare(wl)
    run = G.run_gpu(pp, wl.X)
    G.compare(pp, wl.X, run)


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_zero_input_gives_bias(gpu, fmt):
    wl = synth.custom_workload(64, 256, 512, 16, fmt, "bf16", n_out=2, factor=10.0, seed=5)
    pp = G.prepare(wl)
    X0 = np.zeros_like(wl.X)
    run = G.run_gpu(pp, X0)
    assert np.all(run.codes.view(np.uint8) == 0)
    assert np.array_equal(run.Y, np.broadcast_to(formats.to_bf16(wl.bias.astype(np.float64)), run.Y.shape))


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_repeat_calls_are_bitwise_identical(gpu, fmt):
    wl = synth.custom_workload(200, 512, 512, 32, fmt, "bf16", n_out=4, factor=50.0, seed=9)
    pp = G.prepare(wl)
    a = G.run_gpu(pp, wl.X)
    b = G.run_gpu(pp, wl.X)
    assert np.array_equal(a.Y, b.Y) and np.array_equal(a.codes, b.codes)


@pytest.mark.parametrize("name", ["flux_qkv_int4", "flux_ffn_up_nvfp4", "ffn_down_nvfp4", "ffn_down_int4"])
def test_full_size_config(gpu, name):
    """Full-size FLUX / FFN-down layers in the benchmark's launch configuration:
    every code and scale bit-exact, every output element of Y against the
    oracle, globally and per 128 x 256 tile."""
    pp = G.prepared_preset(name)
    X = pp.wl.X
    run = G.run_gpu(pp, X)
    res = G.compare(pp, X, run)
    print(name, res)


@pytest.mark.parametrize("shape", ["var_up_nvfp4", "var_down_nvfp4"])
def test_var_token_sweep(gpu, shape):
    """Infinity-VAR style projections at every token count of the sweep:
    every code and every output element (globally and per tile)."""
    pp = G.prepared_preset(shape)
    for M in synth.VAR_TOKENS:
        X = pp.wl.X[:M]
        run = G.run_gpu(pp, X)
        print(shape, M, G.compare(pp, X, run))


def test_status_word_clean(gpu):
    assert sv.get_status() == sv.OK


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("M", [1, 5, 16, 17, 64, 65, 100, 128])
def test_small_m_split_k(gpu, dtype, M):
    """Few tokens: the NVFP4 GEMM with the weight tile as the A operand and
    16, 64 or 128 token columns (each width at its edges), splitting K over
    idle SMs up to 64 tokens and adding the partial sums in K order.  Two
    calls in a row give identical bits (the arrival counters reset) and match
    the oracle."""
    wl = synth.custom_workload(M, 2048, 1024, 32, "nvfp4", dtype, n_out=6, factor=60.0, seed=40 + M)
    pp = G.prepare(wl)
    a = G.run_gpu(pp, wl.X)
    b = G.run_gpu(pp, wl.X)
    G.compare(pp, wl.X, a)
    assert np.array_equal(a.Y, b.Y)


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("M", [100, 200])
def test_max_rank(gpu, fmt, dtype, M):
    """Rank 128 (the largest allowed): several low-rank K-steps (up to 6 for
    fp16's three segments) and the activation kernel's two-buffer L1 ring,
    through both NVFP4 GEMM kernels (up to 128 tokens and above)."""
    wl = synth.custom_workload(M, 1024, 512, 128, fmt, dtype, n_out=8, factor=40.0, seed=77 + M)
    pp = G.prepare(wl)
    run = G.run_gpu(pp, wl.X)
    G.compare(pp, wl.X, run)


@pytest.mark.parametrize("fmt,K", [("int4", 256), ("nvfp4", 256)])
def test_smallest_shapes(gpu, fmt, K):
    """One K slab and one 256-column output tile."""
    wl = synth.custom_workload(7, K, 256, 16, fmt, "bf16", n_out=2, factor=30.0, seed=3)
    pp = G.prepare(wl)
    run = G.run_gpu(pp, wl.X)
    G.compare(pp, wl.X, run)


def test_zero_tokens_is_a_no_op(gpu):
    import torch
    wl = synth.custom_workload(4, 512, 512, 16, "nvfp4", "bf16", n_out=2, factor=10.0, seed=1)
    pp = G.prepare(wl)
    blob = torch.from_numpy(pp.blob).cuda()
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    x = torch.empty((0, 512), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((0, 512), dtype=torch.bfloat16, device="cuda")
    sv.linear(pp.p, blob, x, 0, y, ws)
    assert sv.get_status() == sv.OK


def test_bounded_wait_reports_timeout_and_context_survives(gpu):
    """A wait that nothing completes gives up after its limit, the status word
    reports SVDQ_ERR_TIMEOUT once, and the next layer call still matches the
    oracle (no fault, no hang)."""
    import torch
    assert sv.get_status() == sv.OK
    sv.probe_timeout(50_000_000)            # 50 ms
    torch.cuda.synchronize()
    assert sv.get_status() == sv.ERR_TIMEOUT
    assert sv.get_status() == sv.OK         # read and cleared
    wl = synth.custom_workload(33, 512, 512, 16, "nvfp4", "bf16", n_out=2, factor=20.0, seed=8)
    pp = G.prepare(wl)
    G.compare(pp, wl.X, G.run_gpu(pp, wl.X))


@pytest.mark.parametrize("M,K,N,rank,dtype", [
    (2, 4096, 512, 0, "bf16"),      # K split over 8 CTA pairs, no low-rank branch
    (6, 4096, 512, 32, "fp16"),     # three low-rank segments
    (8, 2048, 1024, 32, "bf16"),
    (3, 4096, 9728, 16, "bf16"),    # 38 output tiles: just past the K-split limit
])
def test_few_token_path(gpu, M, K, N, rank, dtype):
    """A handful of tokens (the decode-like VAR steps): codes bit-exact, Y
    against the oracle, and two calls give identical bits (K-split partials
    are added in K order)."""
    wl = synth.custom_workload(M, K, N, rank, "nvfp4", dtype, n_out=6, factor=60.0, seed=90 + M)
    pp = G.prepare(wl)
    a = G.run_gpu(pp, wl.X)
    b = G.run_gpu(pp, wl.X)
    G.compare(pp, wl.X, a)
    assert np.array_equal(a.Y, b.Y)


@pytest.mark.parametrize("fmt,dtype,M", [("nvfp4", "bf16", 300), ("int4", "fp16", 96), ("nvfp4", "bf16", 3)])
def test_lora_appended_layer(gpu, fmt, dtype, M):
    """A layer with a LoRA adapter appended by svdq_append_lora (no
    re-quantisation) against the oracle's appended layer."""
    from oracle import svdquant as sq
    wl = synth.custom_workload(M, 1024, 512, 32, fmt, dtype, n_out=4, factor=40.0, seed=61)
    pp = G.prepare(wl)
    A, B = synth.make_lora(3, wl.K, wl.N, 32)
    q, blob2 = sv.append_lora(pp.p, pp.blob, A, B)
    pp2 = G.Prepared(wl, q, blob2, pp.sigma, sq.append_lora(pp.ref, A, B), pp.x64)
    G.compare(pp2, wl.X, G.run_gpu(pp2, wl.X))


@pytest.mark.parametrize("fmt,dtype", [("nvfp4", "bf16"), ("int4", "fp16")])
def test_column_shards_reassemble_the_layer(gpu, fmt, dtype):
    """Column shards (one per GPU in column-parallel use) each match the
    oracle's shard, and side by side they are the full layer's output, bit
    for bit (same tiles, same K order)."""
    from oracle import svdquant as sq
    wl = synth.custom_workload(300, 1024, 1024, 32, fmt, dtype, n_out=4, factor=40.0, seed=71)
    pp = G.prepare(wl)
    full = G.run_gpu(pp, wl.X)
    parts = []
    for n0, n1 in ((0, 256), (256, 768), (768, 1024)):
        q, b = sv.shard_columns(pp.p, pp.blob, n0, n1)
        pps = G.Prepared(wl, q, b, pp.sigma, sq.shard_columns(pp.ref, n0, n1), pp.x64)
        run = G.run_gpu(pps, wl.X)
        G.compare(pps, wl.X, run)
        parts.append(run.Y)
    assert np.array_equal(np.hstack(parts), full.Y)
