"""C-ABI library on the CPU: symbols, argument checks, blob integrity and the
host preparation against the oracle (no GPU calls)."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import rank_gemm_svdq_b200 as sv
import synth
from oracle import svdquant as sq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    txt = open(os.path.join(ROOT, "include", "svdq.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(svdq_[a-z_]+)\s*\(", txt)))


def test_library_exports_every_declared_function():
    names = header_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(sv.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(sv.EXPORTED)


def test_status_strings():
    for s in range(9):
        assert sv.status_string(s) and sv.status_string(s) != "unknown status"


@pytest.mark.parametrize("bad", [dict(K=100), dict(N=100), dict(rank=8), dict(rank=-16), dict(rank=256),
                                 dict(fmt="x"), dict(alpha=1.5), dict(K=384, fmt="nvfp4"), dict(K=384, fmt="int4")])
def test_invalid_params_rejected(bad):
    kw = dict(K=256, N=256, rank=16, fmt="int4", dtype="bf16", alpha=0.5)
    if bad.get("fmt") == "x":
        p = sv.params(256, 256, 16, "int4", "bf16"); p.fmt = 7
    else:
        kw.update(bad); p = sv.params(**kw)
    assert sv.blob_bytes(p) == 0
    Wt = np.zeros((max(p.N, 1), max(p.K, 1)), np.float32)
    blob = np.zeros(16, np.uint8)
    st = sv.lib().svdq_prepare(ctypes.byref(p), Wt.ctypes.data, None, None, 0, blob.ctypes.data, 16, None)
    assert st in (sv.ERR_INVALID_ARG, sv.ERR_UNSUPPORTED)


def test_prepare_rejects_small_blob_and_null():
    p = sv.params(256, 256, 16, "nvfp4", "bf16")
    Wt = np.ones((256, 256), np.float32)
    blob = np.zeros(sv.blob_bytes(p) - 1, np.uint8)
    assert sv.lib().svdq_prepare(ctypes.byref(p), Wt.ctypes.data, None, None, 0, blob.ctypes.data,
                                 blob.nbytes, None) == sv.ERR_INVALID_ARG
    blob = np.zeros(sv.blob_bytes(p), np.uint8)
    assert sv.lib().svdq_prepare(ctypes.byref(p), None, None, None, 0, blob.ctypes.data, blob.nbytes,
                                 None) == sv.ERR_INVALID_ARG


def test_blob_check_detects_corruption():
    wl = synth.custom_workload(64, 256, 256, 16, "nvfp4", "bf16", n_out=2, factor=30.0)
    p = sv.params(256, 256, 16, "nvfp4", "bf16")
    blob, _ = sv.prepare(p, wl.Wt, wl.bias, wl.X)
    assert sv.blob_check(p, blob) == sv.OK
    bad = blob.copy(); bad[5000] ^= 1
    assert sv.blob_check(p, bad) == sv.ERR_BLOB
    bad = blob.copy(); bad[0] ^= 1
    assert sv.blob_check(p, bad) == sv.ERR_BLOB
    q = sv.params(256, 256, 32, "nvfp4", "bf16")
    assert sv.blob_check(q, blob) == sv.ERR_BLOB


def test_workspace_bytes_grows_with_tokens():
    p = sv.params(3072, 12288, 32, "nvfp4", "bf16")
    a, b = sv.workspace_bytes(p, 1), sv.workspace_bytes(p, 4608)
    assert 0 < a < b
    assert b >= 4608 * 3072 // 2 + 4608 * 3072 // 16 + 4608 * 64 * 2


def _factors(p, c):
    dt = np.float16 if p.act_dtype == sv.F16 else None
    if dt is not None:
        L1 = c.L1.view(np.float16).astype(np.float64); L2 = c.L2.view(np.float16).astype(np.float64)
    else:
        L1 = synth.bf16_bits_to_f64(c.L1); L2 = synth.bf16_bits_to_f64(c.L2)
    return L1, L2


CASES = [
    ("int4", "fp16", 16, True), ("nvfp4", "fp16", 16, True),
    ("int4", "bf16", 32, True), ("nvfp4", "bf16", 32, True),
    ("nvfp4", "bf16", 0, True), ("int4", "bf16", 16, False),
]


@pytest.mark.parametrize("fmt,dtype,rank,smooth", CASES)
def test_prepare_matches_oracle(fmt, dtype, rank, smooth):
    """Weight codes/scales bit-exact against the oracle's quantisation of R
    recomputed from the library's stored lambda and factors; lambda and the
    tensor scales bit-exact; the truncated SVD within rounding of the
    Eckart-Young optimum the oracle's Jacobi SVD gives."""
    M, N = 96, 512
    K = 768 if fmt == "int4" else 512
    wl = synth.custom_workload(M, K, N, rank, fmt, dtype, n_out=3, factor=60.0, smooth=smooth, seed=3)
    p = sv.params(K, N, rank, fmt, dtype, smooth=smooth)
    blob, sigma = sv.prepare(p, wl.Wt, wl.bias, wl.X)
    c = sv.blob_export(p, blob)
    x = wl.x_f64()
    ref = sq.prepare(x, wl.Wt, wl.bias, rank, fmt, dtype, smooth=smooth)
    assert np.array_equal(c.inv_lambda.view(np.uint32), ref.inv_lambda.view(np.uint32))
    L1, L2 = _factors(p, c)
    po = sq.prepare(x, wl.Wt, wl.bias, rank, fmt, dtype, smooth=smooth, factors=(c.inv_lambda, L1, L2))
    assert np.array_equal(c.wcodes, po.wq.codes)
    assert np.array_equal(c.wscales.view(np.uint8), po.wq.scales.view(np.uint8))
    assert c.s_gw.view(np.uint32) == np.float32(po.wq.s_g).view(np.uint32)
    assert c.s_gx.view(np.uint32) == np.float32(po.s_gx).view(np.uint32)
    assert np.array_equal(c.bias, wl.bias)
    if rank > 0:
        W_hat = sq.smooth_weight(wl.Wt, ref.lam_eff)
        tail = math.sqrt(np.sum(ref.sigma[rank:] ** 2))
        err = np.linalg.norm(W_hat - L1 @ L2)
        assert err >= tail * (1 - 1e-9)
        assert err <= tail * 1.01 + 4 * 2.0 ** -8 * np.linalg.norm(L1 @ L2)
        assert np.allclose(sigma[:rank], ref.sigma[:rank], rtol=0.02)
        if smooth:
            # smoothing makes the 3 outlier channels dominant singular directions,
            # which subspace iteration resolves to high accuracy
            assert np.allclose(sigma[:3], ref.sigma[:3], rtol=1e-9)


def test_zero_weight_and_zero_calibration():
    K, N = 256, 256
    p = sv.params(K, N, 16, "nvfp4", "bf16")
    blob, sigma = sv.prepare(p, np.zeros((N, K), np.float32), None, None)
    c = sv.blob_export(p, blob)
    assert np.all(c.inv_lambda == 1.0) and np.all(c.wcodes == 0) and np.all(c.bias == 0)
    assert c.s_gx == 1.0 and c.s_gw == 1.0 and np.all(sigma == 0)


def test_kv_codec_argument_checks_need_no_gpu():
    """svdq_kv_encode / svdq_kv_decode reject bad shapes, dtypes, workspaces
    and misaligned pointers before touching a device (the pointers below are
    never dereferenced)."""
    L = sv.lib()
    A = 1 << 20                                # a 16-byte aligned fake address
    assert L.svdq_kv_workspace_bytes(0, 256) == 0
    assert L.svdq_kv_workspace_bytes(257, 512) == 2 * 2 * 512 * 4
    ws = L.svdq_kv_workspace_bytes(300, 512)
    enc = lambda X, T, C, dt, q, s, z, w, wb: L.svdq_kv_encode(X, T, C, dt, q, s, z, w, wb, None)
    assert enc(A, 0, 512, sv.BF16, A, A, A, A, ws) == sv.ERR_INVALID_ARG        # no tokens
    assert enc(A, 300, 320, sv.BF16, A, A, A, A, ws) == sv.ERR_INVALID_ARG      # C % 256
    assert enc(A, 300, 512, 9, A, A, A, A, ws) == sv.ERR_INVALID_ARG            # dtype
    assert enc(None, 300, 512, sv.BF16, A, A, A, A, ws) == sv.ERR_INVALID_ARG   # null
    assert enc(A, 300, 512, sv.BF16, A, A, A, A, ws - 1) == sv.ERR_WORKSPACE
    assert enc(A + 2, 300, 512, sv.BF16, A, A, A, A, ws) == sv.ERR_ALIGNMENT
    dec = lambda q, s, z, T, C, dt, Y: L.svdq_kv_decode(q, s, z, T, C, dt, Y, None)
    assert dec(A, A, A, 10, 12, sv.BF16, A) == sv.ERR_INVALID_ARG               # C % 8
    assert dec(A, A, A, 10, 64, sv.F16, A + 8) == sv.ERR_ALIGNMENT
