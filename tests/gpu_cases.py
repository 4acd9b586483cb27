"""Shared machinery of the GPU parity tests: prepare a layer with the library,
re-derive the oracle's layer from the library's stored factors, run
svdq_linear through the C ABI and compare."""
from __future__ import annotations

import functools
from dataclasses import dataclass

import numpy as np

import rank_gemm_svdq_b200 as sv
import synth
from oracle import formats, svdquant as sq

Y_TOL = 1e-3       # ||Y_gpu - bf16(Y_oracle)||_F / ||bf16(Y_oracle)||_F
U_TOL = 2e-5       # relative error of the down projection u (fp32 accumulate, bf16 hi+lo)
CANARY = 0x5A


def factors_f64(p, c):
    if p.act_dtype == sv.F16:
        return c.L1.view(np.float16).astype(np.float64), c.L2.view(np.float16).astype(np.float64)
    return synth.bf16_bits_to_f64(c.L1), synth.bf16_bits_to_f64(c.L2)


@dataclass
class Prepared:
    wl: synth.Workload
    p: object
    blob: np.ndarray
    sigma: np.ndarray
    ref: object          # oracle layer built from the library's lambda and factors
    x64: np.ndarray


def prepare(wl: synth.Workload) -> Prepared:
    p = sv.params(wl.K, wl.N, wl.rank, wl.fmt, wl.dtype, wl.alpha, wl.smooth)
    blob, sigma = sv.prepare(p, wl.Wt, wl.bias, wl.X)
    c = sv.blob_export(p, blob)
    L1, L2 = factors_f64(p, c)
    x64 = wl.x_f64()
    ref = sq.prepare(x64, wl.Wt, wl.bias, wl.rank, wl.fmt, wl.dtype, wl.alpha, wl.smooth,
                     factors=(c.inv_lambda, L1, L2))
    assert np.array_equal(c.wcodes, ref.wq.codes), "weight codes differ from the oracle"
    assert np.array_equal(c.wscales.view(np.uint8), ref.wq.scales.view(np.uint8)), "weight scales differ"
    return Prepared(wl, p, blob, sigma, ref, x64)


@functools.lru_cache(maxsize=4)
def prepared_preset(name: str) -> Prepared:
    return prepare(synth.make_workload(name))


def to_device_x(X: np.ndarray, dtype: str):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).cuda()
    return t.view(torch.bfloat16 if dtype == "bf16" else torch.float16)


@dataclass
class Run:
    Y: np.ndarray        # M x N float64 (bf16 values)
    codes: np.ndarray
    scales: np.ndarray
    u: np.ndarray        # M x r, u as the oracle defines it (tensor scales undone)


def run_gpu(pp: Prepared, X: np.ndarray, check_canaries: bool = True) -> Run:
    import torch
    p = pp.p
    M = X.shape[0]
    xd = to_device_x(X, pp.wl.dtype)
    blob = torch.from_numpy(pp.blob).cuda()
    # output with one guard row above and below; workspace with a guard tail
    ybuf = torch.full((M + 2, p.N), -7.0, dtype=torch.bfloat16, device="cuda")
    y = ybuf[1:M + 1]
    wsz = sv.workspace_bytes(p, M)
    wbuf = torch.full((wsz + 4096,), CANARY, dtype=torch.uint8, device="cuda")
    ws = wbuf[:wsz]
    sv.linear(p, blob, xd, M, y, ws)
    st = sv.get_status()
    assert st == sv.OK, sv.status_string(st)
    torch.cuda.synchronize()
    if check_canaries:
        assert torch.all(ybuf[0] == -7.0) and torch.all(ybuf[M + 1] == -7.0), "write outside Y"
        assert torch.all(wbuf[wsz:] == CANARY), "write outside the workspace"
    codes, scales, u = sv.export_act(p, ws, M)
    Y = y.float().cpu().numpy().astype(np.float64)
    u = u.astype(np.float64)
    if p.fmt == sv.NVFP4:
        c = sv.blob_export(p, pp.blob)
        u = u * (float(c.s_gx) * float(c.s_gw))
    return Run(Y, codes, scales, u)


def compare(pp: Prepared, X: np.ndarray, run: Run, rows=None, code_rows=None) -> dict:
    """Bit-exact codes/scales on `code_rows`, Y within Y_TOL on `rows`."""
    M = X.shape[0]
    rows = np.arange(M) if rows is None else np.asarray(rows)
    code_rows = rows if code_rows is None else np.asarray(code_rows)
    x64 = synth.dtype_to_f64(X, pp.wl.dtype)
    a = sq.quantize_act(x64[code_rows], pp.ref)
    gc = run.codes[code_rows]
    assert np.array_equal(gc.view(np.uint8), a.codes.view(np.uint8)), \
        f"activation codes differ at {np.argwhere(gc.view(np.uint8) != a.codes.view(np.uint8))[:5]}"
    gs = run.scales[code_rows]
    assert np.array_equal(gs.view(np.uint8), a.scales.view(np.uint8)), \
        f"activation scales differ at {np.argwhere(gs.view(np.uint8) != a.scales.view(np.uint8))[:5]}"
    out = {}
    if pp.p.rank > 0:
        uerr = np.linalg.norm(run.u[code_rows] - a.u) / max(np.linalg.norm(a.u), 1e-300)
        assert uerr <= U_TOL, f"u rel err {uerr}"
        out["u_rel_err"] = float(uerr)
    Yref = formats.to_bf16(sq.forward(x64[rows], pp.ref))
    err = sq.rel_fro(run.Y[rows], Yref)
    out["y_rel_err"] = err
    assert err <= Y_TOL, f"Y rel err {err}"
    if len(rows) == M:
        # every output tile on its own: a wrong tile cannot hide in the global norm
        worst, where = tile_errors(run.Y, Yref)
        out["y_worst_tile_rel_err"] = worst
        out["y_worst_tile"] = where
        assert worst <= Y_TOL, f"Y rel err {worst} in the {TILE_M}x{TILE_N} tile at {where}"
    return out


TILE_M, TILE_N = 128, 256


def tile_errors(Y: np.ndarray, Yref: np.ndarray):
    """Largest relative Frobenius error over the (TILE_M x TILE_N) output
    tiles (ragged at the edges), and that tile's (row, column) origin."""
    worst, where = 0.0, (0, 0)
    for r0 in range(0, Y.shape[0], TILE_M):
        for c0 in range(0, Y.shape[1], TILE_N):
            a = Y[r0:r0 + TILE_M, c0:c0 + TILE_N]
            b = Yref[r0:r0 + TILE_M, c0:c0 + TILE_N]
            nb = np.linalg.norm(b)
            e = float(np.linalg.norm(a - b) / nb) if nb > 0 else float(np.linalg.norm(a - b))
            if e > worst:
                worst, where = e, (r0, c0)
    return worst, where
