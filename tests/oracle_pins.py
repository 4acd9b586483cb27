"""Pins of the CPU oracle: checks against what the pages and the mathematics fix.

Every pin takes the oracle modules it checks as arguments, so the mutation
test can hand it an oracle with a planted mistake and see it fail.  None of
them re-derives a value by calling the code path it checks: expected values
come from format standards, exact rational arithmetic (fractions), LAPACK,
closed forms, invariants and brute force over small code tables.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ------------------------------------------------------------------ formats
def pin_format_tables(formats):
    """Code tables equal the OCP standard values (golden file)."""
    with open(os.path.join(GOLDEN, "formats_ocp.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            fmt, code, value = line.split()
            code = int(code, 16)
            dec = formats.e2m1_decode if fmt == "e2m1" else formats.e4m3_decode
            got = float(dec(np.array([code]))[0])
            assert got == float(value), (fmt, hex(code), got, value)
    assert math.isnan(formats.e4m3_decode(np.array([0x7F]))[0])
    assert formats.E2M1_MAX == 6.0 and formats.E4M3_MAX == 448.0


def _bruteforce_encode(x, table, max_code, sign_bit):
    """Nearest code by exhaustive search; ties -> code with mantissa LSB 0;
    beyond the largest finite value -> the largest finite value."""
    vals = table[: max_code + 1]
    out = np.empty(len(x), dtype=np.int64)
    for i, v in enumerate(x):
        a = abs(v)
        if a >= vals[-1]:
            c = max_code
        else:
            d = np.abs(vals - a)
            best = np.flatnonzero(d == d.min())
            c = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
        out[i] = c | (sign_bit if math.copysign(1.0, v) < 0 else 0)
    return out


def pin_encoders_bruteforce(formats, n=4000, seed=11):
    rng = np.random.default_rng(seed)
    for table, enc, max_code, sb, top in ((formats.E2M1_VALUES, formats.e2m1_encode, 7, 0x8, 6.0),
                                          (formats.E4M3_VALUES, formats.e4m3_encode, 0x7E, 0x80, 448.0)):
        mags = table[: max_code + 1]
        mids = 0.5 * (mags[:-1] + mags[1:])
        f32 = np.float32
        # every midpoint, one fp32 ulp either side, random values over the range and beyond
        pts = np.concatenate([mids,
                              np.nextafter(mids.astype(f32), f32(np.inf)).astype(np.float64),
                              np.nextafter(mids.astype(f32), f32(0)).astype(np.float64),
                              mags, rng.uniform(0, top * 1.3, n),
                              np.exp(rng.uniform(np.log(1e-4), np.log(top), n)),
                              [top * 2, top * 1e6, 0.0]])
        pts = np.concatenate([pts, -pts])
        got = enc(pts).astype(np.int64)
        exp = _bruteforce_encode(pts, table, max_code, sb)
        bad = np.flatnonzero(got != exp)
        assert len(bad) == 0, (pts[bad[:5]], got[bad[:5]], exp[bad[:5]])


def pin_fp16_rounding(formats, n=20000, seed=3):
    """float64 -> fp16 RNE equals numpy's float16 conversion (library routine)."""
    rng = np.random.default_rng(seed)
    x = np.concatenate([rng.standard_normal(n) * 10.0 ** rng.uniform(-9, 4, n),
                        np.ldexp(1.0 + np.arange(1, 64) * 2.0 ** -11 + 2.0 ** -12, 0)])
    x = x[np.abs(x) < 65000]
    assert np.array_equal(formats.to_fp16(x), x.astype(np.float16).astype(np.float64))


def pin_bf16_rounding(formats, n=20000, seed=4):
    """float64 -> bf16 RNE equals exact rational rounding."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(n) * 10.0 ** rng.uniform(-30, 30, n)
    # exact ties and near-ties built from bf16 neighbours
    base = np.ldexp(1.0 + rng.integers(0, 128, 200) / 128.0, rng.integers(-20, 20, 200))
    x = np.concatenate([x, base * (1 + 2.0 ** -8), base * (1 + 2.0 ** -8 + 2.0 ** -40),
                        base * (1 + 3 * 2.0 ** -8)])
    got = formats.to_bf16(x)
    for v, g in zip(x[:3000:7].tolist() + x[n:].tolist(), np.concatenate([got[:3000:7], got[n:]]).tolist()):
        fv = Fraction(v)
        e = math.frexp(abs(v))[1] - 1
        q = Fraction(2) ** (e - 7)
        k = fv / q
        lo = math.floor(k)
        r = k - lo
        kk = lo + 1 if (r > Fraction(1, 2) or (r == Fraction(1, 2) and lo % 2 == 1)) else lo
        assert Fraction(g) == kk * q, (v, g, float(kk * q))


# ------------------------------------------------------------------ quantisers
def pin_int4_golden(quant):
    """The W4A8 page's symmetric quantiser, worked by hand (golden file)."""
    with open(os.path.join(GOLDEN, "int4_quantizer_w4a8_page.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            vals, scale, codes = [p.split() for p in line.split("|")]
            v = np.array([[float(t) for t in vals]], dtype=np.float32)
            q, s = quant.int4_group_quant(v, group=v.shape[1])
            assert s[0, 0] == np.float32(float(scale[0])), (vals, s)
            assert q[0].tolist() == [int(t) for t in codes], (vals, q)


def pin_int4_bruteforce(quant, seed=5):
    """Each INT4 code is the nearest of -8..7 to fl32(v / s) (ties to even) and
    the dequantised value is within half a step of v."""
    rng = np.random.default_rng(seed)
    v = (rng.standard_normal((16, 256)) * rng.uniform(0.01, 50, (16, 1))).astype(np.float32)
    v[3, 64:128] = 0.0
    v[5, :64] = np.float32(2.5) * np.arange(-32, 32) / 7          # near-ties
    q, s = quant.int4_group_quant(v, 64)
    grid = np.arange(-8, 8)
    for r in range(v.shape[0]):
        for k in range(v.shape[1]):
            sc = s[r, k // 64]
            if sc == 0:
                assert q[r, k] == 0
                continue
            t = float(np.float32(v[r, k]) / np.float32(sc))
            d = np.abs(grid - t)
            best = grid[d == d.min()]
            exp = best[0] if len(best) == 1 else best[best % 2 == 0][0]
            assert q[r, k] == exp, (r, k, t, q[r, k], exp)
            assert abs(float(v[r, k]) - float(sc) * int(q[r, k])) <= 0.5 * float(sc) * (1 + 2 ** -20)
        # scale = group absmax / 7
        for g in range(4):
            m = np.abs(v[r, g * 64:(g + 1) * 64]).max()
            assert s[r, g] == np.float32(m) / np.float32(7)


def pin_nvfp4_bounds(quant, formats, seed=6):
    """NVFP4: block scale = E4M3(block amax / (6 s_g)), element error within half
    the local E2M1 spacing of the block step (or the saturation excess)."""
    rng = np.random.default_rng(seed)
    v = (rng.standard_normal((8, 512)) * np.exp(rng.uniform(-4, 4, (8, 1)))).astype(np.float32)
    v[2, 16:32] = 0
    v[4, :16] *= 1e-6                                   # tiny block -> tiny / zero scale
    s_g = quant.nvfp4_tensor_scale(float(np.abs(v).max()))
    assert s_g == np.float32(np.float32(np.abs(v).max()) / np.float32(2688.0))
    c, e = quant.nvfp4_quant(v, s_g)
    vals = formats.E2M1_VALUES[:8]
    for r in range(v.shape[0]):
        for b in range(v.shape[1] // 16):
            blk = v[r, b * 16:(b + 1) * 16].astype(np.float64)
            ev = float(formats.e4m3_decode(np.array([e[r, b]]))[0])
            ratio = float(np.float32(np.float32(np.abs(blk).max()) / np.float32(np.float32(6) * s_g)))
            # scale code is the nearest E4M3 value to the ratio (relative 2^-4 for normals)
            assert ev <= 448.0
            if ratio >= 2.0 ** -6:
                assert abs(ev - ratio) <= ratio * 2.0 ** -4 + 1e-300
            else:
                assert abs(ev - ratio) <= 2.0 ** -10
            d = float(np.float32(np.float32(ev) * s_g))
            for j in range(16):
                qv = float(formats.e2m1_decode(np.array([c[r, b * 16 + j]]))[0])
                x = blk[j]
                if d == 0:
                    assert c[r, b * 16 + j] == 0
                    continue
                a = abs(x) / d
                if a >= 6.0:
                    assert abs(qv) == 6.0
                    assert abs(x - qv * d) <= (a - 6.0) * d + 1e-12 * abs(x)
                else:
                    i = int(np.searchsorted(vals, a, side="right")) - 1
                    i = min(max(i, 0), 6)
                    half = 0.5 * (vals[i + 1] - vals[i])
                    assert abs(abs(x) - abs(qv) * d) <= half * d * (1 + 2.0 ** -20), (x, qv, d)
                    assert qv == 0 or math.copysign(1, qv) == math.copysign(1, x)


# ------------------------------------------------------------------ SVD
def pin_svd_known_answers(svd):
    rng = np.random.default_rng(7)
    # diagonal
    d = np.array([3.0, -7.0, 0.5, 2.0])
    U, s, Vt = svd.jacobi_svd(np.diag(d))
    assert np.allclose(s, [7.0, 3.0, 2.0, 0.5], rtol=0, atol=1e-15)
    # rank one: c u v^T has one singular value c |u| |v|
    u = rng.standard_normal(9); v = rng.standard_normal(5)
    U, s, Vt = svd.jacobi_svd(2.5 * np.outer(u, v))
    assert abs(s[0] - 2.5 * np.linalg.norm(u) * np.linalg.norm(v)) <= 1e-13 * s[0]
    assert np.all(s[1:] <= 1e-13 * s[0])
    # Householder . diag . Householder: singular values are |diag|
    def house(n):
        w = rng.standard_normal(n); w /= np.linalg.norm(w)
        return np.eye(n) - 2 * np.outer(w, w)
    sig = np.array([10.0, 4.0, 4.0 - 1e-3, 1.0, 1e-3, 0.0])
    A = house(8)[:, :6] @ np.diag(sig) @ house(6)
    U, s, Vt = svd.jacobi_svd(A)
    assert np.allclose(s, sig, rtol=0, atol=1e-13)


def pin_svd_vs_lapack(svd, shapes=((40, 60), (96, 64), (128, 128))):
    rng = np.random.default_rng(8)
    for m, n in shapes:
        A = rng.standard_normal((m, n)) * np.exp(rng.uniform(-3, 3, (1, n)))
        U, s, Vt = svd.jacobi_svd(A)
        s_ref = np.linalg.svd(A, compute_uv=False)
        assert np.max(np.abs(s - s_ref)) <= 1e-10 * s_ref[0]
        p = min(m, n)
        assert np.max(np.abs(U.T @ U - np.eye(p))) <= 1e-12
        assert np.max(np.abs(Vt @ Vt.T - np.eye(p))) <= 1e-12
        assert np.max(np.abs(U @ np.diag(s) @ Vt - A)) <= 1e-12 * s[0]


def pin_eckart_young(svd, sq):
    """||W^ - U_r S_r V_r^T||_F^2 = sum_{i>r} s_i^2 (Eckart-Young-Mirsky, the
    theorem the SVDQuant page cites), and the oracle's residual from rounded
    factors stays within rounding of that optimum (and never below it)."""
    rng = np.random.default_rng(9)
    K, N, r = 96, 80, 8
    Wt = (rng.standard_normal((N, K)) / math.sqrt(K)).astype(np.float32)
    x = rng.standard_normal((64, K)); x[:, [3, 17, 50]] *= 80
    inv_l, lam = sq.smoothing_factors(x, Wt, 0.5)
    W_hat = sq.smooth_weight(Wt, lam)
    U, s, Vt = svd.jacobi_svd(W_hat)
    for rr in (0, 1, r, 20):
        E = W_hat - U[:, :rr] @ np.diag(s[:rr]) @ Vt[:rr]
        assert abs(np.sum(E * E) - np.sum(s[rr:] ** 2)) <= 1e-10 * np.sum(s ** 2)
    L1, L2, sig = sq.low_rank_factors(W_hat, r, "bf16")
    R = sq.residual(W_hat, L1, L2).astype(np.float64)
    tail = math.sqrt(np.sum(s[r:] ** 2))
    nR = np.linalg.norm(R)
    assert nR >= tail * (1 - 1e-6)
    assert nR <= tail + 2 * 2.0 ** -8 * np.linalg.norm(L1 @ L2) + 1e-6 * tail
    # R is W^ minus the product of the stored factors (not of unrounded ones)
    assert np.max(np.abs(R - (W_hat - L1 @ L2))) <= 1e-6 * np.max(np.abs(W_hat))


# ------------------------------------------------------------------ the method
def pin_smoothing(sq):
    """X^ W^ = X W without quantisation; at alpha = 0.5 the smoothed activation
    and weight ranges of every channel are equal (the balance the smoothing
    rule is built for); at alpha = 1 every activation channel range is 1."""
    rng = np.random.default_rng(10)
    M, K, N = 32, 64, 48
    x = rng.standard_normal((M, K)); x[:, [2, 40]] *= 100
    Wt = rng.standard_normal((N, K)).astype(np.float32)
    inv_l, lam = sq.smoothing_factors(x, Wt, 0.5)
    W_hat = sq.smooth_weight(Wt, lam)
    X_hat = x / lam[None, :]
    ref = x @ Wt.astype(np.float64).T
    assert np.max(np.abs(X_hat @ W_hat - ref)) <= 1e-12 * np.max(np.abs(ref))
    a = np.abs(X_hat).max(axis=0)
    w = np.abs(W_hat).max(axis=1)
    assert np.allclose(a, w, rtol=1e-6)
    inv_l1, lam1 = sq.smoothing_factors(x, Wt, 1.0)
    assert np.allclose(np.abs(x / lam1[None, :]).max(axis=0), 1.0, rtol=1e-6)
    inv_l0, lam0 = sq.smoothing_factors(x, Wt, 0.5, smooth=False)
    assert np.all(lam0 == 1.0)


def pin_rank0_plain_rtn(sq):
    """Rank 0 without smoothing is plain symmetric W4A4 round-to-nearest with
    groups along K (the Min-Max baseline of the VAR-Compressor page), computed
    here by a naive element loop."""
    rng = np.random.default_rng(12)
    M, K, N, g = 3, 16, 4, 8
    x = rng.standard_normal((M, K)).astype(np.float16).astype(np.float64)
    Wt = rng.standard_normal((N, K)).astype(np.float32)
    b = rng.standard_normal(N).astype(np.float32)
    p = sq.prepare(x, Wt, b, 0, "int4", "fp16", smooth=False, group=g)
    Y = sq.forward(x, p, group=g)

    def rtn(row):
        q, s = [], []
        for j in range(0, len(row), g):
            grp = [np.float32(t) for t in row[j:j + g]]
            m = max(abs(t) for t in grp)
            sc = np.float32(m) / np.float32(7.0)
            s.append(float(sc))
            for t in grp:
                q.append(0 if m == 0 else max(-8, min(7, round(float(np.float32(t) / sc)))))
        return q, s

    for m in range(M):
        qx, sx = rtn(x[m])
        for n in range(N):
            qw, sw = rtn(Wt[n])
            y = 0.0
            for j in range(K // g):
                dot = sum(qx[j * g + t] * qw[j * g + t] for t in range(g))
                y += sx[j] * sw[j] * dot
            y += float(b[n])
            assert abs(Y[m, n] - y) <= 1e-12 * (abs(y) + 1), (m, n, Y[m, n], y)


def _exact_tiny(sq, fmt, M, K, N, r, g, seed):
    """Y by exact rational arithmetic from the oracle's codes and scales:
    dequantise every element, naive triple loop, exact low-rank term from an
    independently rounded X^16 (numpy float16) and the stored factors."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)); x[:, 1] *= 30
    x = x.astype(np.float16).astype(np.float64)
    Wt = rng.standard_normal((N, K)).astype(np.float32)
    b = rng.standard_normal(N).astype(np.float32)
    p = sq.prepare(x, Wt, b, r, fmt, "fp16", group=g)
    Y, a, _, _ = sq.forward(x, p, group=g, return_parts=True)
    from oracle import formats
    if fmt == "int4":
        dx = [[Fraction(float(a.scales[m, k // g])) * int(a.codes[m, k]) for k in range(K)] for m in range(M)]
        dw = [[Fraction(float(p.wq.scales[n, k // g])) * int(p.wq.codes[n, k]) for k in range(K)] for n in range(N)]
    else:
        sgx, sgw = Fraction(float(p.s_gx)), Fraction(float(p.wq.s_g))
        dx = [[sgx * Fraction(float(formats.E4M3_VALUES[a.scales[m, k // 16]]))
               * Fraction(float(formats.E2M1_VALUES[a.codes[m, k]])) for k in range(K)] for m in range(M)]
        dw = [[sgw * Fraction(float(formats.E4M3_VALUES[p.wq.scales[n, k // 16]]))
               * Fraction(float(formats.E2M1_VALUES[p.wq.codes[n, k]])) for k in range(K)] for n in range(N)]
    xh = (x.astype(np.float32) * p.inv_lambda).astype(np.float32)
    x16 = xh.astype(np.float16)
    for m in range(M):
        u = [sum(Fraction(float(x16[m, k])) * Fraction(float(p.L1[k, i])) for k in range(K)) for i in range(r)]
        for n in range(N):
            y = sum(dx[m][k] * dw[n][k] for k in range(K))
            y += sum(u[i] * Fraction(float(p.L2[i, n])) for i in range(r))
            y += Fraction(float(b[n]))
            assert abs(Y[m, n] - float(y)) <= 1e-12 * (abs(float(y)) + 1), (fmt, m, n, Y[m, n], float(y))
    # the weight codes quantise W^ - L1 L2 computed exactly, up to the fp32 rounding of R
    W_hat = [[Fraction(float(Wt[n, k])) * Fraction(float(p.lam_eff[k])) for n in range(N)] for k in range(K)]
    for k in range(K):
        for n in range(N):
            rr = W_hat[k][n] - sum(Fraction(float(p.L1[k, i])) * Fraction(float(p.L2[i, n])) for i in range(r))
            assert abs(float(p.R[k, n]) - float(rr)) <= 2.0 ** -23 * abs(float(rr)) + 1e-30
    return p


def pin_bruteforce_int4(sq):
    _exact_tiny(sq, "int4", 4, 8, 8, 2, 8, 13)


def pin_bruteforce_nvfp4(sq):
    _exact_tiny(sq, "nvfp4", 4, 16, 8, 2, 16, 14)


def pin_special_cases(sq):
    """X = 0 -> Y = b;  W = 0 -> Y = b  (both formats, with a rank-r branch)."""
    rng = np.random.default_rng(15)
    M, K, N = 4, 128, 64
    b = rng.standard_normal(N).astype(np.float32)
    Wt = rng.standard_normal((N, K)).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float16).astype(np.float64)
    for fmt in ("int4", "nvfp4"):
        p = sq.prepare(np.zeros((M, K)), Wt, b, 4, fmt, "fp16")
        assert np.array_equal(sq.forward(np.zeros((M, K)), p), np.broadcast_to(b.astype(np.float64), (M, N)))
        p = sq.prepare(x, np.zeros((N, K), np.float32), b, 4, fmt, "fp16")
        assert np.array_equal(sq.forward(x, p), np.broadcast_to(b.astype(np.float64), (M, N)))


def pin_on_grid_lossless(sq):
    """Inputs already on the quantisation grid pass through unchanged, so with
    rank 0 and no smoothing Y = X W + b up to float64 rounding."""
    rng = np.random.default_rng(16)
    M, K, N = 4, 128, 32
    # INT4: each group of 64 holds k * 2^e, k in -7..7, with +-7 * 2^e present
    def int4_grid(rows):
        v = rng.integers(-7, 8, (rows, K)).astype(np.float64)
        v[:, ::64] = 7 * np.where(rng.random((rows, K // 64)) < 0.5, -1, 1)
        e = rng.integers(-3, 3, (rows, K // 64)).astype(np.float64)
        return v * np.repeat(2.0 ** e, 64, axis=1)
    x = int4_grid(M); Wt = int4_grid(N).astype(np.float32)
    b = rng.standard_normal(N).astype(np.float32)
    p = sq.prepare(x, Wt, b, 0, "int4", "fp16", smooth=False)
    ref = x @ Wt.astype(np.float64).T + b.astype(np.float64)
    assert np.max(np.abs(sq.forward(x, p) - ref)) <= 1e-13 * np.max(np.abs(ref))
    # NVFP4: tensor amax 2688 * 2^t, block amax 6 * E4M3 value * 2^t, elements on the E2M1 grid
    from oracle import formats
    def fp4_grid(rows, t):
        q = formats.E2M1_VALUES[rng.integers(0, 16, (rows, K))]
        q[:, ::16] = 6.0 * np.where(rng.random((rows, K // 16)) < 0.5, -1, 1)
        ev = formats.E4M3_VALUES[rng.integers(0x20, 0x7E, (rows, K // 16))]
        ev[0, 0] = 448.0
        return q * np.repeat(ev, 16, axis=1) * 2.0 ** t
    x = fp4_grid(M, -8); Wt = fp4_grid(N, -10).astype(np.float32)
    p = sq.prepare(x, Wt, b, 0, "nvfp4", "bf16", smooth=False)
    ref = x @ Wt.astype(np.float64).T + b.astype(np.float64)
    assert np.max(np.abs(sq.forward(x, p) - ref)) <= 1e-13 * np.max(np.abs(ref))


def pin_low_rank_helps(sq):
    """The pages' qualitative claim: with outlier channels, the rank-r branch
    lowers the layer error against the unquantised X W + b."""
    rng = np.random.default_rng(17)
    M, K, N = 64, 256, 128
    x = rng.standard_normal((M, K)); x[:, [5, 77, 200]] *= 100
    x = x.astype(np.float16).astype(np.float64)
    Wt = (rng.standard_normal((N, K)) / math.sqrt(K)).astype(np.float32)
    b = rng.standard_normal(N).astype(np.float32)
    ref = sq.exact_output(x, Wt, b)
    for fmt in ("int4", "nvfp4"):
        e0 = sq.rel_fro(sq.forward(x, sq.prepare(x, Wt, b, 0, fmt, "fp16", smooth=False)), ref)
        er = sq.rel_fro(sq.forward(x, sq.prepare(x, Wt, b, 16, fmt, "fp16")), ref)
        assert er < e0, (fmt, er, e0)


# ------------------------------------------------------------------ activation side
def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                yield [part.strip() for part in line.split("|")]


def pin_act_tensor_scale_golden(sq):
    """The static NVFP4 activation tensor scale is amax of the SMOOTHED
    calibration activations over 2688, bit for bit on hand-worked cases
    (golden file: the amax of X and of X^ sit in different places)."""
    for rows, inv, bits in _golden_lines("act_tensor_scale.txt"):
        x_cal = np.array([[float(t) for t in r.split()] for r in rows.split(";")])
        inv_l = np.array([float(t) for t in inv.split()], dtype=np.float32)
        s = sq.act_tensor_scale(x_cal, inv_l)
        assert np.float32(s).view(np.uint32) == np.uint32(int(bits, 16)), (rows, float(s), bits)


def _bare_layer(sq, fmt, inv_l, s_gx):
    """A rank-0 layer holding only what the activation side reads."""
    K = len(inv_l)
    return sq.Prepared(fmt, "fp16", 0, inv_l, 1.0 / inv_l.astype(np.float64), np.zeros((K, 0)),
                       np.zeros((0, 1)), None, None, None, np.float32(s_gx), np.zeros(1, np.float32))


def pin_act_codes_golden(sq):
    """Per-token activation codes and scales of quantize_act are those of
    X^ = fl32(x) * inv_lambda (hand-worked golden file: ties to even, signed
    zero, the block scale from the smoothed block amax)."""
    for fmt, sg, inv, xs, scale, codes in _golden_lines("act_codes_smoothed.txt"):
        inv_l = np.array([float(t) for t in inv.split()], dtype=np.float32)
        x = np.array([[float(t) for t in xs.split()]])
        a = sq.quantize_act(x, _bare_layer(sq, fmt, inv_l, float(sg)), group=64)
        if fmt == "nvfp4":
            assert a.scales.ravel().tolist() == [int(t, 16) for t in scale.split()], (a.scales, scale)
            assert a.codes.ravel().tolist() == [int(t, 16) for t in codes.split()], a.codes
        else:
            assert a.scales.ravel().tolist() == [float(t) for t in scale.split()], (a.scales, scale)
            assert a.codes.ravel().tolist() == [int(t) for t in codes.split()], a.codes


def pin_act_scale_in_prepare(sq):
    """prepare() takes s_gX from the calibration activations after smoothing:
    recomputed here with plain loops over every element on a layer with
    outlier channels (where amax(X) and amax(X^) differ by far)."""
    rng = np.random.default_rng(18)
    M, K, N = 24, 64, 32
    x = rng.standard_normal((M, K)); x[:, [4, 33]] *= 60
    x = x.astype(np.float16).astype(np.float64)
    Wt = (rng.standard_normal((N, K)) / 8).astype(np.float32)
    p = sq.prepare(x, Wt, None, 0, "nvfp4", "fp16")
    amax = 0.0
    for m in range(M):
        for j in range(K):
            v = abs(float(np.float32(np.float32(x[m, j]) * p.inv_lambda[j])))
            amax = v if v > amax else amax
    assert amax < 0.5 * float(np.abs(x).max())        # the smoothing really moved the range
    expect = Fraction(amax) / 2688
    got = Fraction(float(p.s_gx))
    # fl32 of the exact quotient: within half an fp32 ulp of it
    ulp = Fraction(2) ** (math.frexp(float(expect))[1] - 24)
    assert abs(got - expect) <= ulp / 2, (float(got), float(expect))


def pin_lapack_factors_match_jacobi(sq):
    """The LAPACK route to the truncated factors gives the same rank-r
    product as the oracle's Jacobi sweeps (both are the Eckart-Young optimum;
    singular vectors may differ in sign, which cancels in L1 L2), so either
    can prepare a layer: the products agree to the 16-bit rounding of the
    factors, and the residual norms to the same order."""
    rng = np.random.default_rng(19)
    for (K, N, r, dt) in ((96, 80, 8, "bf16"), (64, 160, 16, "fp16")):
        Wt = (rng.standard_normal((N, K)) / math.sqrt(K)).astype(np.float32)
        x = rng.standard_normal((32, K)); x[:, [3, 40]] *= 50
        _, lam = sq.smoothing_factors(x, Wt, 0.5)
        W_hat = sq.smooth_weight(Wt, lam)
        A1, A2, sa = sq.low_rank_factors(W_hat, r, dt, "jacobi")
        B1, B2, sb = sq.low_rank_factors(W_hat, r, dt, "lapack")
        assert np.max(np.abs(sa - sb)) <= 1e-12 * sa[0]
        P, Q = A1 @ A2, B1 @ B2
        u = 2.0 ** (-8 if dt == "bf16" else -11)
        assert np.linalg.norm(P - Q) <= 4 * u * np.linalg.norm(P)
        ra = np.linalg.norm(W_hat - P); rb = np.linalg.norm(W_hat - Q)
        assert abs(ra - rb) <= 4 * u * np.linalg.norm(P)


# ---------------------------------------------------------------- chained layers
def _bf16_exact(q: Fraction) -> float:
    """An exact rational rounded to the nearest bf16 value (8 significant bits),
    ties to the even significand (normal range only)."""
    if q == 0:
        return 0.0
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = math.frexp(float(a))[1] - 1                 # 2^e <= a < 2^(e+1), fixed up exactly below
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - 7)
    n = a / ulp
    k = n.numerator // n.denominator
    rem = n - k
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and k % 2 == 1):
        k += 1
    return sign * float(k * ulp)


def _nearest_code(t: float, values, max_code: int) -> int:
    """Exhaustive nearest non-negative code to |t| among codes 0..max_code,
    ties to the even code, magnitudes past the largest clamped to it."""
    a = abs(t)
    best, best_err = 0, None
    for c in range(max_code + 1):
        err = abs(Fraction(a) - Fraction(float(values[c])))
        if best_err is None or err < best_err or (err == best_err and c % 2 == 0):
            best, best_err = c, err
    return best


def pin_next_layer_input_bruteforce(sq):
    """The next layer's quantised input, by brute force on a tiny pair of
    NVFP4 layers: this layer's Y in exact rationals from its (pinned) codes,
    rounded to bf16 by exact arithmetic, smoothed by the NEXT layer's
    1/lambda in fp32, block scales and codes by exhaustive nearest search
    over the E4M3 / E2M1 grids under the next layer's tensor scale, and u'
    exact from the bf16-rounded smoothed values and the next layer's L1."""
    from oracle import formats
    rng = np.random.default_rng(31)
    M, K, N, N2, r = 3, 16, 32, 16, 2
    x = rng.standard_normal((M, K)); x[:, 3] *= 20
    x = formats.to_bf16(x)
    Wt1 = rng.standard_normal((N, K)).astype(np.float32); b1 = rng.standard_normal(N).astype(np.float32)
    Wt2 = (rng.standard_normal((N2, N)) * 0.2).astype(np.float32); b2 = rng.standard_normal(N2).astype(np.float32)
    p1 = sq.prepare(x, Wt1, b1, r, "nvfp4", "bf16")
    y_cal = sq.forward_bf16(x, p1)                  # the next layer is calibrated on what it sees
    y_cal[:, ::5] *= 3.0                            # ... widened so that its outliers differ from Y's
    p2 = sq.prepare(formats.to_bf16(y_cal), Wt2, b2, r, "nvfp4", "bf16")
    a = sq.next_layer_input(x, p1, p2)
    _, a1, _, _ = sq.forward(x, p1, return_parts=True)
    sgx1, sgw1 = Fraction(float(p1.s_gx)), Fraction(float(p1.wq.s_g))
    dx = [[sgx1 * Fraction(float(formats.E4M3_VALUES[a1.scales[m, k // 16]]))
           * Fraction(float(formats.E2M1_VALUES[a1.codes[m, k]])) for k in range(K)] for m in range(M)]
    dw = [[sgw1 * Fraction(float(formats.E4M3_VALUES[p1.wq.scales[n, k // 16]]))
           * Fraction(float(formats.E2M1_VALUES[p1.wq.codes[n, k]])) for k in range(K)] for n in range(N)]
    x16 = [[Fraction(_bf16_exact(Fraction(float(np.float32(x[m, k]) * np.float32(p1.inv_lambda[k])))))
            for k in range(K)] for m in range(M)]
    s_g2 = np.float32(p2.s_gx)
    six = np.float32(np.float32(6.0) * s_g2)
    for m in range(M):
        u1 = [sum(x16[m][k] * Fraction(float(p1.L1[k, i])) for k in range(K)) for i in range(r)]
        y = [_bf16_exact(sum(dx[m][k] * dw[n][k] for k in range(K))
                         + sum(u1[i] * Fraction(float(p1.L2[i, n])) for i in range(r)) + Fraction(float(b1[n])))
             for n in range(N)]
        xh = [np.float32(y[n]) * np.float32(p2.inv_lambda[n]) for n in range(N)]
        for blk in range(N // 16):
            vals = xh[16 * blk:16 * blk + 16]
            amax = max(abs(float(v)) for v in vals)
            ratio = np.float32(np.float32(amax) / six)
            e = _nearest_code(float(ratio), formats.E4M3_VALUES, 0x7E)
            assert a.scales[m, blk] == e, (m, blk, a.scales[m, blk], e)
            d = np.float32(np.float32(formats.E4M3_VALUES[e]) * s_g2)
            for j, v in enumerate(vals):
                if d == 0:
                    code = 0
                else:
                    t = np.float32(v / d)
                    code = _nearest_code(float(t), formats.E2M1_VALUES, 7) | (8 if math.copysign(1.0, float(t)) < 0 else 0)
                assert a.codes[m, 16 * blk + j] == code, (m, blk, j, a.codes[m, 16 * blk + j], code)
        for i in range(r):
            u = sum(Fraction(_bf16_exact(Fraction(float(xh[n])))) * Fraction(float(p2.L1[n, i])) for n in range(N))
            assert abs(a.u[m, i] - float(u)) <= 1e-12 * (abs(float(u)) + 1), (m, i, a.u[m, i], float(u))
