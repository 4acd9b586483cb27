"""The SVDQuant linear layer, step by step, in the pages' order and notation.

Test infrastructure only (see the package docstring).

    X^ = X diag(lambda)^-1,  W^ = diag(lambda) W          smoothing
    W^ = U S V^T,  L1 = U_r S_r,  L2 = V_r^T              rank-r branch, 16-bit
    R  = W^ - L1 L2                                       residual
    Y  = Q(X^) Q(R) + (X^ L1) L2 + b                      layer output

Sources: "SVDQuant是什么？…" 技术原理 (smoothing moves activation outliers into
the weight, SVD splits the weight into a 16-bit low-rank branch and a 4-bit
residual, Eckart-Young-Mirsky); "AI图像生成4-bit量化技术解析与应用" 2.2 (the
three SVD steps) and 3.1 (dynamic activation quantisation); "DeepCompressor…"
SVDQuant section (low-rank branch summed with the 4-bit branch).

Readings where the pages are silent (each listed in the design notes):
  * lambda: per input channel j, lambda_j = a_j^alpha / w_j^(1-alpha) with
    a_j = max_m |X_cal[m, j]| and w_j = max_n |W[j, n]| (the SmoothQuant rule
    the DeepCompressor page names as the ancestor); lambda_j = 1 when a_j or
    w_j is 0 or smoothing is off.  The device keeps inv_lambda = fp32(1/lambda)
    and the weight is smoothed with lambda_eff = 1 / (double) inv_lambda, so the
    two sides use the same factor.
  * L1 = U_r S_r, L2 = V_r^T, both rounded to the activation dtype; R is taken
    from the rounded factors so it absorbs their rounding.
  * Activations are quantised per token (row) in groups along K; the NVFP4
    tensor scale of the activations is static (from calibration).
  * The low-rank input X^ is rounded to the activation dtype (the branch runs
    in 16 bits); u = X^16 L1 is exact in float64.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import formats, quant
from .svd import jacobi_svd, lapack_svd

F32 = np.float32


# ---------------------------------------------------------------- offline side
def smoothing_factors(x_cal: np.ndarray, Wt: np.ndarray, alpha: float, smooth: bool = True):
    """inv_lambda (fp32 [K]) and the effective lambda used on the weight (f64 [K]).

    x_cal: calibration activations as float64 values (M_cal x K).
    Wt:    weight in nn.Linear layout (N x K, fp32); W = Wt^T is K x N.
    """
    K = Wt.shape[1]
    if not smooth:
        lam = np.ones(K, dtype=np.float64)
    else:
        a = np.abs(np.asarray(x_cal, dtype=np.float64)).max(axis=0) if x_cal.shape[0] else np.zeros(K)
        w = np.abs(np.asarray(Wt, dtype=np.float64)).max(axis=0)        # max over n of |W[j, n]|
        ok = (a > 0) & (w > 0)
        lam = np.ones(K, dtype=np.float64)
        lam[ok] = np.power(a[ok], alpha) / np.power(w[ok], 1.0 - alpha)
    inv_lambda = (1.0 / lam).astype(F32)
    lam_eff = 1.0 / inv_lambda.astype(np.float64)
    return inv_lambda, lam_eff


def smooth_weight(Wt: np.ndarray, lam_eff: np.ndarray) -> np.ndarray:
    """W^ = diag(lambda) W, float64, K x N."""
    return np.asarray(Wt, dtype=np.float64).T * lam_eff[:, None]


def low_rank_factors(W_hat: np.ndarray, rank: int, dtype: str, svd: str = "jacobi"):
    """Top-`rank` SVD factors of W^, rounded to the 16-bit dtype.

    Returns (L1 K x r, L2 r x N, all singular values), factors as float64
    holding dtype values.  svd: "jacobi" (the oracle's own sweeps) or
    "lapack" (numpy's routine, for full-size layers).
    """
    U, s, Vt = jacobi_svd(W_hat) if svd == "jacobi" else lapack_svd(W_hat)
    L1 = formats.to_dtype(U[:, :rank] * s[None, :rank], dtype)
    L2 = formats.to_dtype(Vt[:rank, :], dtype)
    return L1, L2, s


def residual(W_hat: np.ndarray, L1: np.ndarray, L2: np.ndarray) -> np.ndarray:
    """R = W^ - L1 L2 in float64 with the rank-1 terms summed in ascending
    order (each product rounded, then added; no fused multiply-add), then
    rounded to fp32."""
    S = np.zeros_like(W_hat)
    for i in range(L1.shape[1]):
        S = S + L1[:, i:i + 1] * L2[i:i + 1, :]
    return (W_hat - S).astype(F32)


@dataclass
class WeightQ:
    fmt: str
    codes: np.ndarray          # N x K: int8 INT4 codes, or uint8 E2M1 codes
    scales: np.ndarray         # N x K/g: fp32 (INT4) or uint8 E4M3 codes (NVFP4)
    s_g: np.float32 = F32(1.0)


def quantize_weight(R32: np.ndarray, fmt: str, group: int = 64) -> WeightQ:
    """Quantise the fp32 residual (K x N) per output channel along K."""
    Rt = np.ascontiguousarray(R32.T)                          # N x K
    if fmt == "int4":
        q, s = quant.int4_group_quant(Rt, group)
        return WeightQ("int4", q, s)
    s_g = quant.nvfp4_tensor_scale(np.abs(Rt).max() if Rt.size else 0.0)
    c, e = quant.nvfp4_quant(Rt, s_g)
    return WeightQ("nvfp4", c, e, s_g)


@dataclass
class Prepared:
    fmt: str
    dtype: str
    rank: int
    inv_lambda: np.ndarray     # fp32 K
    lam_eff: np.ndarray        # f64 K
    L1: np.ndarray             # f64 K x r (dtype values)
    L2: np.ndarray             # f64 r x N (dtype values)
    sigma: np.ndarray | None
    R: np.ndarray              # fp32 K x N
    wq: WeightQ
    s_gx: np.float32           # NVFP4 static activation tensor scale (1 for INT4)
    bias: np.ndarray           # fp32 N


def act_tensor_scale(x_cal: np.ndarray, inv_lambda: np.ndarray) -> np.float32:
    """NVFP4 activation tensor scale from calibration: amax(X^_cal) / 2688."""
    xh = smooth_act(x_cal, inv_lambda)
    return quant.nvfp4_tensor_scale(np.abs(xh).max() if xh.size else 0.0)


def prepare(x_cal, Wt, bias, rank, fmt, dtype, alpha=0.5, smooth=True, group=64,
            factors=None, svd="jacobi") -> Prepared:
    """Offline side of the layer.  `factors` = (inv_lambda, L1, L2) replaces the
    oracle's own smoothing/SVD (used to re-derive R and its codes from another
    implementation's stored factors).  `svd` picks the SVD routine (see
    low_rank_factors)."""
    if factors is None:
        inv_lambda, lam_eff = smoothing_factors(x_cal, Wt, alpha, smooth)
        W_hat = smooth_weight(Wt, lam_eff)
        if rank > 0:
            L1, L2, sigma = low_rank_factors(W_hat, rank, dtype, svd)
        else:
            L1 = np.zeros((W_hat.shape[0], 0)); L2 = np.zeros((0, W_hat.shape[1])); sigma = None
    else:
        inv_lambda, L1, L2 = factors
        inv_lambda = np.asarray(inv_lambda, dtype=F32)
        lam_eff = 1.0 / inv_lambda.astype(np.float64)
        W_hat = smooth_weight(Wt, lam_eff)
        sigma = None
    R = residual(W_hat, L1, L2)
    wq = quantize_weight(R, fmt, group)
    s_gx = act_tensor_scale(x_cal, inv_lambda) if fmt == "nvfp4" else F32(1.0)
    b = np.zeros(Wt.shape[0], dtype=F32) if bias is None else np.asarray(bias, dtype=F32)
    return Prepared(fmt, dtype, L1.shape[1], inv_lambda, lam_eff, L1, L2, sigma, R, wq, s_gx, b)


def append_lora(p: Prepared, A: np.ndarray, B: np.ndarray) -> Prepared:
    """A LoRA adapter X A B added to a prepared layer with no re-quantisation
    ("SVDQuant是什么？…" 概述简介 and 功能特色, LoRA集成).  Reading: the adapter
    joins the 16-bit branch.  X = X^ diag(lambda), so X A B = X^ (diag(lambda) A) B:
    L1 gains the columns dtype(lambda_eff A) and L2 the rows dtype(B); the
    residual R, its codes and scales, lambda and the bias stay as they are."""
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    L1 = np.hstack([p.L1, formats.to_dtype(p.lam_eff[:, None] * A, p.dtype)])
    L2 = np.vstack([p.L2, formats.to_dtype(B, p.dtype)])
    return Prepared(p.fmt, p.dtype, p.rank + A.shape[1], p.inv_lambda, p.lam_eff, L1, L2, p.sigma, p.R, p.wq,
                    p.s_gx, p.bias)


def shard_columns(p: Prepared, n0: int, n1: int) -> Prepared:
    """Output features [n0, n1) of a prepared layer: the columns of L2, R, the
    weight codes and scales and the bias; lambda, L1 and the tensor scales are
    the whole layer's.  Every output column of the layer depends only on its
    own weight row, so the shard computes exactly those columns."""
    wq = WeightQ(p.wq.fmt, p.wq.codes[n0:n1], p.wq.scales[n0:n1], p.wq.s_g)
    return Prepared(p.fmt, p.dtype, p.rank, p.inv_lambda, p.lam_eff, p.L1, p.L2[:, n0:n1], p.sigma,
                    p.R[:, n0:n1], wq, p.s_gx, p.bias[n0:n1])


# ----------------------------------------------------------------- online side
def smooth_act(x: np.ndarray, inv_lambda: np.ndarray) -> np.ndarray:
    """X^ = fp32(x) * inv_lambda, one fp32 multiply per element."""
    return (np.asarray(x, dtype=np.float64).astype(F32) * np.asarray(inv_lambda, dtype=F32)).astype(F32)


@dataclass
class ActQ:
    fmt: str
    codes: np.ndarray          # M x K: int8 INT4 codes or uint8 E2M1 codes
    scales: np.ndarray         # M x K/g: fp32 (INT4) or uint8 E4M3 (NVFP4)
    u: np.ndarray              # M x r float64: X^16 L1


def quantize_act(x: np.ndarray, p: Prepared, group: int = 64) -> ActQ:
    """Dynamic activation quantisation (per token, groups along K) and the
    low-rank down projection u = X^16 L1 (X^16 = X^ rounded to the dtype)."""
    xh = smooth_act(x, p.inv_lambda)
    if p.fmt == "int4":
        codes, scales = quant.int4_group_quant(xh, group)
    else:
        codes, scales = quant.nvfp4_quant(xh, p.s_gx)
    x16 = formats.to_dtype(xh.astype(np.float64), p.dtype)
    u = x16 @ p.L1 if p.rank > 0 else np.zeros((x16.shape[0], 0))
    return ActQ(p.fmt, codes, scales, u)


def main_product(a: ActQ, p: Prepared, group: int = 64) -> np.ndarray:
    """Q(X^) Q(R) in float64.

    INT4: sum over groups g of sx[m,g] * sw[n,g] * (integer dot product over the
    group); the integer dots are exact (float64 holds them exactly).
    NVFP4: s_gX * s_gW * sum_k (qx ex)(qw ew); each product is exact in float64.
    """
    if p.fmt == "int4":
        M, K = a.codes.shape
        N = p.wq.codes.shape[0]
        Y = np.zeros((M, N), dtype=np.float64)
        for g in range(K // group):
            sl = slice(g * group, (g + 1) * group)
            dots = a.codes[:, sl].astype(np.float64) @ p.wq.codes[:, sl].astype(np.float64).T
            Y += (a.scales[:, g].astype(np.float64)[:, None]
                  * p.wq.scales[:, g].astype(np.float64)[None, :]) * dots
        return Y
    xd = quant.nvfp4_dequant(a.codes, a.scales, 1.0)
    wd = quant.nvfp4_dequant(p.wq.codes, p.wq.scales, 1.0)
    return (float(p.s_gx) * float(p.wq.s_g)) * (xd @ wd.T)


def forward(x: np.ndarray, p: Prepared, group: int = 64, return_parts: bool = False):
    """Y = Q(X^) Q(R) + u L2 + b in float64 (before the output rounding)."""
    a = quantize_act(x, p, group)
    main = main_product(a, p, group)
    low = a.u @ p.L2 if p.rank > 0 else 0.0
    Y = main + low + p.bias.astype(np.float64)[None, :]
    if return_parts:
        return Y, a, main, low
    return Y


def forward_bf16(x: np.ndarray, p: Prepared, group: int = 64) -> np.ndarray:
    """The layer output rounded to bf16 (the device writes bf16)."""
    return formats.to_bf16(forward(x, p, group))


def next_layer_input(x: np.ndarray, p: Prepared, p_next: Prepared, group: int = 64) -> ActQ:
    """The quantised input of the next layer when this layer feeds it.

    The next layer reads this layer's output as the layer writes it (bf16 Y)
    and treats it like any activation: its own smoothing, dynamic
    quantisation and low-rank down projection, i.e. quantize_act(bf16(Y),
    p_next).  Fusing this into this layer's epilogue only moves where it is
    computed ("DeepCompressor…" SVDQuant section: the low-rank branch is
    folded into the low-bit kernel to save the activation round trip; the
    same saving at the boundary between two layers).
    """
    y = forward_bf16(x, p, group)
    return quantize_act(y, p_next, group)


def exact_output(x: np.ndarray, Wt: np.ndarray, bias) -> np.ndarray:
    """The unquantised layer X W + b in float64 (for error reports)."""
    b = 0.0 if bias is None else np.asarray(bias, dtype=np.float64)[None, :]
    return np.asarray(x, dtype=np.float64) @ np.asarray(Wt, dtype=np.float64).T + b


def rel_fro(a: np.ndarray, b: np.ndarray) -> float:
    """||a - b||_F / ||b||_F."""
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / nb) if nb > 0 else float(np.linalg.norm(a - b))
