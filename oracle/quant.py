"""4-bit quantisers of the oracle (fp32 IEEE arithmetic, round-to-nearest).

Both quantisers work on rows: a (rows x K) fp32 matrix is quantised in
groups of consecutive elements along K inside each row.  For activations a
row is a token; for the weight residual a row is one output channel n of
R^T (N x K), i.e. groups run along the reduction dimension K.

INT4, group 64 -- the symmetric absmax quantiser of the W4A8 page (3.1,
权重量化) with b = 4, applied per group:
    m = max |v| over the group;  s = m / 7;  q = clamp(rint(v / s), -8, 7)
    (s = 0 and q = 0 when m = 0).
The 4-bit page (3.1) speaks of 16x16 blocks with a zero point; a zero point
would add cross terms that a fused 4-bit GEMM cannot absorb, so the oracle
takes the symmetric form the W4A8 page prints, with groups of 64 along K.

NVFP4 -- E2M1 elements, one E4M3 scale per 16 consecutive elements and one
fp32 tensor scale s_g (4-bit page, 3.2, read as the standard NVFP4 recipe):
    s_g = amax / 2688  (2688 = 6 * 448; s_g = 1 when amax = 0)
    per block: e = E4M3(m_b / (6 * s_g));  d = e * s_g
               q = E2M1(v / d)  (all codes 0 when d = 0)
For the weight, amax is over the whole residual; for activations s_g is
static, taken from the calibration activations.
All operations are single fp32 operations (numpy float32), no fused
multiply-add, divisions are IEEE divisions.
"""
from __future__ import annotations

import numpy as np

from . import formats

F32 = np.float32


def int4_group_quant(v: np.ndarray, group: int = 64):
    """Symmetric INT4 per-group quantisation along the last axis.

    Returns (q int8 [rows, K], s fp32 [rows, K // group]).
    """
    v = np.asarray(v, dtype=F32)
    rows, K = v.shape
    assert K % group == 0
    vg = v.reshape(rows, K // group, group)
    m = np.abs(vg).max(axis=2)                               # fp32, exact
    s = (m / F32(7.0)).astype(F32)                           # IEEE fp32 division
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (vg / s[:, :, None]).astype(F32)                 # fp32 division
    q = np.rint(t)                                           # ties to even
    q = np.where(m[:, :, None] == 0, 0.0, q)
    q = np.clip(q, -8, 7).astype(np.int8)
    return q.reshape(rows, K), s


def int4_dequant(q: np.ndarray, s: np.ndarray, group: int = 64) -> np.ndarray:
    rows, K = q.shape
    return (q.reshape(rows, K // group, group).astype(np.float64)
            * s.astype(np.float64)[:, :, None]).reshape(rows, K)


def nvfp4_tensor_scale(amax: float) -> np.float32:
    """s_g = amax / 2688 in fp32; 1 when amax is 0."""
    s = F32(F32(amax) / F32(2688.0))
    return F32(1.0) if s == 0 else s


def nvfp4_quant(v: np.ndarray, s_g: np.float32, block: int = 16):
    """NVFP4 quantisation along the last axis with a given fp32 tensor scale.

    Returns (codes uint8 [rows, K] -- one E2M1 code per element, low nibble,
             scales uint8 [rows, K // block] -- E4M3 codes).
    """
    v = np.asarray(v, dtype=F32)
    rows, K = v.shape
    assert K % block == 0
    s_g = F32(s_g)
    vb = v.reshape(rows, K // block, block)
    mb = np.abs(vb).max(axis=2)                              # block amax, fp32
    six_sg = F32(F32(6.0) * s_g)                             # fp32 product
    ratio = (mb / six_sg).astype(F32)                        # fp32 division
    e = formats.e4m3_encode(ratio.astype(np.float64))        # exact fp32 -> E4M3 RNE satfinite
    ev = formats.e4m3_decode(e).astype(F32)
    d = (ev * s_g).astype(F32)                               # fp32 product
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (vb / d[:, :, None]).astype(F32)                 # fp32 division
    t = np.where(d[:, :, None] == 0, F32(0.0), t)
    codes = formats.e2m1_encode(t.astype(np.float64))
    codes = np.where(d[:, :, None] == 0, np.uint8(0), codes).astype(np.uint8)
    return codes.reshape(rows, K), e.reshape(rows, K // block)


def nvfp4_dequant(codes: np.ndarray, scales: np.ndarray, s_g, block: int = 16) -> np.ndarray:
    """Element value = E2M1(code) * E4M3(scale) * s_g, in float64 (exact)."""
    rows, K = codes.shape
    q = formats.e2m1_decode(codes).reshape(rows, K // block, block)
    e = formats.e4m3_decode(scales)[:, :, None]
    return (q * e * float(s_g)).reshape(rows, K)
