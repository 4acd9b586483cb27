"""Asymmetric per-channel INT8 KV-cache codec -- test infrastructure only.

Source: "VAR-Compressor：在边缘GPU上实现80亿参数视觉自回归模型的高效量化部署",
INT8 KV缓存量化 and KV缓存特性研究.  The VAR KV cache grows with the sequence,
its variance is driven by channels (CV_channel > 1.2) and it is skewed
(skewness about 0.85), so it is quantised to INT8 per channel with an
asymmetric (non-centred) zero point.

Readings where the page is silent:
  * A block of T cached tokens x C channels (row-major, fp16 / bf16) is
    quantised with one (scale, zero point) per channel, from that channel's
    range over the block's tokens.  The range is widened to contain 0, so a
    zero entry (padding) is exact.
  * Codes are unsigned bytes 0..255; the zero point is an integer in 0..255.
  * All arithmetic in fp32, round to nearest even, no fused multiply-add:
      lo = min(0, min_t x), hi = max(0, max_t x)
      s  = (hi - lo) / 255          (s = 1 when hi == lo, i.e. an all-zero channel)
      z  = clamp(rint(-lo / s), 0, 255)
      q  = clamp(rint(x / s) + z, 0, 255)
      x' = (q - z) * s              (decoded, then rounded to the cache dtype)
"""
from __future__ import annotations

import numpy as np

F32 = np.float32


def channel_params(x: np.ndarray):
    """Per-channel fp32 scale and uint8 zero point of a T x C block (values as
    float64 holding fp16/bf16 numbers)."""
    x32 = np.asarray(x, dtype=np.float64).astype(F32)
    lo = np.minimum(x32.min(axis=0), F32(0.0)).astype(F32)
    hi = np.maximum(x32.max(axis=0), F32(0.0)).astype(F32)
    s = ((hi - lo) / F32(255.0)).astype(F32)
    s = np.where(s == 0, F32(1.0), s).astype(F32)
    z = np.clip(np.rint((-lo) / s), 0, 255).astype(np.uint8)
    return s, z


def encode(x: np.ndarray):
    """T x C block -> (codes uint8 T x C, scale fp32 C, zero uint8 C)."""
    s, z = channel_params(x)
    x32 = np.asarray(x, dtype=np.float64).astype(F32)
    q = np.rint(x32 / s[None, :]).astype(np.float64) + z[None, :].astype(np.float64)
    return np.clip(q, 0, 255).astype(np.uint8), s, z


def decode(q: np.ndarray, s: np.ndarray, z: np.ndarray) -> np.ndarray:
    """(q - z) * s in fp32 (float64 out, holding the fp32 values)."""
    d = (q.astype(np.int32) - z[None, :].astype(np.int32)).astype(F32)
    return (d * np.asarray(s, dtype=F32)[None, :]).astype(F32).astype(np.float64)


def attention(Q: np.ndarray, kq, ks, kz, vq, vs, vz, heads: int) -> np.ndarray:
    """Attention reads over the INT8 cache: for each head h (channels
    [h d, (h + 1) d), d = C / heads) and query row i,
        S[i, t] = sum_c Q[i, c] K^[t, c] / sqrt(d),   P = softmax_t(S),
        O[i, c] = sum_t P[i, t] V^[t, c],
    with K^ = decode(kq, ks, kz) and V^ = decode(vq, vs, vz) -- the cached
    keys and values as the codec restores them (exact fp32 values) -- in
    float64.  Q: Mq x C values (float64 holding fp16/bf16 numbers).
    Scaled dot-product attention is the VAR transformer's attention; the
    VAR-Compressor page (INT8 KV缓存量化) stores its cache as INT8, and this is
    the read of that cache."""
    Q = np.asarray(Q, dtype=np.float64)
    K = decode(kq, ks, kz)
    V = decode(vq, vs, vz)
    Mq, C = Q.shape
    d = C // heads
    out = np.empty((Mq, C), dtype=np.float64)
    for h in range(heads):
        cols = slice(h * d, (h + 1) * d)
        S = Q[:, cols] @ K[:, cols].T / np.sqrt(d)
        S = S - S.max(axis=1, keepdims=True)
        P = np.exp(S)
        P = P / P.sum(axis=1, keepdims=True)
        out[:, cols] = P @ V[:, cols]
    return out
