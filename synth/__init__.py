"""Seeded synthetic inputs for the SVDQuant linear layer.

This module only draws numbers.  It holds none of the method's arithmetic
(no smoothing, no SVD, no quantisation), so both the CPU oracle's tests and
the CUDA path's tests/benchmarks can take their inputs from here without
sharing any code of the method.

Random numbers: a counter-based SplitMix64 stream per (seed, tag), uniform
doubles from its top 53 bits, normals by Box-Muller in float64.  Every array
is a pure function of (seed, tag, shape), so the same inputs can be rebuilt on
any machine without files.

Workload shapes follow the pages' workloads: FLUX.1 DiT linears (4096 image +
512 text tokens, hidden 3072, FFN 12288) and Infinity-VAR FFN projections
(hidden 4096 / FFN 16384) with heavy per-channel activation outliers
(VAR-Compressor page, "W4A4权重激活量化": max/median ratio up to 353x in the
FFN down projection).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

TAGS = {"X": 1, "W": 2, "outlier": 3, "bias": 4, "gelu": 5, "extra": 6, "lora_A": 7, "lora_B": 8}


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_seed(seed: int, tag: str | int) -> np.uint64:
    """SplitMix64 finaliser of (seed, tag): the base of one sub-stream."""
    t = TAGS[tag] if isinstance(tag, str) else int(tag)
    with np.errstate(over="ignore"):
        z = np.array([(seed * 0x100000001B3 + t * 0x9E3779B97F4A7C15) & 0xFFFFFFFFFFFFFFFF],
                     dtype=np.uint64)
        return _mix(z)[0]


def u64(seed: int, tag: str | int, n: int, offset: int = 0) -> np.ndarray:
    """n SplitMix64 outputs of sub-stream (seed, tag), counters offset..offset+n-1."""
    base = stream_seed(seed, tag)
    with np.errstate(over="ignore"):
        ctr = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
        return _mix(base + ctr * _GOLDEN)


def uniform(seed: int, tag: str | int, n: int, offset: int = 0) -> np.ndarray:
    """Uniform doubles in (0, 1): (top 53 bits + 0.5) * 2^-53."""
    return ((u64(seed, tag, n, offset) >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normal(seed: int, tag: str | int, n: int) -> np.ndarray:
    """n standard normals by Box-Muller over consecutive uniform pairs."""
    m = (n + 1) // 2
    u = uniform(seed, tag, 2 * m)
    u1, u2 = u[0::2], u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    out = np.empty(2 * m, dtype=np.float64)
    out[0::2] = r * np.cos(2.0 * math.pi * u2)
    out[1::2] = r * np.sin(2.0 * math.pi * u2)
    return out[:n]


def sample_channels(seed: int, K: int, count: int) -> np.ndarray:
    """`count` distinct channel indices out of K (seeded, without replacement), sorted."""
    keys = u64(seed, "outlier", K)
    return np.sort(np.argsort(keys, kind="stable")[:count])


def to_dtype(x64: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to fp16 or bf16 (round to nearest even).

    fp16 uses numpy's float16 conversion.  bf16 is returned as uint16 bit
    patterns (numpy has no bf16); round-to-nearest-even from float64 is done in
    one step on the float64 significand so there is no double rounding.
    """
    if dtype == "fp16":
        return x64.astype(np.float16)
    if dtype == "bf16":
        return f64_to_bf16_bits(x64)
    raise ValueError(dtype)


def f64_to_bf16_bits(x64: np.ndarray) -> np.ndarray:
    x = np.asarray(x64, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m * 2^e, 0.5 <= |m| < 1
    # bf16 keeps 8 significant bits; normal range only (inputs here are far from
    # the bf16 subnormal/overflow limits, checked below).
    q = np.rint(np.ldexp(m, 8))             # exact scaling, rint = ties-to-even
    y = np.ldexp(q, e - 8)
    bad = (x != 0) & ((np.abs(y) < 2.0 ** -126) | (np.abs(y) > 3.3e38))
    if np.any(bad):
        raise ValueError("value outside the bf16 normal range")
    y32 = y.astype(np.float32)              # exact: y has <= 8 significant bits
    return (y32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def dtype_to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "fp16":
        return np.asarray(x, dtype=np.float16).astype(np.float64)
    return bf16_bits_to_f64(x)


@dataclass
class Workload:
    """One synthetic layer: activations X (M x K, fp16 or bf16 bits), weight
    Wt (N x K fp32, nn.Linear layout, W = Wt^T), bias (N fp32) and the layer's
    quantisation settings."""
    name: str
    M: int
    K: int
    N: int
    rank: int
    fmt: str            # "int4" or "nvfp4"
    dtype: str          # "fp16" or "bf16"
    alpha: float = 0.5
    smooth: bool = True
    seed: int = 0
    X: np.ndarray | None = None
    Wt: np.ndarray | None = None
    bias: np.ndarray | None = None
    info: dict = field(default_factory=dict)

    def x_f64(self) -> np.ndarray:
        return dtype_to_f64(self.X, self.dtype)


def gelu_exact(x: np.ndarray) -> np.ndarray:
    from scipy.special import erf
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def make_x(seed: int, M: int, K: int, dtype: str, n_out: int, factor: float,
           kind: str = "normal", ratio: float | None = None, info: dict | None = None):
    """Activations: N(0,1) (or GELU(N(0,1))) with `n_out` seeded outlier channels.

    Outlier channels are multiplied by `factor` in float64 before rounding to the
    16-bit dtype.  With `ratio` given, the factor is chosen so that the
    per-channel absmax statistic max_j amax_j / median_j amax_j equals `ratio`.
    """
    x = normal(seed, "X", M * K).reshape(M, K)
    if kind == "gelu":
        x = gelu_exact(x)
    ch = sample_channels(seed, K, n_out) if n_out > 0 else np.zeros(0, dtype=np.int64)
    if ratio is not None and n_out > 0:
        amax = np.abs(x).max(axis=0)
        rest = np.sort(np.delete(amax, ch))
        # outliers end up above the median, so the median of all K channels is
        # the median position taken among the non-outlier channels
        lo, hi = (K - 1) // 2, K // 2
        med = 0.5 * (rest[lo] + rest[hi])
        factor = ratio * med / amax[ch].max()
    if n_out > 0:
        x[:, ch] *= factor
    xd = to_dtype(x, dtype)
    if info is not None:
        a = np.abs(dtype_to_f64(xd, dtype)).max(axis=0)
        info["outlier_channels"] = int(n_out)
        info["outlier_factor"] = float(factor)
        info["max_over_median_amax"] = float(a.max() / np.median(a))
    return xd


def make_weight(seed: int, N: int, K: int) -> np.ndarray:
    """Wt (N x K) fp32 ~ N(0, std = 1/sqrt(K))."""
    return (normal(seed, "W", N * K) / math.sqrt(K)).astype(np.float32).reshape(N, K)


def make_bias(seed: int, N: int) -> np.ndarray:
    return normal(seed, "bias", N).astype(np.float32)


def make_lora(seed: int, K: int, N: int, r: int) -> tuple[np.ndarray, np.ndarray]:
    """A LoRA adapter: A (K x r) fp32 ~ N(0, 1/sqrt(K)), B (r x N) fp32 ~ N(0, 0.5/sqrt(r))."""
    A = (normal(seed, "lora_A", K * r) / math.sqrt(K)).astype(np.float32).reshape(K, r)
    B = (normal(seed, "lora_B", r * N) * (0.5 / math.sqrt(r))).astype(np.float32).reshape(r, N)
    return A, B


# Workloads.  Shapes and distributions of the pages' layers; no dataset or
# trained weights exist here, so these stand in for FLUX.1 / Infinity-VAR
# activations and weights.
PRESETS = {
    "tiny_int4": dict(M=256, K=512, N=512, rank=16, fmt="int4", dtype="fp16",
                      x=dict(n_out=4, factor=100.0)),
    "flux_qkv_int4": dict(M=4608, K=3072, N=9216, rank=32, fmt="int4", dtype="bf16",
                          x=dict(n_out=31, factor=50.0)),
    "flux_ffn_up_nvfp4": dict(M=4608, K=3072, N=12288, rank=32, fmt="nvfp4", dtype="bf16",
                              x=dict(n_out=31, factor=50.0)),
    "ffn_down_nvfp4": dict(M=4608, K=12288, N=3072, rank=32, fmt="nvfp4", dtype="bf16",
                           x=dict(n_out=61, factor=None, kind="gelu", ratio=353.0)),
    "ffn_down_int4": dict(M=4608, K=12288, N=3072, rank=32, fmt="int4", dtype="bf16",
                          x=dict(n_out=61, factor=None, kind="gelu", ratio=353.0)),
    "var_up_nvfp4": dict(M=4096, K=4096, N=16384, rank=32, fmt="nvfp4", dtype="bf16",
                         x=dict(n_out=41, factor=100.0)),
    "var_down_nvfp4": dict(M=4096, K=16384, N=4096, rank=32, fmt="nvfp4", dtype="bf16",
                           x=dict(n_out=164, factor=100.0)),
}

VAR_TOKENS = (1, 4, 16, 64, 256, 1024, 4096)


def make_workload(name: str, seed: int = 0, M: int | None = None, with_x: bool = True,
                  with_w: bool = True, **over) -> Workload:
    """Build a preset workload (optionally with a different token count M)."""
    p = dict(PRESETS[name])
    p.update(over)
    xs = dict(p.pop("x"))
    wl = Workload(name=name, M=M if M is not None else p["M"], K=p["K"], N=p["N"],
                  rank=p["rank"], fmt=p["fmt"], dtype=p["dtype"], seed=seed,
                  alpha=p.get("alpha", 0.5), smooth=p.get("smooth", True))
    if with_x:
        wl.X = make_x(seed, wl.M, wl.K, wl.dtype, xs["n_out"], xs.get("factor") or 1.0,
                      kind=xs.get("kind", "normal"), ratio=xs.get("ratio"), info=wl.info)
    if with_w:
        wl.Wt = make_weight(seed, wl.N, wl.K)
        wl.bias = make_bias(seed, wl.N)
    return wl


def custom_workload(M: int, K: int, N: int, rank: int, fmt: str, dtype: str, seed: int = 0,
                    n_out: int = 0, factor: float = 1.0, alpha: float = 0.5,
                    smooth: bool = True, name: str = "custom") -> Workload:
    wl = Workload(name=name, M=M, K=K, N=N, rank=rank, fmt=fmt, dtype=dtype, seed=seed,
                  alpha=alpha, smooth=smooth)
    wl.X = make_x(seed, M, K, dtype, n_out, factor, info=wl.info)
    wl.Wt = make_weight(seed, N, K)
    wl.bias = make_bias(seed, N)
    return wl
