"""INT8 KV-cache codec ("VAR-Compressor…" INT8 KV缓存量化): the oracle against
a hand-worked fixture and the rule's invariants (CPU), the CUDA kernels
against the oracle (GPU, bit-exact codes / scales / zero points and decoded
values)."""
import os

import numpy as np
import pytest

import synth
from oracle import kvcache as kv

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kv_int8_asym.txt")


def load_golden():
    chans = []
    for line in open(GOLDEN):
        if not line.strip() or line.startswith("#"):
            continue
        f = line.split()
        pairs = [tuple(map(float, t.split(":"))) for t in f[3:]]
        chans.append((float(f[1]), int(f[2]), [p[0] for p in pairs], [int(p[1]) for p in pairs]))
    return chans


def test_golden_codes():
    chans = load_golden()
    x = np.array([c[2] for c in chans]).T            # T x C
    q, s, z = kv.encode(x)
    assert np.array_equal(s, np.array([c[0] for c in chans], np.float32))
    assert np.array_equal(z, np.array([c[1] for c in chans], np.uint8))
    assert np.array_equal(q, np.array([c[3] for c in chans], np.uint8).T)


def skewed_block(T, C, seed):
    """Channel-driven variance (per-channel scales spread over 3 decades) and
    positive skew (a shifted log-normal), as the page describes the cache."""
    g = synth.normal(seed, "X", T * C).reshape(T, C)
    scale = np.exp(synth.normal(seed, "extra", C) * 1.2)
    x = (np.exp(0.6 * g) - 1.2) * scale[None, :]
    return synth.dtype_to_f64(synth.to_dtype(x, "fp16"), "fp16")


def test_round_trip_error_is_half_a_step():
    x = skewed_block(257, 192, 3)
    q, s, z = kv.encode(x)
    err = np.abs(kv.decode(q, s, z) - x)
    assert np.all(err <= 0.5 * s[None, :] * (1 + 1e-5) + 1e-30)


def test_range_ends_map_to_the_code_ends():
    x = skewed_block(64, 256, 4)
    q, s, z = kv.encode(x)
    lo, hi = np.minimum(x.min(0), 0), np.maximum(x.max(0), 0)
    rows_lo, rows_hi = x.argmin(0), x.argmax(0)
    c = np.arange(x.shape[1])
    assert np.all(q[rows_lo, c][lo < 0] == 0)
    assert np.all(np.isin(q[rows_hi, c][hi > 0], (254, 255)))
    # a zero entry is exact: it decodes to 0
    assert np.all(kv.decode(np.broadcast_to(z, (1, z.size)).copy(), s, z) == 0)


def test_asymmetric_beats_symmetric_on_skewed_data():
    """The page's reason for the zero point: on the skewed cache the
    asymmetric step is finer than a symmetric int8 step (absmax / 127)."""
    x = skewed_block(128, 128, 5)
    q, s, z = kv.encode(x)
    sym = np.abs(x).max(0) / 127.0
    assert np.all(s <= sym * (1 + 1e-6))
    assert np.mean(np.abs(kv.decode(q, s, z) - x)) < 0.75 * np.mean(
        np.abs(np.clip(np.rint(x / sym), -127, 127) * sym - x))
