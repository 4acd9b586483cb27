"""Planted mistakes in the oracle's next-row functions (KV-cache codec and
attention reads, LoRA append, column shards, the chained next-layer input)
must each fail at least one of their pins (the CPU tests of tests/test_kv.py,
tests/test_lora.py, tests/test_shard.py and the brute-force chain pin)."""
import dataclasses

import numpy as np
import pytest

import oracle.formats as formats
import oracle.kvcache as kv
import oracle.svdquant as sq
from tests import oracle_pins as P
from tests import test_kv as TK
from tests import test_lora as TL
from tests import test_shard as TS

F32 = np.float32


def _run(pins):
    failures = 0
    for pin in pins:
        try:
            pin()
        except Exception:
            failures += 1
    return failures


KV_PINS = [TK.test_golden_codes, TK.test_round_trip_error_is_half_a_step, TK.test_range_ends_map_to_the_code_ends,
           TK.test_asymmetric_beats_symmetric_on_skewed_data]
LORA_PINS = [lambda: TL.test_oracle_lora_adds_exactly_xab_without_smoothing("nvfp4"),
             lambda: TL.test_oracle_lora_with_smoothing_matches_xab_to_the_dtype("int4", "fp16")]
ATT_PINS = [TK.test_attention_matches_sdpa_on_decoded_cache, TK.test_attention_closed_forms]
SHARD_PINS = [lambda: TS.test_oracle_shard_is_the_full_layers_columns("int4", "fp16"),
              lambda: TS.test_oracle_shard_is_the_full_layers_columns("nvfp4", "bf16")]


def _params(divisor=255.0, widen=True, zsign=-1.0):
    def channel_params(x):
        x32 = np.asarray(x, dtype=np.float64).astype(F32)
        lo, hi = x32.min(axis=0), x32.max(axis=0)
        if widen:
            lo, hi = np.minimum(lo, F32(0)), np.maximum(hi, F32(0))
        s = ((hi - lo) / F32(divisor)).astype(F32)
        s = np.where(s == 0, F32(1.0), s).astype(F32)
        z = np.clip(np.rint((F32(zsign) * lo) / s), 0, 255).astype(np.uint8)
        return s, z
    return channel_params


def _encode_ties_up(x):
    s, z = kv.channel_params(x)
    x32 = np.asarray(x, dtype=np.float64).astype(F32)
    q = np.floor(x32 / s[None, :] + 0.5).astype(np.float64) + z[None, :]
    return np.clip(q, 0, 255).astype(np.uint8), s, z


def _decode_plus_zero(q, s, z):
    d = (q.astype(np.int32) + z[None, :].astype(np.int32)).astype(F32)
    return (d * s[None, :]).astype(F32).astype(np.float64)


def _lora_without_lambda(p, A, B):
    A = np.asarray(A, dtype=np.float64); B = np.asarray(B, dtype=np.float64)
    return sq.Prepared(p.fmt, p.dtype, p.rank + A.shape[1], p.inv_lambda, p.lam_eff,
                       np.hstack([p.L1, formats.to_dtype(A, p.dtype)]), np.vstack([p.L2, formats.to_dtype(B, p.dtype)]),
                       p.sigma, p.R, p.wq, p.s_gx, p.bias)


def _lora_lambda_divides(p, A, B):
    A = np.asarray(A, dtype=np.float64); B = np.asarray(B, dtype=np.float64)
    return sq.Prepared(p.fmt, p.dtype, p.rank + A.shape[1], p.inv_lambda, p.lam_eff,
                       np.hstack([p.L1, formats.to_dtype(A / p.lam_eff[:, None], p.dtype)]),
                       np.vstack([p.L2, formats.to_dtype(B, p.dtype)]), p.sigma, p.R, p.wq, p.s_gx, p.bias)


def _shard_bias_unshifted(p, n0, n1):
    wq = sq.WeightQ(p.wq.fmt, p.wq.codes[n0:n1], p.wq.scales[n0:n1], p.wq.s_g)
    return sq.Prepared(p.fmt, p.dtype, p.rank, p.inv_lambda, p.lam_eff, p.L1, p.L2[:, n0:n1], p.sigma,
                       p.R[:, n0:n1], wq, p.s_gx, p.bias[:n1 - n0])


def _shard_l2_unshifted(p, n0, n1):
    wq = sq.WeightQ(p.wq.fmt, p.wq.codes[n0:n1], p.wq.scales[n0:n1], p.wq.s_g)
    return sq.Prepared(p.fmt, p.dtype, p.rank, p.inv_lambda, p.lam_eff, p.L1, p.L2[:, :n1 - n0], p.sigma,
                       p.R[:, n0:n1], wq, p.s_gx, p.bias[n0:n1])


def _attention_variant(scale_all=False, softmax_axis=1, heads_mix=False):
    def attention(Q, kq, ks, kz, vq, vs, vz, heads):
        Q = np.asarray(Q, dtype=np.float64)
        K = kv.decode(kq, ks, kz); V = kv.decode(vq, vs, vz)
        Mq, C = Q.shape
        d = C // heads
        out = np.empty((Mq, C))
        for h in range(heads):
            cols = slice(h * d, (h + 1) * d)
            qc = Q if heads_mix else Q[:, cols]
            kc = K if heads_mix else K[:, cols]
            S = qc @ kc.T / np.sqrt(C if scale_all else d)
            S = S - S.max(axis=softmax_axis, keepdims=True)
            P = np.exp(S); P = P / P.sum(axis=softmax_axis, keepdims=True)
            out[:, cols] = P @ V[:, cols]
        return out
    return attention


CHAIN_PINS = [lambda: P.pin_next_layer_input_bruteforce(sq)]


def _next_input_unrounded_y(x, p, p_next, group=64):
    return sq.quantize_act(sq.forward(x, p, group), p_next, group)


def _next_input_unsmoothed(x, p, p_next, group=64):
    q = dataclasses.replace(p_next, inv_lambda=np.ones_like(p_next.inv_lambda))
    return sq.quantize_act(sq.forward_bf16(x, p, group), q, group)


def _next_input_this_layers_tensor_scale(x, p, p_next, group=64):
    q = dataclasses.replace(p_next, s_gx=p.s_gx)
    return sq.quantize_act(sq.forward_bf16(x, p, group), q, group)


MUTATIONS = {
    "chain_y_not_rounded_to_bf16": (sq, "next_layer_input", _next_input_unrounded_y, CHAIN_PINS),
    "chain_next_smoothing_dropped": (sq, "next_layer_input", _next_input_unsmoothed, CHAIN_PINS),
    "chain_tensor_scale_of_this_layer": (sq, "next_layer_input", _next_input_this_layers_tensor_scale, CHAIN_PINS),
    "kv_divisor_256": (kv, "channel_params", _params(divisor=256.0), KV_PINS),
    "kv_zero_point_sign": (kv, "channel_params", _params(zsign=1.0), KV_PINS),
    "kv_range_not_widened": (kv, "channel_params", _params(widen=False), KV_PINS),
    "kv_ties_up": (kv, "encode", _encode_ties_up, KV_PINS),
    "kv_decode_adds_zero": (kv, "decode", _decode_plus_zero, KV_PINS),
    "lora_lambda_dropped": (sq, "append_lora", _lora_without_lambda, LORA_PINS),
    "lora_lambda_divides": (sq, "append_lora", _lora_lambda_divides, LORA_PINS),
    "shard_bias_unshifted": (sq, "shard_columns", _shard_bias_unshifted, SHARD_PINS),
    "shard_l2_unshifted": (sq, "shard_columns", _shard_l2_unshifted, SHARD_PINS),
    "attention_scaled_by_all_channels": (kv, "attention", _attention_variant(scale_all=True), ATT_PINS),
    "attention_softmax_over_queries": (kv, "attention", _attention_variant(softmax_axis=0), ATT_PINS),
    "attention_heads_mixed": (kv, "attention", _attention_variant(heads_mix=True), ATT_PINS),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    mod, attr, fn, pins = MUTATIONS[name]
    monkeypatch.setattr(mod, attr, fn)
    assert _run(pins) > 0, f"no pin caught the planted mistake {name!r}"


def test_unmutated_pins_pass():
    assert _run(KV_PINS + LORA_PINS + SHARD_PINS + ATT_PINS + CHAIN_PINS) == 0
