"""Planted mistakes in the CPU oracle must each fail at least one pin.

Each case patches one function of the oracle with a plausible slip (a sign,
an index, a dropped term, a wrong constant, a wrong rounding tie) and runs the
pins; the test passes only if some pin rejects the patched oracle.
"""
import numpy as np
import pytest

import oracle.formats as formats
import oracle.quant as quant
import oracle.svd as svd
import oracle.svdquant as sq
from tests import oracle_pins as P

F32 = np.float32


def _run_all_pins():
    pins = [
        lambda: P.pin_format_tables(formats),
        lambda: P.pin_encoders_bruteforce(formats, n=500),
        lambda: P.pin_int4_golden(quant),
        lambda: P.pin_int4_bruteforce(quant),
        lambda: P.pin_nvfp4_bounds(quant, formats),
        lambda: P.pin_eckart_young(svd, sq),
        lambda: P.pin_smoothing(sq),
        lambda: P.pin_rank0_plain_rtn(sq),
        lambda: P.pin_bruteforce_int4(sq),
        lambda: P.pin_bruteforce_nvfp4(sq),
        lambda: P.pin_special_cases(sq),
        lambda: P.pin_on_grid_lossless(sq),
        lambda: P.pin_low_rank_helps(sq),
        lambda: P.pin_act_tensor_scale_golden(sq),
        lambda: P.pin_act_codes_golden(sq),
        lambda: P.pin_act_scale_in_prepare(sq),
    ]
    failures = 0
    for pin in pins:
        try:
            pin()
        except Exception:
            failures += 1
    return failures


def _residual_plus(W_hat, L1, L2):
    S = np.zeros_like(W_hat)
    for i in range(L1.shape[1]):
        S = S + L1[:, i:i + 1] * L2[i:i + 1, :]
    return (W_hat + S).astype(F32)


def _smooth_weight_divides(Wt, lam_eff):
    return np.asarray(Wt, dtype=np.float64).T / lam_eff[:, None]


def _int4_by_8(v, group=64):
    v = np.asarray(v, dtype=F32)
    rows, K = v.shape
    vg = v.reshape(rows, K // group, group)
    m = np.abs(vg).max(axis=2)
    s = (m / F32(8.0)).astype(F32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.rint((vg / s[:, :, None]).astype(F32))
    q = np.clip(np.where(m[:, :, None] == 0, 0, q), -8, 7).astype(np.int8)
    return q.reshape(rows, K), s


def _tensor_scale_448(amax):
    s = F32(F32(amax) / F32(448.0))
    return F32(1.0) if s == 0 else s


_orig_forward = sq.forward


def _forward_no_bias(x, p, group=64, return_parts=False):
    Y, a, main, low = _orig_forward(x, p, group, return_parts=True)
    Y = Y - p.bias.astype(np.float64)[None, :]
    return (Y, a, main, low) if return_parts else Y


_orig_qa = sq.quantize_act


def _quantize_act_unsmoothed_u(x, p, group=64):
    a = _orig_qa(x, p, group)
    x16 = formats.to_dtype(np.asarray(x, dtype=np.float64), p.dtype)
    a.u = x16 @ p.L1 if p.rank > 0 else a.u
    return a


def _main_product_swapped_group(a, p, group=64):
    if p.fmt != "int4":
        return _orig_main(a, p, group)
    M, K = a.codes.shape
    N = p.wq.codes.shape[0]
    G = K // group
    Y = np.zeros((M, N))
    for g in range(G):
        sl = slice(g * group, (g + 1) * group)
        dots = a.codes[:, sl].astype(np.float64) @ p.wq.codes[:, sl].astype(np.float64).T
        Y += (a.scales[:, g].astype(np.float64)[:, None]
              * p.wq.scales[:, (g + 1) % G].astype(np.float64)[None, :]) * dots
    return Y


_orig_main = sq.main_product


def _e2m1_tie_up(x):
    x = np.asarray(x, dtype=np.float64)
    mags = formats.E2M1_VALUES[:8]
    mids = 0.5 * (mags[:-1] + mags[1:])
    j = np.searchsorted(mids, np.abs(x), side="right")       # ties go up
    return (np.minimum(j, 7) | np.where(np.signbit(x), 8, 0)).astype(np.uint8)


def _to_dtype_truncate(x, dtype):
    x = np.asarray(x, dtype=np.float64)
    bits = 8 if dtype == "bf16" else 11
    m, e = np.frexp(x)
    return np.ldexp(np.trunc(np.ldexp(m, bits)), e - bits)


def _act_tensor_scale_unsmoothed(x_cal, inv_lambda):
    x = np.asarray(x_cal, dtype=np.float64).astype(F32)
    return quant.nvfp4_tensor_scale(np.abs(x).max() if x.size else 0.0)


def _quantize_act_codes_unsmoothed(x, p, group=64):
    a = _orig_qa(x, p, group)
    x32 = np.asarray(x, dtype=np.float64).astype(F32)
    if p.fmt == "int4":
        a.codes, a.scales = quant.int4_group_quant(x32, group)
    else:
        a.codes, a.scales = quant.nvfp4_quant(x32, p.s_gx)
    return a


def _smooth_act_divides(x, inv_lambda):
    return (np.asarray(x, dtype=np.float64).astype(F32) / np.asarray(inv_lambda, dtype=F32)).astype(F32)


MUTATIONS = {
    "residual_sign": (sq, "residual", _residual_plus),
    "smoothing_direction": (sq, "smooth_weight", _smooth_weight_divides),
    "int4_divisor": (quant, "int4_group_quant", _int4_by_8),
    "nvfp4_tensor_scale_constant": (quant, "nvfp4_tensor_scale", _tensor_scale_448),
    "bias_dropped": (sq, "forward", _forward_no_bias),
    "low_rank_input_unsmoothed": (sq, "quantize_act", _quantize_act_unsmoothed_u),
    "group_scale_index": (sq, "main_product", _main_product_swapped_group),
    "e2m1_ties_up": (formats, "e2m1_encode", _e2m1_tie_up),
    "dtype_rounding_truncates": (formats, "to_dtype", _to_dtype_truncate),
    "act_tensor_scale_from_unsmoothed_x": (sq, "act_tensor_scale", _act_tensor_scale_unsmoothed),
    "act_codes_from_unsmoothed_x": (sq, "quantize_act", _quantize_act_codes_unsmoothed),
    "act_smoothing_divides": (sq, "smooth_act", _smooth_act_divides),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    mod, attr, fn = MUTATIONS[name]
    monkeypatch.setattr(mod, attr, fn)
    assert _run_all_pins() > 0, f"no pin caught the planted mistake {name!r}"
