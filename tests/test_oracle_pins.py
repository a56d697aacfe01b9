"""The oracle against its pins, and planted mistakes that the pins must catch."""
import types

import numpy as np
import pytest

import oracle
from oracle import smoothquant as sq
from tests import oracle_pins as P

PRIMS = [
    "widen_bf16", "bf16_round", "column_max_abs", "smoothing_factor", "calibrate",
    "fold_and_quantize_weight", "quantize_activation", "int8_gemm", "dequant_epilogue",
    "reference_linear_f64", "quantization_error", "fold_and_quantize_weight_f64",
    "quantize_activation_f64", "near_tie_mask",
]


def real():
    return types.SimpleNamespace(**{n: getattr(sq, n) for n in PRIMS})


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(real())


def test_pins_on_proj_workload():
    o = real()
    P.pin_error_bound_and_smoothing_gain(o, names=("proj",))


# --------------------------------------------------------------- planted mistakes
def _widen(b):
    return sq.widen_bf16(b)


def mut_act_multiplies_by_s(X_bits, s):
    X = _widen(X_bits)
    Xt = X * np.asarray(s, np.float32)[None, :]
    m = np.maximum(np.abs(Xt).max(axis=1), sq.CLAMP_FLOOR)
    xs = m / np.float32(127)
    return np.clip(np.rint(Xt / xs[:, None]), -127, 127).astype(np.int8), xs


def mut_act_clamp_128(X_bits, s):
    X = _widen(X_bits)
    Xt = X / np.asarray(s, np.float32)[None, :]
    m = np.maximum(np.abs(Xt).max(axis=1), sq.CLAMP_FLOOR)
    xs = m / np.float32(128)
    return np.clip(np.rint(Xt / xs[:, None]), -128, 127).astype(np.int8), xs


def mut_act_half_up(X_bits, s):
    X = _widen(X_bits)
    Xt = X / np.asarray(s, np.float32)[None, :]
    m = np.maximum(np.abs(Xt).max(axis=1), sq.CLAMP_FLOOR)
    xs = m / np.float32(127)
    return np.clip(np.floor(Xt / xs[:, None] + np.float32(0.5)), -127, 127).astype(np.int8), xs


def mut_act_per_tensor(X_bits, s):
    X = _widen(X_bits)
    Xt = X / np.asarray(s, np.float32)[None, :]
    m = np.maximum(np.abs(Xt).max(), sq.CLAMP_FLOOR)
    xs = np.full(X.shape[0], m / np.float32(127), np.float32)
    return np.clip(np.rint(Xt / xs[:, None]), -127, 127).astype(np.int8), xs


def mut_w_divides_by_s(W_bits, s):
    W = _widen(W_bits)
    Wt = W / np.asarray(s, np.float32)[None, :]
    m = np.maximum(np.abs(Wt).max(axis=1), sq.CLAMP_FLOOR)
    ws = m / np.float32(127)
    return np.clip(np.rint(Wt / ws[:, None]), -127, 127).astype(np.int8), ws


def mut_w_scale_per_column(W_bits, s):
    W = _widen(W_bits)
    Wt = W * np.asarray(s, np.float32)[None, :]
    m = np.maximum(np.abs(Wt).max(axis=0), sq.CLAMP_FLOOR)       # wrong axis
    ws = m / np.float32(127)
    q = np.clip(np.rint(Wt / ws[None, :]), -127, 127).astype(np.int8)
    return q, np.resize(ws, W.shape[0]).astype(np.float32)


def mut_s_swapped_alpha(mx, mw, alpha):
    return sq.smoothing_factor(mx, mw, 1.0 - float(alpha))


def mut_s_no_floor(mx, mw, alpha):
    a = float(alpha)
    x = np.asarray(mx, np.float64)
    w = np.maximum(np.asarray(mw, np.float64), 1e-8)
    return (np.power(x, a) / np.power(w, 1.0 - a)).astype(np.float32)


def mut_calibrate_w_rows(C_bits, W_bits, alpha, mx_prev=None):
    C = _widen(C_bits)
    W = _widen(W_bits)
    mx = np.abs(C).max(axis=0)
    if mx_prev is not None:
        mx = np.maximum(mx, mx_prev)
    mw = np.resize(np.abs(W).max(axis=1), W.shape[1])              # per output row
    return sq.smoothing_factor(mx, mw, alpha), mx


def mut_gemm_no_transpose(Xq, Wq):
    return (Xq.astype(np.float64) @ Wq.astype(np.float64)[: Xq.shape[1]].reshape(Xq.shape[1], -1)).astype(np.int64)


def mut_gemm_int8_wrap(Xq, Wq):
    return (Xq.astype(np.int32) @ Wq.astype(np.int32).T).astype(np.int16).astype(np.int64)


def mut_epilogue_no_bias(acc, xs, ws, bias_bits=None):
    return sq.dequant_epilogue(acc, xs, ws, None)


def mut_epilogue_double_round(acc, xs, ws, bias_bits=None):
    y = np.asarray(acc, np.float64) * np.asarray(xs, np.float64)[:, None] * np.asarray(ws, np.float64)[None, :]
    if bias_bits is not None:
        y = y + sq.widen_bf16(bias_bits)[None, :]
    f = y.astype(np.float32)                                        # rounds twice
    u = f.view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def mut_bf16_truncate(y):
    f = np.asarray(y, np.float64).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


MUTATIONS = {
    "act_multiplies_by_s": {"quantize_activation": mut_act_multiplies_by_s},
    "act_clamp_128": {"quantize_activation": mut_act_clamp_128},
    "act_half_up": {"quantize_activation": mut_act_half_up},
    "act_per_tensor": {"quantize_activation": mut_act_per_tensor},
    "w_divides_by_s": {"fold_and_quantize_weight": mut_w_divides_by_s},
    "w_scale_per_column": {"fold_and_quantize_weight": mut_w_scale_per_column},
    "s_swapped_alpha": {"smoothing_factor": mut_s_swapped_alpha},
    "s_no_floor": {"smoothing_factor": mut_s_no_floor},
    "calibrate_w_rows": {"calibrate": mut_calibrate_w_rows},
    "gemm_no_transpose": {"int8_gemm": mut_gemm_no_transpose},
    "gemm_narrow_acc": {"int8_gemm": mut_gemm_int8_wrap},
    "epilogue_no_bias": {"dequant_epilogue": mut_epilogue_no_bias},
    "epilogue_double_round": {"dequant_epilogue": mut_epilogue_double_round},
    "bf16_truncate": {"bf16_round": mut_bf16_truncate},
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name):
    o = real()
    for k, v in MUTATIONS[name].items():
        setattr(o, k, v)
    caught = []
    for pin in P.ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(o)
        except Exception as e:  # AssertionError, or a shape error from a wrong axis
            caught.append((pin.__name__, type(e).__name__))
    assert caught, f"no pin caught the planted mistake {name}"
