"""The per-tensor oracle against its pins, and planted mistakes the pins catch."""
import types

import numpy as np
import pytest

from oracle import per_tensor as PT
from oracle import smoothquant as SQ
from tests import per_tensor_pins as P


def real():
    return types.SimpleNamespace(tensor_scale=PT.tensor_scale, quantize_per_tensor=PT.quantize_per_tensor,
                                 linear_per_tensor=PT.linear_per_tensor)


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(real())


# --------------------------------------------------------------- planted mistakes
def _x(x_bits):
    return SQ.widen_bf16(np.asarray(x_bits))


def _scale(x, qmax=127, floor=True):
    m = np.float32(np.max(np.abs(x))) if x.size else np.float32(0)
    sc = np.float32(m / np.float32(qmax))
    if floor and sc < PT.SCALE_FLOOR_PT:
        sc = np.float32(1.0)
    return sc


def mut_qmax_128(x_bits):
    x = _x(x_bits)
    sc = _scale(x, qmax=128)
    return np.clip(np.rint((x / sc).astype(np.float32)), -128, 127).astype(np.int8), sc


def mut_round_half_up(x_bits):
    x = _x(x_bits)
    sc = _scale(x)
    return np.clip(np.floor((x / sc).astype(np.float32) + 0.5), -128, 127).astype(np.int8), sc


def mut_per_row_scale(x_bits):
    x = _x(x_bits)
    sc = np.maximum(np.abs(x).max(axis=1, keepdims=True) / np.float32(127), np.float32(1e-8)).astype(np.float32)
    q = np.clip(np.rint((x / sc).astype(np.float32)), -128, 127).astype(np.int8)
    return q, np.float32(sc.max())


def mut_no_floor(x_bits):
    x = _x(x_bits)
    sc = _scale(x, floor=False)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = (x / sc).astype(np.float32)
    return np.clip(np.nan_to_num(np.rint(v)), -128, 127).astype(np.int8), sc


def mut_multiply_by_reciprocal(x_bits):
    x = _x(x_bits)
    sc = _scale(x)
    r = np.float32(np.float32(1.0) / sc)
    return np.clip(np.rint((x * r).astype(np.float32)), -128, 127).astype(np.int8), sc


def _with_quant(fn):
    def linear(X_bits, W_bits, bias_bits=None):
        Xq, sx = fn(X_bits)
        Wq, sw = fn(W_bits)
        acc = SQ.int8_gemm(Xq, Wq)
        xs = np.full(Xq.shape[0], sx, np.float32)
        ws = np.full(Wq.shape[0], sw, np.float32)
        return SQ.dequant_epilogue(acc, xs, ws, bias_bits), Xq, sx, Wq, sw
    return types.SimpleNamespace(tensor_scale=lambda x: fn(x)[1], quantize_per_tensor=fn, linear_per_tensor=linear)


MUTANTS = [mut_qmax_128, mut_round_half_up, mut_per_row_scale, mut_no_floor, mut_multiply_by_reciprocal]


@pytest.mark.parametrize("mut", MUTANTS, ids=lambda f: f.__name__)
def test_mutant_is_caught(mut):
    o = _with_quant(mut)
    caught = []
    for pin in P.ALL_PINS:
        try:
            pin(o)
        except (AssertionError, FloatingPointError, ValueError, ZeroDivisionError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches {mut.__name__}"
