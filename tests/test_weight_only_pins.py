"""Pins of the weight-only oracle (oracle/weight_only.py) to facts outside it:
exact rational brute force on small inputs, the dequantised-weight form of the
torchao page's formula, and an all-ones case with a closed form."""
from fractions import Fraction

import numpy as np

import workloads
from oracle import smoothquant as SQ
from oracle import weight_only as WO
from tests import exact
from tests.oracle_pins import bits


def test_brute_force_small():
    X = workloads.random_bf16((3, 32), seed=901, scale=2.0, outlier_cols=[5], outlier_scale=40.0)
    W = workloads.random_bf16((6, 32), seed=902, scale=0.05)
    b = workloads.random_bf16((6,), seed=903, scale=0.01)
    Wq, ws = SQ.fold_and_quantize_weight(W, np.ones(32, np.float32))
    Y, y = WO.weight_only_linear(X, Wq, ws, b)
    xv = SQ.widen_bf16(X)
    bv = SQ.widen_bf16(b)
    for m in range(3):
        for n in range(6):
            acc = sum(Fraction(float(xv[m, k])) * int(Wq[n, k]) for k in range(32))
            e = acc * Fraction(float(ws[n])) + Fraction(float(bv[n]))
            assert abs(Fraction(float(y[m, n])) - e) <= abs(e) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 80)
            assert int(Y[m, n]) == exact.bf16_bits_of(exact.to_bf16(e)), (m, n)


def test_matches_dequantised_weight_form():
    """The page dequantises nothing explicitly; X @ (Wq * w_scale)^T + b is the
    same number (up to float64 rounding)."""
    wl = workloads.get("tiny")
    inp = workloads.make_inputs(wl, ("X", "W", "bias"))
    Wq, ws = SQ.fold_and_quantize_weight(inp["W"], np.ones(wl.K, np.float32))
    _, y = WO.weight_only_linear(inp["X"], Wq, ws, inp["bias"])
    Wdq = Wq.astype(np.float64) * ws.astype(np.float64)[:, None]
    y2 = SQ.widen_bf16(inp["X"]).astype(np.float64) @ Wdq.T + SQ.widen_bf16(inp["bias"]).astype(np.float64)
    assert np.allclose(y, y2, rtol=1e-12, atol=1e-12)


def test_closed_form_ones():
    # x = 1 everywhere, every code 127, scale 2^-7: y = K * 127 * 2^-7 exactly
    K = 64
    X = bits(np.ones((2, K)))
    Wq = np.full((3, K), 127, np.int8)
    ws = np.full(3, 2.0 ** -7, np.float32)
    Y, y = WO.weight_only_linear(X, Wq, ws)
    assert np.all(y == K * 127 * 2.0 ** -7)
    assert np.all(SQ.widen_bf16(Y) == np.float32(K * 127 * 2.0 ** -7))
    S = WO.abs_product_sum(X, -Wq, ws)
    assert np.all(S == K * 127 * 2.0 ** -7)


# --------------------------------------------------------------- planted mistakes
import pytest  # noqa: E402


def _mut(kind):
    def linear(X_bits, Wq, w_scale, bias_bits=None):
        X = SQ.widen_bf16(np.asarray(X_bits)).astype(np.float64)
        Q = np.asarray(Wq).astype(np.float64)
        ws = np.asarray(w_scale, dtype=np.float64)
        if kind == "scale_per_input_channel":
            y = (X * np.resize(ws, X.shape[1])[None, :]) @ Q.T
        elif kind == "transposed_codes":
            y = (X @ Q[:, ::-1].T) * ws[None, :]
        elif kind == "dropped_bias":
            y = (X @ Q.T) * ws[None, :]
            return SQ.bf16_round(y), y
        elif kind == "bf16_per_product":
            y = np.zeros((X.shape[0], Q.shape[0]))
            for k in range(X.shape[1]):
                y = SQ.widen_bf16(SQ.bf16_round(y + np.outer(X[:, k], Q[:, k]))).astype(np.float64)
            y = y * ws[None, :]
        else:
            y = (X @ Q.T) * ws[None, :]
        if bias_bits is not None:
            y = y + SQ.widen_bf16(np.asarray(bias_bits)).astype(np.float64)[None, :]
        return SQ.bf16_round(y), y
    return linear


@pytest.mark.parametrize("kind", ["scale_per_input_channel", "transposed_codes", "dropped_bias", "bf16_per_product"])
def test_mutant_is_caught(kind, monkeypatch):
    caught = []
    for pin in (test_brute_force_small, test_matches_dequantised_weight_form, test_closed_form_ones):
        monkeypatch.setattr(WO, "weight_only_linear", _mut(kind))
        try:
            pin()
        except AssertionError:
            caught.append(pin.__name__)
        finally:
            monkeypatch.undo()
    assert caught, f"no pin catches {kind}"
