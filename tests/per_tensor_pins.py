"""Pins of the per-tensor oracle (oracle/per_tensor.py) to facts outside it.

Page: "quantized_linear.py -- QuantizedLinear + apply_w8a8 (V5 -- bug fix
critico)", ``quantize_tensor`` and ``QuantizedLinear.forward``.  Each
``pin_*`` takes a namespace ``o`` with ``tensor_scale``,
``quantize_per_tensor`` and ``linear_per_tensor`` and raises AssertionError
when the oracle disagrees with:

* a worked example whose scale and codes are exact (ties included);
* the page's 1e-8 rule (zero and tiny tensors get scale 1);
* brute force in exact rational arithmetic with IEEE rounding written out;
* the range of the codes (the maximum maps to +-127; -128 never occurs) and
  the reconstruction bound |x - q*scale| <= scale/2;
* an integer triple loop for the product and exact rationals for the
  dequantised output;
* the purpose of the comparison: with outlier channels, one scale per tensor
  loses more accuracy than SmoothQuant's per-channel smoothing.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

import workloads
from oracle import smoothquant as SQ
from tests import exact
from tests.oracle_pins import bits

F32_FLOOR = Fraction(float(np.float32(1e-8)))


def pin_pt_worked_example(o):
    # max |x| = 254 -> scale = 254/127 = 2 exactly; x/2 is exact, ties to even
    x = bits([[254.0, 3.0, 5.0, 7.0], [-254.0, -3.0, 1.0, -1.5]])
    q, sc = o.quantize_per_tensor(x)
    assert sc == np.float32(2.0)
    assert q.tolist() == [[127, 2, 2, 4], [-127, -2, 0, -1]]


def pin_pt_scale_rule(o):
    z = bits([[0.0, 0.0], [0.0, 0.0]])
    q, sc = o.quantize_per_tensor(z)
    assert sc == np.float32(1.0) and not q.any()
    # max 2^-20 ~ 9.5e-7: max/127 ~ 7.5e-9 < 1e-8 -> scale 1, every code 0
    tiny = bits([[2.0 ** -20, -(2.0 ** -21)], [2.0 ** -22, 0.0]])
    q, sc = o.quantize_per_tensor(tiny)
    assert sc == np.float32(1.0) and not q.any()
    # max 2^-16 ~ 1.5e-5: max/127 ~ 1.2e-7 >= 1e-8 -> the ordinary scale
    small = bits([[2.0 ** -16, 2.0 ** -18]])
    q, sc = o.quantize_per_tensor(small)
    assert Fraction(float(sc)) == exact.to_f32(Fraction(2) ** -16 / 127)
    assert q.tolist() == [[127, exact.rne_int(exact.to_f32(Fraction(2) ** -18 / Fraction(float(sc))))]]


def _brute(vals):
    m = max(abs(v) for row in vals for v in row)
    sc = exact.to_f32(m / 127)
    if sc < F32_FLOOR:
        sc = Fraction(1)
    q = [[max(-128, min(127, exact.rne_int(exact.to_f32(v / sc)))) for v in row] for row in vals]
    return q, sc


def pin_pt_brute_force(o, trials=8):
    # 60 / fl(120/127) is a hair off 63.5: the correctly rounded quotient rounds
    # to 64, while 60 * fl(127/120) lands on the other side and gives 63
    fixed = bits([[120.0, 60.0, -60.0, 30.0]])
    q, sc = o.quantize_per_tensor(fixed)
    bq, bsc = _brute([[Fraction(float(v)) for v in r] for r in SQ.widen_bf16(fixed)])
    assert Fraction(float(sc)) == bsc and q.tolist() == bq, (q.tolist(), bq)
    for t in range(trials):
        x = workloads.random_bf16((3, 8), seed=500 + t, scale=2.0 + t, outlier_cols=[t % 8], outlier_scale=30.0)
        vals = [[Fraction(float(v)) for v in r] for r in SQ.widen_bf16(x)]
        q, sc = o.quantize_per_tensor(x)
        bq, bsc = _brute(vals)
        assert Fraction(float(sc)) == bsc, t
        assert q.tolist() == bq, t


def pin_pt_range_and_reconstruction(o):
    for name in ("tiny", "proj"):
        inp = workloads.make_inputs(workloads.get(name), ("X", "W"))
        for key in ("X", "W"):
            q, sc = o.quantize_per_tensor(inp[key])
            assert int(q.min()) >= -127 and int(q.max()) <= 127
            assert int(np.abs(q.astype(np.int32)).max()) == 127
            x = SQ.widen_bf16(inp[key]).astype(np.float64)
            err = np.abs(x - q.astype(np.float64) * float(sc))
            assert float(err.max()) <= float(sc) / 2 * (1 + 2.0 ** -20)


def pin_pt_linear_brute(o, seed=77):
    X = workloads.random_bf16((3, 16), seed=seed, scale=1.0, outlier_cols=[2], outlier_scale=20.0)
    W = workloads.random_bf16((5, 16), seed=seed + 1, scale=0.05)
    b = workloads.random_bf16((5,), seed=seed + 2, scale=0.01)
    Y, Xq, sx, Wq, sw = o.linear_per_tensor(X, W, b)
    bias = [Fraction(float(v)) for v in SQ.widen_bf16(b)]
    for m in range(3):
        for n in range(5):
            acc = sum(int(Xq[m, k]) * int(Wq[n, k]) for k in range(16))
            want = exact.to_bf16(acc * Fraction(float(sx)) * Fraction(float(sw)) + bias[n])
            assert Fraction(float(SQ.widen_bf16(Y[m:m + 1, n:n + 1])[0, 0])) == want, (m, n)


def pin_pt_less_accurate_than_smoothquant(o):
    wl = workloads.get("proj")
    inp = workloads.make_inputs(wl)
    Y_fp = SQ.reference_linear_f64(inp["X"], inp["W"], inp["bias"])
    Y_pt = o.linear_per_tensor(inp["X"], inp["W"], inp["bias"])[0]
    s, _ = SQ.calibrate(inp["C"], inp["W"], wl.alpha_f32)
    Wq, ws = SQ.fold_and_quantize_weight(inp["W"], s)
    Y_sq = SQ.forward(inp["X"], s, Wq, ws, inp["bias"])[0]
    e_pt = SQ.quantization_error(Y_fp, SQ.widen_bf16(Y_pt).astype(np.float64))
    e_sq = SQ.quantization_error(Y_fp, SQ.widen_bf16(Y_sq).astype(np.float64))
    assert e_pt > 2 * e_sq, (e_pt, e_sq)


ALL_PINS = [
    pin_pt_worked_example,
    pin_pt_scale_rule,
    pin_pt_brute_force,
    pin_pt_range_and_reconstruction,
    pin_pt_linear_brute,
    pin_pt_less_accurate_than_smoothquant,
]
