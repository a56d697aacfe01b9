"""Pins of the CPU oracle to facts outside itself.

Each ``pin_*`` takes a namespace ``o`` with the oracle's primitives and raises
AssertionError when the oracle disagrees with what the SmoothQuant page and the
mathematics fix (page: "w8a8_smoothquant.py -- W8A8 com SmoothQuant e alpha
APRENDIVEL (V5)"):

* worked examples with exact ties (tests/golden/rne_ties.txt);
* brute force in exact rational arithmetic, with IEEE rounding written out
  (tests/exact.py), on tiny inputs;
* closed forms of the smoothing factor; the alpha = 0 and alpha = 1 invariants;
* the reconstruction bound of a symmetric quantiser (|x - q*scale| <= scale/2);
* the error bound stated in the module docstring ("Limite de erro") and the
  purpose of smoothing (less error than s = 1 when activations have outlier
  channels).

``test_oracle_pins.py`` runs every pin on the real oracle, and plants mistakes
in copies of it to check that some pin catches each one.
"""
from __future__ import annotations

import os
import random
from fractions import Fraction

import numpy as np

import workloads
from tests import exact

HERE = os.path.dirname(os.path.abspath(__file__))
F32_FLOOR = Fraction(float(np.float32(1e-8)))


def bits(vals):
    """Exact bf16 bit patterns of a list of numbers representable in bf16."""
    f = np.asarray(vals, dtype=np.float32)
    b = (f.view(np.uint32) >> 16).astype(np.uint16)
    back = (b.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(back, f), "value not exact in bf16"
    return b


def _fr(x) -> Fraction:
    return Fraction(float(x))


# ----------------------------------------------------------------- golden ties
def load_golden_ties():
    rows = []
    with open(os.path.join(HERE, "golden", "rne_ties.txt")) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            kind, s, vals, scale, codes = [p.strip() for p in line.split("|")]
            rows.append((kind, float(s), [float(v) for v in vals.split()], scale,
                         [int(c) for c in codes.split()]))
    return rows


def pin_golden_ties(o):
    for kind, s, vals, scale, codes in load_golden_ties():
        sv = np.full(len(vals), s, dtype=np.float32)
        b = bits(vals)[None, :]
        if kind == "act":
            q, sc = o.quantize_activation(b, sv)
        else:
            q, sc = o.fold_and_quantize_weight(b, sv)
        if scale == "FLOOR/127":
            want = exact.to_f32(F32_FLOOR / 127)
        else:
            want = Fraction(scale)
        assert _fr(sc[0]) == want, (kind, vals, sc[0], want)
        assert list(q[0].astype(int)) == codes, (kind, vals, list(q[0]), codes)


# ------------------------------------------------------ brute force, exact maths
def _brute_quant_rows(vals_rows, s, divide: bool):
    """The page's fp32 step sequence in exact arithmetic + explicit rounding.

    divide=True : activation path  x~ = fl(x / s_j)   (forward: X / s)
    divide=False: weight path      w~ = fl(w * s_j)   (freeze: weight_fp * s)
    then scale = fl(max(max|x~|, 1e-8) / 127), q = clamp(rne(fl(x~ / scale))).
    """
    codes, scales = [], []
    for row in vals_rows:
        t = []
        for j, x in enumerate(row):
            e = Fraction(x) / s[j] if divide else Fraction(x) * s[j]
            t.append(exact.to_f32(e))
        m = max(abs(v) for v in t)
        m = max(m, F32_FLOOR)
        sc = exact.to_f32(m / 127)
        q = [max(-127, min(127, exact.rne_int(exact.to_f32(v / sc)))) for v in t]
        codes.append(q)
        scales.append(sc)
    return codes, scales


def pin_brute_force_quant(o, seed=7, rows=4, cols=8, trials=6):
    rng = np.random.default_rng(seed)
    for trial in range(trials):
        X = workloads.random_bf16((rows, cols), seed=seed * 100 + trial, scale=3.0,
                                  outlier_cols=[trial % cols], outlier_scale=40.0)
        s32 = (rng.uniform(0.05, 20.0, cols)).astype(np.float32)
        if trial == 0:
            s32[:] = 1.0
        s_fr = [_fr(v) for v in s32]
        xv = [[_fr(v) for v in r] for r in o.widen_bf16(X)]
        for divide, fn in ((True, o.quantize_activation), (False, o.fold_and_quantize_weight)):
            q, sc = fn(X, s32)
            bq, bsc = _brute_quant_rows(xv, s_fr, divide)
            assert [list(map(int, r)) for r in q] == bq, ("codes", divide, trial)
            assert [_fr(v) for v in sc] == bsc, ("scales", divide, trial)


def pin_gemm_brute(o, seed=11):
    rng = np.random.default_rng(seed)
    for (M, N, K) in ((4, 8, 8), (3, 5, 16), (1, 1, 32)):
        Xq = rng.integers(-127, 128, (M, K), dtype=np.int64).astype(np.int8)
        Wq = rng.integers(-127, 128, (N, K), dtype=np.int64).astype(np.int8)
        acc = o.int8_gemm(Xq, Wq)
        assert acc.shape == (M, N)
        for m in range(M):
            for n in range(N):
                want = sum(int(Xq[m, j]) * int(Wq[n, j]) for j in range(K))
                assert int(acc[m, n]) == want, (M, N, K, m, n)
    # extreme magnitudes: |acc| = 127^2 * K at K = 8192
    K = 8192
    Xq = np.full((2, K), 127, np.int8)
    Xq[1] = -127
    Wq = np.full((1, K), 127, np.int8)
    acc = o.int8_gemm(Xq, Wq)
    assert int(acc[0, 0]) == 132128768 and int(acc[1, 0]) == -132128768


def pin_bf16_round(o, seed=3):
    # ties: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7 -> even (1.0);
    # 1 + 3*2^-8 halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even) -> 1 + 2^-6
    cases = [(1 + 2.0 ** -8, 1.0), (1 + 3 * 2.0 ** -8, 1 + 2.0 ** -6),
             (-(1 + 2.0 ** -8), -1.0), (1 + 2.0 ** -8 + 2.0 ** -30, 1 + 2.0 ** -7),
             (3.0, 3.0), (0.0, 0.0), (255.5, 256.0), (257.0, 256.0), (259.0, 260.0)]
    got = o.bf16_round(np.array([c[0] for c in cases]))
    want = bits([c[1] for c in cases])
    assert np.array_equal(got, want), (got, want)
    rnd = random.Random(seed)
    vals = [rnd.uniform(-1e4, 1e4) * 2.0 ** rnd.randint(-40, 40) for _ in range(400)]
    got = o.bf16_round(np.array(vals))
    for v, g in zip(vals, got):
        assert int(g) == exact.bf16_bits_of(exact.to_bf16(Fraction(v))), v


def pin_epilogue_brute(o, seed=5):
    rng = np.random.default_rng(seed)
    M, N = 3, 5
    acc = rng.integers(-132128768, 132128769, (M, N), dtype=np.int64)
    acc[:, :2] = rng.integers(-2000, 2001, (M, 2))   # products comparable to the bias
    xs = rng.uniform(1e-4, 1.0, M).astype(np.float32)
    ws = rng.uniform(1e-6, 1e-3, N).astype(np.float32)
    b = workloads.random_bf16((N,), seed=seed, scale=0.5)
    # one rounding, not two: acc*xs*ws = 1 + 2^-8 + 2^-24 lies just above the
    # bf16 tie 1 + 2^-8, so it rounds up to 1 + 2^-7 (bits 0x3F81); an fp32
    # intermediate would land on the tie and round down to 1.0.
    one = o.dequant_epilogue(np.array([[2 ** 24 + 2 ** 16 + 1]], np.int64),
                             np.array([2.0 ** -24], np.float32), np.array([1.0], np.float32))
    assert int(one[0, 0]) == 0x3F81, hex(int(one[0, 0]))
    y = o.dequant_epilogue(acc, xs, ws, b)
    y0 = o.dequant_epilogue(acc, xs, ws, None)
    bv = o.widen_bf16(b)
    for m in range(M):
        for n in range(N):
            e = Fraction(int(acc[m, n])) * _fr(xs[m]) * _fr(ws[n])
            assert int(y0[m, n]) == exact.bf16_bits_of(exact.to_bf16(e)), (m, n)
            e = e + _fr(bv[n])
            assert int(y[m, n]) == exact.bf16_bits_of(exact.to_bf16(e)), (m, n)


# ---------------------------------------------------------------- calibration
def pin_smoothing_closed_form(o):
    mx = np.array([4.0, 1.0, 16.0, 16.0], np.float32)
    mw = np.array([1.0, 4.0, 0.25, 0.0625], np.float32)
    # alpha = 0.25: s = mx^(1/4) / mw^(3/4)
    cases = {0.5: [2.0, 0.5, 8.0, 16.0], 1.0: [4.0, 1.0, 16.0, 16.0],
             0.0: [1.0, 0.25, 4.0, 16.0],
             0.25: [4 ** 0.25, 1.0 / 4 ** 0.75, 16 ** 0.25 / 0.25 ** 0.75, 2.0 * 8.0]}
    for a, want in cases.items():
        s = o.smoothing_factor(mx, mw, a)
        assert s.dtype == np.float32
        for got, w in zip(s, want):
            assert _fr(got) == exact.to_f32(Fraction(w)) or abs(float(got) / w - 1) < 2 ** -23, (a, got, w)
    # exact ones (powers of two) must be exact
    s = o.smoothing_factor(mx, mw, 0.5)
    assert list(map(float, s)) == [2.0, 0.5, 8.0, 16.0]
    # floors: mx = 0 with alpha = 1 gives s = the fp32 1e-8 floor; mw = 0 is clamped
    s = o.smoothing_factor(np.array([0.0], np.float32), np.array([5.0], np.float32), 1.0)
    assert _fr(s[0]) == F32_FLOOR
    s = o.smoothing_factor(np.array([1.0], np.float32), np.array([0.0], np.float32), 0.0)
    assert np.isfinite(s[0]) and _fr(s[0]) == exact.to_f32(1 / F32_FLOOR)


def pin_calibrate_stats(o, seed=21):
    R, N, K = 12, 7, 16
    C = workloads.random_bf16((R, K), seed=seed, outlier_cols=[3], outlier_scale=40.0)
    W = workloads.random_bf16((N, K), seed=seed + 1, scale=0.02)
    Cv, Wv = o.widen_bf16(C), o.widen_bf16(W)
    s, mx = o.calibrate(C, W, 0.5)
    for j in range(K):
        assert mx[j] == max(abs(Cv[r, j]) for r in range(R))
    # running max over two batches equals one pass over both
    s1, mx1 = o.calibrate(C[:5], W, 0.5)
    s2, mx2 = o.calibrate(C[5:], W, 0.5, mx_prev=mx1)
    assert np.array_equal(mx2, mx) and np.array_equal(s2, s)
    # the weight statistic is taken per INPUT channel (over output rows):
    # a large weight at (n=2, j=9) changes s_9 only.
    W2 = W.copy()
    W2[2, 9] = bits([30.0])[0]
    s3, _ = o.calibrate(C, W2, 0.5)
    diff = np.nonzero(s3 != s)[0]
    assert list(diff) == [9], diff
    assert s3[9] < s[9]
    # a large activation at column 4 raises s_4 only
    C2 = C.copy()
    C2[0, 4] = bits([512.0])[0]
    s4, _ = o.calibrate(C2, W, 0.5)
    assert list(np.nonzero(s4 != s)[0]) == [4] and s4[4] > s[4]


def pin_alpha_invariants(o, seed=31):
    R, N, K = 16, 24, 32
    C = workloads.random_bf16((R, K), seed=seed, outlier_cols=[1, 7], outlier_scale=50.0)
    W = workloads.random_bf16((N, K), seed=seed + 1, scale=0.02)
    W_other = workloads.random_bf16((N, K), seed=seed + 2, scale=0.5)
    C_other = workloads.random_bf16((R, K), seed=seed + 3)
    Cv, Wv = o.widen_bf16(C).astype(np.float64), o.widen_bf16(W).astype(np.float64)
    # alpha = 1: every calibration column of X/s has max exactly 1 (up to the
    # rounding of s), and s does not depend on W.
    s, _ = o.calibrate(C, W, 1.0)
    colmax = np.abs(Cv / s.astype(np.float64)).max(axis=0)
    assert np.all(np.abs(colmax - 1.0) <= 2 ** -23), colmax
    assert np.array_equal(o.calibrate(C, W_other, 1.0)[0], s)
    # alpha = 0: every column of W*s has max exactly 1 and s does not depend on C
    s, _ = o.calibrate(C, W, 0.0)
    colmax = np.abs(Wv * s.astype(np.float64)).max(axis=0)
    assert np.all(np.abs(colmax - 1.0) <= 2 ** -23), colmax
    assert np.array_equal(o.calibrate(C_other, W, 0.0)[0], s)


# ------------------------------------------------------- quantiser properties
def pin_reconstruction(o, seed=41):
    """|X/s - Xq*xs| <= xs/2 and |W*s - Wq*ws| <= ws/2 (symmetric quantiser
    with round-to-nearest), the row max maps to +-127, and codes stay in range."""
    M, N, K = 9, 10, 64
    X = workloads.random_bf16((M, K), seed=seed, outlier_cols=[5], outlier_scale=40.0)
    W = workloads.random_bf16((N, K), seed=seed + 1, scale=0.02)
    s = np.random.default_rng(seed).uniform(0.1, 10.0, K).astype(np.float32)
    Xv = o.widen_bf16(X).astype(np.float64)
    Wv = o.widen_bf16(W).astype(np.float64)
    s64 = s.astype(np.float64)
    Xq, xs = o.quantize_activation(X, s)
    Wq, ws = o.fold_and_quantize_weight(W, s)
    assert Xq.dtype == np.int8 and Wq.dtype == np.int8
    assert Xq.min() >= -127 and Wq.min() >= -127
    xt, wt = Xv / s64[None, :], Wv * s64[None, :]
    tol = 1 + 1e-6
    assert np.all(np.abs(xt - Xq * xs.astype(np.float64)[:, None]) <= 0.5 * xs[:, None] * tol + 1e-30)
    assert np.all(np.abs(wt - Wq * ws.astype(np.float64)[:, None]) <= 0.5 * ws[:, None] * tol + 1e-30)
    assert np.all(np.abs(Xq).max(axis=1) == 127) and np.all(np.abs(Wq).max(axis=1) == 127)
    # the scale is the row max over 127
    assert np.all(np.abs(xs * 127 / np.abs(xt).max(axis=1) - 1) < 1e-6)
    assert np.all(np.abs(ws * 127 / np.abs(wt).max(axis=1) - 1) < 1e-6)


def pin_zero_rows(o):
    K = 16
    X = np.zeros((2, K), np.uint16)
    X[1] = bits(np.arange(-8, 8) * 0.25)
    s = np.ones(K, np.float32)
    Xq, xs = o.quantize_activation(X, s)
    floor_scale = exact.to_f32(F32_FLOOR / 127)
    assert _fr(xs[0]) == floor_scale and not Xq[0].any()
    Wq, ws = o.fold_and_quantize_weight(X, s)
    assert _fr(ws[0]) == floor_scale and not Wq[0].any()
    # an all-zero weight column leaves s finite and positive
    C = workloads.random_bf16((4, K), seed=1)
    W = workloads.random_bf16((3, K), seed=2, scale=0.02)
    W[:, 6] = 0
    s, _ = o.calibrate(C, W, 0.5)
    assert np.all(np.isfinite(s)) and np.all(s > 0)


def _quantised_layer(o, wl, s):
    inp = workloads.make_inputs(wl)
    Wq, ws = o.fold_and_quantize_weight(inp["W"], s)
    Xq, xs = o.quantize_activation(inp["X"], s)
    acc = o.int8_gemm(Xq, Wq)
    yq = acc.astype(np.float64) * xs.astype(np.float64)[:, None] * ws.astype(np.float64)[None, :]
    yfp = o.reference_linear_f64(inp["X"], inp["W"], None)
    X = o.widen_bf16(inp["X"]).astype(np.float64)
    W = o.widen_bf16(inp["W"]).astype(np.float64)
    return yq, yfp, X, W, inp


def pin_error_bound_and_smoothing_gain(o, names=("tiny",)):
    """Docstring bound ||Y_fp - Y_q|| <= (eps_w + eps_x) ||W||_F ||X||_F with
    eps <= 2^-7, and smoothing beats s = 1 on outlier-channel activations."""
    for name in names:
        wl = workloads.get(name)
        inp = workloads.make_inputs(wl, ("C", "W"))
        s, _ = o.calibrate(inp["C"], inp["W"], wl.alpha_f32)
        yq, yfp, X, W, _ = _quantised_layer(o, wl, s)
        err = np.linalg.norm(yfp - yq)
        bound = 2 * 2.0 ** -7 * np.linalg.norm(W) * np.linalg.norm(X)
        assert err <= bound, (name, err, bound)
        rel = o.quantization_error(yfp, yq)
        yq1, _, _, _, _ = _quantised_layer(o, wl, np.ones(wl.K, np.float32))
        rel1 = o.quantization_error(yfp, yq1)
        assert rel < 0.05, (name, rel)
        assert rel < 0.8 * rel1, (name, rel, rel1)


def pin_f64_reading_close(o, names=("tiny",)):
    """The page-precision (fp32) quantiser and the exact float64 reading agree:
    scales within 2 fp32 ulp; codes equal except within 1e-6 of a tie."""
    for name in names:
        wl = workloads.get(name)
        inp = workloads.make_inputs(wl)
        s, _ = o.calibrate(inp["C"], inp["W"], wl.alpha_f32)
        for f32fn, f64fn, key in ((o.quantize_activation, o.quantize_activation_f64, "X"),
                                  (o.fold_and_quantize_weight, o.fold_and_quantize_weight_f64, "W")):
            q, sc = f32fn(inp[key], s)
            q64, sc64, v64 = f64fn(inp[key], s)
            ulp = np.spacing(sc64.astype(np.float32))
            assert np.all(np.abs(sc.astype(np.float64) - sc64) <= 2 * ulp), (name, key)
            diff = q != q64
            assert np.all(np.abs(q.astype(int) - q64.astype(int)) <= 1)
            assert np.all(o.near_tie_mask(v64[diff], 1e-6)), (name, key, int(diff.sum()))


ALL_PINS = [
    pin_golden_ties,
    pin_brute_force_quant,
    pin_gemm_brute,
    pin_bf16_round,
    pin_epilogue_brute,
    pin_smoothing_closed_form,
    pin_calibrate_stats,
    pin_alpha_invariants,
    pin_reconstruction,
    pin_zero_rows,
    pin_error_bound_and_smoothing_gain,
    pin_f64_reading_close,
]
