"""CPU oracle for the SmoothQuant W8A8 int8 linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
run this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use it.  It shares no code with the CUDA library
(its only shared dependency is the seeded input generator in ``workloads``,
which holds none of the method's arithmetic).

Source of truth: the page "w8a8_smoothquant.py -- W8A8 com SmoothQuant e
alpha APRENDIVEL (V5)" (module docstring "Algoritmo", functions
``_per_channel_max_abs``, ``calibrate_smoothquant``,
``quantize_per_channel_symmetric``, ``quantize_per_token_symmetric`` and the
methods ``SmoothQuantW8A8.calibrate`` / ``freeze_quantization`` / ``forward``
/ ``quantization_error``).

Precision, per step:

* Inputs are bf16 bit patterns, widened exactly.
* Max-abs reductions are exact (a max of exactly representable values).
* The smoothing factor s is evaluated in float64 (``**`` on float64) and
  rounded once to fp32 -- the page evaluates it with ``torch.pow`` on fp32
  tensors, which has no unique bit-level definition, so the mathematical
  value rounded once is the reading.
* The quantisation steps (fold ``W*s``, ``X/s``, ``max/127``, ``v/scale``,
  round-half-even, clamp to +-127) are the page's fp32 tensor operations.
  Each is a single IEEE-754 binary32 operation with one correctly rounded
  result, so the oracle performs exactly those operations in numpy float32,
  in the page's order.  This is where floating point decides an integer
  code; both sides decide it in this (the page's) precision.
* The int8 x int8 product is exact (int64 semantics).
* The dequantising epilogue ``acc * x_scale * w_scale + bias`` is evaluated in
  float64 and rounded once to bf16 (round-to-nearest-even).

An alternative float64 reading of the activation/weight quantisation
(``*_f64`` functions) computes X/s and W*s exactly and rounds only the stored
scales to fp32; it is used to report how far the page-precision codes are
from the ideal ones (the near-tie count).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "CLAMP_FLOOR",
    "QMAX",
    "widen_bf16",
    "bf16_round",
    "column_max_abs",
    "smoothing_factor",
    "calibrate",
    "fold_and_quantize_weight",
    "quantize_activation",
    "int8_gemm",
    "dequant_epilogue",
    "linear_int8",
    "forward",
    "reference_linear_f64",
    "quantization_error",
    "fold_and_quantize_weight_f64",
    "quantize_activation_f64",
    "near_tie_mask",
]

# The page clamps every max-abs (and s itself) at 1e-8 on fp32 tensors, so the
# floor is the fp32 value nearest to 1e-8.
CLAMP_FLOOR = np.float32(1e-8)
# n_bits = 8 symmetric: q in [-(2^7 - 1), 2^7 - 1]  (quantize_per_channel_symmetric)
QMAX = 127


# --------------------------------------------------------------------------- bf16
def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> exact fp32 values."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_round(y: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (nearest, ties to even) in ONE step.

    Returns the bf16 bit patterns (uint16).  Going through fp32 first would
    round twice; here the value is scaled by a power of two so that the bf16
    quantum becomes 1, rounded with ``rint`` (ties to even) and scaled back.
    bf16 keeps 8 significant bits; its smallest quantum is 2^-133.
    Values whose rounded magnitude exceeds the bf16 range become +-inf.
    """
    y = np.asarray(y, dtype=np.float64)
    _, e = np.frexp(y)                       # y = m * 2^e, 0.5 <= |m| < 1
    q = np.maximum(e - 8, -133)              # exponent of the bf16 quantum
    r = np.rint(np.ldexp(y, -q))             # exact scaling, then ties-to-even
    v = np.ldexp(r, q)                       # exactly a bf16 value (or too big)
    with np.errstate(over="ignore"):
        f = v.astype(np.float32)             # exact unless out of range -> inf
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# ------------------------------------------------------------------ calibration
def column_max_abs(A: np.ndarray) -> np.ndarray:
    """max_r |A[r, j]| per column j, exact, WITHOUT the 1e-8 floor.

    ``_per_channel_max_abs`` / the activation statistics of
    ``SmoothQuantW8A8.calibrate`` (reduction over all rows).
    """
    A = np.asarray(A)
    if A.shape[0] == 0:
        return np.zeros(A.shape[1], dtype=np.float32)
    return np.abs(A).max(axis=0).astype(np.float32)


def smoothing_factor(mx: np.ndarray, mw: np.ndarray, alpha: float) -> np.ndarray:
    """s_j = max( max(mx_j,1e-8)^alpha / max(mw_j,1e-8)^(1-alpha), 1e-8 ), fp32.

    ``calibrate_smoothquant``: max_x and max_w are clamped at 1e-8 before the
    powers, s is clamped after.  Evaluated in float64, rounded once to fp32.
    """
    a = float(alpha)
    x = np.maximum(np.asarray(mx, dtype=np.float64), float(CLAMP_FLOOR))
    w = np.maximum(np.asarray(mw, dtype=np.float64), float(CLAMP_FLOOR))
    s = np.power(x, a) / np.power(w, 1.0 - a)
    s = np.maximum(s, float(CLAMP_FLOOR))
    return s.astype(np.float32)


def calibrate(C_bits, W_bits, alpha: float, mx_prev=None):
    """Return ``(s, mx)``: the smoothing factor and the running activation max.

    ``SmoothQuantW8A8.calibrate`` keeps ``calib_max_abs = max(calib_max_abs,
    amax|X| per channel)`` across batches (starting from zeros) and
    ``freeze_quantization`` feeds that running max to ``calibrate_smoothquant``
    together with the weight's per-input-channel max (reduction over the
    output rows of W[d_out, d_in]).  ``C_bits`` may hold zero rows when
    ``mx_prev`` carries the statistics.
    """
    C = widen_bf16(C_bits)
    W = widen_bf16(W_bits)
    mx = column_max_abs(C) if C.shape[0] else np.zeros(W.shape[1], np.float32)
    if mx_prev is not None:
        mx = np.maximum(mx, np.asarray(mx_prev, dtype=np.float32))
    mw = column_max_abs(W)
    return smoothing_factor(mx, mw, alpha), mx


# ------------------------------------------------------------ quantisation (fp32)
def _rne_clamp_int8(v: np.ndarray) -> np.ndarray:
    # torch.round is round-half-to-even (numpy rint is the same rule);
    # clamp to the symmetric range [-127, 127].
    return np.clip(np.rint(v), -QMAX, QMAX).astype(np.int8)


def fold_and_quantize_weight(W_bits, s):
    """Fold s into W and quantise per output channel: ``(Wq[N,K] int8, w_scale[N] fp32)``.

    ``freeze_quantization``: ``W_smooth = weight_fp * s`` (s broadcast over the
    input-channel axis), then ``quantize_per_channel_symmetric(W_smooth,
    axis=0)``: ``scale = max(max_j |W_smooth[n, j]|, 1e-8) / 127`` and
    ``q = clamp(round(W_smooth / scale), -127, 127)``.  All in fp32.
    """
    W = widen_bf16(W_bits)
    s = np.asarray(s, dtype=np.float32)
    Wt = W * s[None, :]                                   # fp32 multiply
    m = np.maximum(np.abs(Wt).max(axis=1), CLAMP_FLOOR)   # per output row
    ws = m / np.float32(QMAX)                             # fp32 divide
    q = _rne_clamp_int8(Wt / ws[:, None])                 # fp32 divide, RNE, clamp
    return q, ws.astype(np.float32)


def quantize_activation(X_bits, s):
    """Dynamic per-token quantisation of X/s: ``(Xq[M,K] int8, x_scale[M] fp32)``.

    ``forward``: ``X_smooth = X / s``; ``quantize_per_token_symmetric``:
    ``scale = max(max_j |X_smooth[m, j]|, 1e-8) / 127`` per row and
    ``q = clamp(round(X_smooth / scale), -127, 127)``.  All in fp32.
    """
    X = widen_bf16(X_bits)
    s = np.asarray(s, dtype=np.float32)
    Xt = X / s[None, :]                                   # fp32 divide
    if Xt.shape[0] == 0:
        return np.zeros(Xt.shape, np.int8), np.zeros(0, np.float32)
    m = np.maximum(np.abs(Xt).max(axis=1), CLAMP_FLOOR)   # per token
    xs = m / np.float32(QMAX)
    q = _rne_clamp_int8(Xt / xs[:, None])
    return q, xs.astype(np.float32)


# ------------------------------------------------------------------- int8 GEMM
def int8_gemm(Xq: np.ndarray, Wq: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_j Xq[m, j] * Wq[n, j]  (exact, int64).

    The page's comment on ``forward`` names the hardware form
    INT8 x INT8 -> INT32.  The float64 BLAS product is exact here: every
    product and partial sum is an integer of magnitude <= 127^2 * K < 2^53.
    """
    K = Xq.shape[1]
    assert 127 * 127 * K < 2 ** 53
    acc = Xq.astype(np.float64) @ Wq.astype(np.float64).T
    return acc.astype(np.int64)


def dequant_epilogue(acc, x_scale, w_scale, bias_bits=None) -> np.ndarray:
    """Y = bf16( acc * x_scale[m] * w_scale[n] + bias[n] ), as bf16 bits.

    ``forward`` dequantises both operands and adds the bias after the
    product; with integer codes that is acc * x_scale * w_scale + bias.
    Evaluated in float64, rounded once to bf16.
    """
    y = np.asarray(acc, dtype=np.float64)
    y = y * np.asarray(x_scale, dtype=np.float64)[:, None]
    y = y * np.asarray(w_scale, dtype=np.float64)[None, :]
    if bias_bits is not None:
        y = y + widen_bf16(bias_bits).astype(np.float64)[None, :]
    return bf16_round(y)


def linear_int8(Xq, x_scale, Wq, w_scale, bias_bits=None) -> np.ndarray:
    """The int8 linear on already-quantised operands -> Y bf16 bits."""
    return dequant_epilogue(int8_gemm(Xq, Wq), x_scale, w_scale, bias_bits)


def forward(X_bits, s, Wq, w_scale, bias_bits=None):
    """Per-batch path: quantise X/s per token, int8 GEMM, dequant + bias.

    Returns ``(Y_bits, Xq, x_scale, acc)``.
    """
    Xq, xs = quantize_activation(X_bits, s)
    acc = int8_gemm(Xq, Wq)
    return dequant_epilogue(acc, xs, w_scale, bias_bits), Xq, xs, acc


# ------------------------------------------------------------- measurement aids
def reference_linear_f64(X_bits, W_bits, bias_bits=None) -> np.ndarray:
    """Y_fp = X W^T + b in float64 (the unquantised layer, ``F.linear``)."""
    X = widen_bf16(X_bits).astype(np.float64)
    W = widen_bf16(W_bits).astype(np.float64)
    y = X @ W.T
    if bias_bits is not None:
        y = y + widen_bf16(bias_bits).astype(np.float64)[None, :]
    return y


def quantization_error(Y_fp: np.ndarray, Y_q: np.ndarray) -> float:
    """||Y_fp - Y_q||_F / max(||Y_fp||_F, 1e-12)  (``quantization_error``)."""
    num = float(np.linalg.norm(np.asarray(Y_fp, np.float64) - np.asarray(Y_q, np.float64)))
    den = max(float(np.linalg.norm(np.asarray(Y_fp, np.float64))), 1e-12)
    return num / den


# ------------------------------------------------- float64 reading (comparison)
def fold_and_quantize_weight_f64(W_bits, s):
    """Same step with W*s exact in float64; only w_scale is rounded to fp32."""
    W = widen_bf16(W_bits).astype(np.float64)
    Wt = W * np.asarray(s, dtype=np.float64)[None, :]
    m = np.maximum(np.abs(Wt).max(axis=1), float(CLAMP_FLOOR))
    ws = (m / QMAX).astype(np.float32)
    v = Wt / ws.astype(np.float64)[:, None]
    return _rne_clamp_int8(v), ws, v


def quantize_activation_f64(X_bits, s):
    """Same step with X/s exact in float64; only x_scale is rounded to fp32."""
    X = widen_bf16(X_bits).astype(np.float64)
    Xt = X / np.asarray(s, dtype=np.float64)[None, :]
    m = np.maximum(np.abs(Xt).max(axis=1), float(CLAMP_FLOOR))
    xs = (m / QMAX).astype(np.float32)
    v = Xt / xs.astype(np.float64)[:, None]
    return _rne_clamp_int8(v), xs, v


def near_tie_mask(v: np.ndarray, rel: float = 1e-6) -> np.ndarray:
    """Elements whose pre-rounding value lies within ``rel`` (relative) of a
    rounding tie k + 1/2."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    frac = a - np.floor(a)
    return np.abs(frac - 0.5) <= rel * np.maximum(a, 1e-30)
