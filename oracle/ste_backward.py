"""CPU oracle for the backward pass of the learnable-alpha SmoothQuant layer.

TEST INFRASTRUCTURE ONLY, like ``oracle.smoothquant``: only ``tests/``,
``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` use it, and it
shares no code with the CUDA library.

Source of truth: the page "w8a8_smoothquant.py -- W8A8 com SmoothQuant e
alpha APRENDIVEL (V5)":

* ``SmoothQuantW8A8.alpha``: alpha = sigmoid(eta_alpha), eta_alpha the
  trainable parameter.
* ``SmoothQuantW8A8.forward`` in quantised mode: s is recomputed from the
  running activation max and the per-input-channel weight max with the
  trainable alpha (the weight max is detached, the activation max a buffer),
  clamped at 1e-8; X_smooth = X / s, W_smooth = weight_fp * s; both are
  fake-quantised with ``ste_quantize`` (per output channel for W, per token
  for X, scales computed from the smoothed tensors); Y = X_q_deq @
  W_q_deq^T + bias.
* ``STEQuantize.backward``: the incoming gradient passes through round and
  clamp unchanged, and the scale receives no gradient.

With G = dL/dY [M, N] the chain rule gives (derived here; the page leaves it
to autograd):

    dXs = G @ Wdq            (dL/dX_smooth, Wdq = Wq * w_scale)
    dWs = G^T @ Xdq          (dL/dW_smooth, Xdq = Xq * x_scale)
    dX  = dXs / s            (X_smooth = X / s)
    dW  = dWs * s            (W_smooth = weight_fp * s)
    db  = sum_m G[m, :]
    ds_j = sum_n dWs[n, j] W[n, j] - sum_m dXs[m, j] X[m, j] / s_j^2
    dalpha = sum_j ds_j * raw_j * (ln mx_j + ln mw_j) * [raw_j >= 1e-8]
    deta = alpha (1 - alpha) dalpha

where raw_j = mx_j^alpha / mw_j^(1-alpha) before the clamp, mx and mw
clamped at 1e-8 (the clamp's gradient passes where its input is at or above
the floor).

Readings:

* The forward values are those of the inference path: s, (Wq, w_scale) and
  (Xq, x_scale) come from ``oracle.smoothquant`` (the page's fp32 steps), so
  the training forward's output equals the W8A8 forward.  The page's own
  fp32 matmul of dequantised operands is the same value up to rounding.
* alpha is the fp32 value the forward uses: sigmoid(eta) evaluated in
  float64 and rounded once to fp32.  d alpha / d eta = alpha (1 - alpha) on
  that value, in float64.
* The dequantised operands are the exact products q * scale (the page
  rounds them to fp32; the difference is below 2^-24 relative).
* Everything after the codes and scales is evaluated in float64.
* The auxiliary relative-MSE loss of the page enters through G: its gradient
  with respect to Y_q is folded into G by ``oracle.aux_loss.add_aux_grad``.
"""
from __future__ import annotations

import math

import numpy as np

from oracle.smoothquant import (CLAMP_FLOOR, column_max_abs, fold_and_quantize_weight, quantize_activation,
                                smoothing_factor, widen_bf16)

__all__ = ["alpha_from_logit", "raw_smoothing", "ste_backward", "ste_error_scales"]


def alpha_from_logit(eta: float) -> np.float32:
    """alpha = sigmoid(eta) (``SmoothQuantW8A8.alpha``), float64 rounded once to fp32."""
    e = float(eta)
    if e >= 0:
        a = 1.0 / (1.0 + math.exp(-e))
    else:
        z = math.exp(e)
        a = z / (1.0 + z)
    return np.float32(a)


def raw_smoothing(mx, mw, alpha):
    """``(raw, mxc, mwc)``: mx^alpha / mw^(1-alpha) before the 1e-8 clamp of
    s, with mx and mw clamped at 1e-8 (float64)."""
    a = float(alpha)
    mxc = np.maximum(np.asarray(mx, dtype=np.float64), float(CLAMP_FLOOR))
    mwc = np.maximum(np.asarray(mw, dtype=np.float64), float(CLAMP_FLOOR))
    return np.power(mxc, a) / np.power(mwc, 1.0 - a), mxc, mwc


def ste_backward(G_bits, X_bits, W_bits, mx, alpha):
    """Gradients of the quantised-mode forward with respect to X, weight_fp,
    bias and eta_alpha, given G = dL/dY (bf16 bits [M, N]).

    ``mx`` is the running activation max (``calib_max_abs``), ``alpha`` the
    fp32 alpha of the forward.  Returns a dict with the forward's s, codes
    and scales and the float64 gradients ``dX [M,K]``, ``dW [N,K]``,
    ``db [N]``, ``ds [K]``, ``dalpha`` and ``deta``, plus the intermediate
    ``dXs``, ``dWs``.
    """
    G = widen_bf16(np.asarray(G_bits)).astype(np.float64)
    X = widen_bf16(np.asarray(X_bits)).astype(np.float64)
    W = widen_bf16(np.asarray(W_bits)).astype(np.float64)
    mw = column_max_abs(widen_bf16(np.asarray(W_bits)))           # detached weight max
    s = smoothing_factor(mx, mw, alpha)                            # forward's s (fp32)
    Wq, ws = fold_and_quantize_weight(W_bits, s)                   # per output channel
    Xq, xs = quantize_activation(X_bits, s)                        # per token
    s64 = s.astype(np.float64)
    Wdq = Wq.astype(np.float64) * ws.astype(np.float64)[:, None]   # W_q_deq
    Xdq = Xq.astype(np.float64) * xs.astype(np.float64)[:, None]   # X_q_deq
    # Y = Xdq @ Wdq^T + b; the straight-through estimator hands G to both operands
    dXs = G @ Wdq
    dWs = G.T @ Xdq
    dX = dXs / s64[None, :]
    dW = dWs * s64[None, :]
    db = G.sum(axis=0)
    ds = (dWs * W).sum(axis=0) - (dXs * X).sum(axis=0) / (s64 * s64)
    raw, mxc, mwc = raw_smoothing(mx, mw, alpha)
    passes = raw >= float(CLAMP_FLOOR)                             # clamp(min=1e-8) gradient mask
    dalpha = float(np.sum(np.where(passes, ds * raw * (np.log(mxc) + np.log(mwc)), 0.0)))
    a = float(alpha)
    deta = a * (1.0 - a) * dalpha
    return dict(s=s, mw=mw, Wq=Wq, w_scale=ws, Xq=Xq, x_scale=xs, dXs=dXs, dWs=dWs, dX=dX, dW=dW, db=db,
                ds=ds, raw=raw, passes=passes, dalpha=dalpha, deta=deta)


def ste_error_scales(G_bits, X_bits, W_bits, r):
    """Magnitudes that bound rounding errors of a finite-precision backward
    (float64): ``aXs = |G| @ |Wdq|``, ``aWs = |G|^T @ |Xdq|``, ``dW_q = W*s -
    Wdq`` and ``dX_q = X/s - Xdq`` (the quantisation errors), and
    ``aT[j] = sum_n aWs |dW_q| + sum_m aXs |dX_q|``; ``r`` is the dict of
    :func:`ste_backward`."""
    G = np.abs(widen_bf16(np.asarray(G_bits)).astype(np.float64))
    X = widen_bf16(np.asarray(X_bits)).astype(np.float64)
    W = widen_bf16(np.asarray(W_bits)).astype(np.float64)
    s64 = r["s"].astype(np.float64)
    Wdq = r["Wq"].astype(np.float64) * r["w_scale"].astype(np.float64)[:, None]
    Xdq = r["Xq"].astype(np.float64) * r["x_scale"].astype(np.float64)[:, None]
    aXs = G @ np.abs(Wdq)
    aWs = G.T @ np.abs(Xdq)
    dWq = W * s64[None, :] - Wdq
    dXq = X / s64[None, :] - Xdq
    aT = (aWs * np.abs(dWq)).sum(axis=0) + (aXs * np.abs(dXq)).sum(axis=0)
    return dict(aXs=aXs, aWs=aWs, dW_q=dWq, dX_q=dXq, aT=aT)
