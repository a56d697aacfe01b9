"""Pins of the learnable-alpha backward oracle (oracle/ste_backward.py) to
facts outside it.

Page: "w8a8_smoothquant.py -- W8A8 com SmoothQuant e alpha APRENDIVEL (V5)",
``STEQuantize``, ``SmoothQuantW8A8.alpha`` and ``SmoothQuantW8A8.forward``.
Each ``pin_*`` takes the backward function ``bwd(G, X, W, mx, alpha)`` (the
signature of ``ste_backward``) and raises AssertionError when it disagrees
with:

* PyTorch autograd in float64 over the page's quantised-mode forward written
  out as tensor operations, with the straight-through estimator in its usual
  form ``v + (q*scale - v).detach()`` (a different computation of the same
  chain rule), including a column whose s sits on the 1e-8 clamp;
* the lossless case: when both quantisers are exact, the straight-through
  gradients are those of the unquantised product X W^T + b, which does not
  depend on s, so ds = 0 and d eta = 0;
* the algebraic form ds_j s_j = sum_n dWs (W s - Wdq) - sum_m dXs (X/s - Xdq)
  (the two ways of writing it agree whatever the codes are);
* linearity in G (the forward fixed, the gradients of G1 + G2 are the sums);
* sigmoid at points where its value is exact.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import workloads
from oracle import smoothquant as SQ
from oracle import ste_backward as STE
from tests.oracle_pins import bits


def _grads_autograd(G_bits, X_bits, W_bits, mx, eta, r):
    """Autograd of the page's forward; the codes and scales (which carry no
    gradient) are taken from ``r``."""
    f64 = torch.float64
    G = torch.tensor(SQ.widen_bf16(G_bits), dtype=f64)
    X = torch.tensor(SQ.widen_bf16(X_bits), dtype=f64, requires_grad=True)
    W = torch.tensor(SQ.widen_bf16(W_bits), dtype=f64, requires_grad=True)
    b = torch.zeros(W.shape[0], dtype=f64, requires_grad=True)
    e = torch.tensor(float(eta), dtype=f64, requires_grad=True)
    alpha = torch.sigmoid(e)
    max_x = torch.tensor(np.asarray(mx, np.float64)).clamp(min=float(SQ.CLAMP_FLOOR))
    max_w = W.detach().abs().amax(dim=0).clamp(min=float(SQ.CLAMP_FLOOR))
    s = (torch.pow(max_x, alpha) / torch.pow(max_w, 1.0 - alpha)).clamp(min=float(SQ.CLAMP_FLOOR))
    Xs = X / s
    Ws = W * s.unsqueeze(0)
    Wdq_val = torch.tensor(r["Wq"].astype(np.float64) * r["w_scale"].astype(np.float64)[:, None])
    Xdq_val = torch.tensor(r["Xq"].astype(np.float64) * r["x_scale"].astype(np.float64)[:, None])
    Wdq = Ws + (Wdq_val - Ws).detach()
    Xdq = Xs + (Xdq_val - Xs).detach()
    Y = Xdq @ Wdq.t() + b
    (Y * G).sum().backward()
    return X.grad.numpy(), W.grad.numpy(), b.grad.numpy(), float(e.grad)


def _close(a, b, rel, scale=None):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    sc = np.max(np.abs(b)) if scale is None else scale
    assert np.all(np.abs(a - b) <= rel * sc + 1e-300), float(np.max(np.abs(a - b)) / max(sc, 1e-300))


def pin_autograd(bwd, seed=61):
    M, N, K = 3, 5, 16
    X = workloads.random_bf16((M, K), seed=seed, scale=1.0, outlier_cols=[4], outlier_scale=30.0)
    Wv = SQ.widen_bf16(workloads.random_bf16((N, K), seed=seed + 1, scale=0.05))
    Wv[:, 9] *= 2.0 ** 40            # a weight column so large that s_9 hits the 1e-8 clamp
    W = bits(Wv)
    G = workloads.random_bf16((M, N), seed=seed + 2, scale=1.0)
    mx = SQ.column_max_abs(SQ.widen_bf16(X)).copy()
    mx[9] = 0.0
    eta = 0.3
    alpha = STE.alpha_from_logit(eta)
    r = bwd(G, X, W, mx, alpha)
    assert not bool(r["passes"][9]) and bool(r["passes"][:9].all()), "the clamped column is column 9 alone"
    dX, dW, db, deta = _grads_autograd(G, X, W, mx, eta, r)
    _close(r["dX"], dX, 1e-6)
    _close(r["dW"], dW, 1e-6)
    _close(r["db"], db, 1e-12)
    _close(r["deta"], deta, 1e-5, scale=max(abs(deta), 1e-12))


def _lossless_case(seed):
    """Integer-valued smoothed tensors with row maxima 127 and s = 2^c per
    column, so that both quantisers are exact (scales 1, codes = the values)."""
    rng = np.random.default_rng(seed)
    M, N, K = 4, 6, 8
    c = rng.integers(-2, 3, size=K)
    Wt = rng.integers(-126, 127, size=(N, K)).astype(np.float64)
    Xt = rng.integers(-126, 127, size=(M, K)).astype(np.float64)
    Wt[np.arange(N), rng.integers(0, K, size=N)] = 127.0 * rng.choice([-1.0, 1.0], size=N)
    Xt[np.arange(M), rng.integers(0, K, size=M)] = 127.0 * rng.choice([-1.0, 1.0], size=M)
    Wt[:, 0] = 127.0                     # every column's weight max is a known power-of-two multiple
    W = Wt / (2.0 ** c)[None, :]         # W * s = Wt exactly
    X = Xt * (2.0 ** c)[None, :]         # X / s = Xt exactly
    mw = np.abs(W).max(axis=0)
    mx = (mw * (4.0 ** c)).astype(np.float32)  # alpha = 1/2: s = sqrt(mx / mw) = 2^c
    G = workloads.random_bf16((M, N), seed=seed + 5, scale=1.0)
    return bits(X), bits(W), G, mx, c, Xt, Wt


def pin_lossless(bwd, seed=71):
    Xb, Wb, G, mx, c, Xt, Wt = _lossless_case(seed)
    r = bwd(G, Xb, Wb, mx, np.float32(0.5))
    assert np.array_equal(r["s"], (2.0 ** c).astype(np.float32)), "precondition: s = 2^c"
    assert np.array_equal(r["Wq"], Wt.astype(np.int8)) and np.all(r["w_scale"] == 1.0)
    assert np.array_equal(r["Xq"], Xt.astype(np.int8)) and np.all(r["x_scale"] == 1.0)
    Gv = SQ.widen_bf16(G).astype(np.float64)
    X = SQ.widen_bf16(Xb).astype(np.float64)
    W = SQ.widen_bf16(Wb).astype(np.float64)
    _close(r["dX"], Gv @ W, 1e-13)
    _close(r["dW"], Gv.T @ X, 1e-13)
    _close(r["db"], Gv.sum(axis=0), 1e-13)
    scale = float(np.abs(Gv).sum() * np.abs(X).max() * np.abs(W).max())
    assert np.all(np.abs(r["ds"] * r["s"]) <= 1e-12 * scale), "ds must vanish when quantisation is exact"
    assert abs(r["deta"]) <= 1e-11 * scale


def pin_error_form(bwd, seed=81):
    wl = workloads.get("tiny")
    inp = workloads.make_inputs(wl, ("X", "W", "C"))
    G = workloads.random_bf16((wl.M, wl.N), seed=seed, scale=1.0)
    mx = SQ.column_max_abs(SQ.widen_bf16(inp["C"]))
    r = bwd(G, inp["X"], inp["W"], mx, np.float32(wl.alpha_f32))
    e = STE.ste_error_scales(G, inp["X"], inp["W"], r)
    s = r["s"].astype(np.float64)
    T = (r["dWs"] * e["dW_q"]).sum(axis=0) - (r["dXs"] * e["dX_q"]).sum(axis=0)
    X = SQ.widen_bf16(inp["X"]).astype(np.float64)
    W = SQ.widen_bf16(inp["W"]).astype(np.float64)
    big = (np.abs(r["dWs"] * W).sum(axis=0) * s + np.abs(r["dXs"] * X).sum(axis=0) / s)
    assert np.all(np.abs(r["ds"] * s - T) <= 1e-12 * big)
    assert np.max(np.abs(T)) > 1e-6 * np.max(big), "the case must be lossy"


def pin_linear_in_G(bwd, seed=91):
    """With the forward fixed, every straight-through gradient is linear in
    G = dL/dY: the gradients of G1 + G2 are the sums of those of G1 and G2
    (G1, G2 small integers times 2^-10, so that G1 + G2 is exact in bf16)."""
    wl = workloads.get("tiny")
    inp = workloads.make_inputs(wl, ("X", "W", "C"))
    mx = SQ.column_max_abs(SQ.widen_bf16(inp["C"]))
    rng = np.random.default_rng(seed)
    g1 = rng.integers(-60, 61, size=(wl.M, wl.N)) * 2.0 ** -10
    g2 = rng.integers(-60, 61, size=(wl.M, wl.N)) * 2.0 ** -10
    a = np.float32(wl.alpha_f32)
    r1 = bwd(bits(g1), inp["X"], inp["W"], mx, a)
    r2 = bwd(bits(g2), inp["X"], inp["W"], mx, a)
    r12 = bwd(bits(g1 + g2), inp["X"], inp["W"], mx, a)
    for k in ("dX", "dW", "db", "ds"):
        _close(r12[k], r1[k] + r2[k], 1e-12, scale=np.max(np.abs(r1[k])) + np.max(np.abs(r2[k])))
    _close(r12["deta"], r1["deta"] + r2["deta"], 1e-9, scale=abs(r1["deta"]) + abs(r2["deta"]))


def pin_sigmoid():
    assert STE.alpha_from_logit(0.0) == np.float32(0.5)
    assert STE.alpha_from_logit(math.log(3.0)) == np.float32(0.75)
    assert STE.alpha_from_logit(-math.log(3.0)) == np.float32(0.25)
    assert STE.alpha_from_logit(-800.0) == np.float32(0.0)
    assert STE.alpha_from_logit(800.0) == np.float32(1.0)


ALL_PINS = [pin_autograd, pin_lossless, pin_error_form, pin_linear_in_G]
