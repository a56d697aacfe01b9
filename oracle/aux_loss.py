"""CPU oracle for the relative-MSE auxiliary loss of the learnable-alpha layer.

TEST INFRASTRUCTURE ONLY, like ``oracle.smoothquant``: only ``tests/``,
``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` use it, and it
shares no code with the CUDA library.

Source of truth: the page "w8a8_smoothquant.py -- W8A8 com SmoothQuant e
alpha APRENDIVEL (V5)", module docstring (V5): the auxiliary loss
||Y_fp - Y_q||_F^2 / ||Y_fp||_F^2 (relative MSE) is added to the total loss,
so that its gradient reaches eta_alpha; ``SmoothQuantW8A8.quantization_error``
reports the unsquared ratio, with the norm of Y_fp floored at 1e-12.

Readings (the page states the loss, not its gradient or its floor):

* Y_fp = F.linear(X, weight_fp, bias) is the unquantised layer and does not
  depend on alpha, so the loss reaches eta_alpha through Y_q alone:
      d aux / d Y_q = 2 (Y_q - Y_fp) / ||Y_fp||_F^2.
  The gradient through Y_fp (which would reach weight_fp) is not formed.
* The denominator is floored at (1e-12)^2 = 1e-24, the square of the page's
  floor on the norm.
* Y_fp and Y_q are the layer's bf16 outputs; everything is evaluated in
  float64.
* With a weight lambda, a caller's gradient G = dL/dY_q of the task loss
  becomes bf16(G + lambda * d aux / d Y_q), evaluated in float64 and rounded
  once to bf16 (nearest, ties to even) -- the G that the straight-through
  backward (``oracle.ste_backward``) takes.
"""
from __future__ import annotations

import numpy as np

from oracle.smoothquant import bf16_round, widen_bf16

DEN_FLOOR = 1e-24  # (1e-12)^2


def _f64(bits) -> np.ndarray:
    return widen_bf16(bits).astype(np.float64)


def rel_mse(Yfp_bits, Yq_bits):
    """(loss, num, den): num = sum (Y_fp - Y_q)^2, den = sum Y_fp^2, loss =
    num / max(den, 1e-24), all in float64."""
    yfp, yq = _f64(Yfp_bits), _f64(Yq_bits)
    d = yfp - yq
    num = float(np.sum(d * d))
    den = float(np.sum(yfp * yfp))
    return num / max(den, DEN_FLOOR), num, den


def rel_mse_grad(Yfp_bits, Yq_bits) -> np.ndarray:
    """d aux / d Y_q = 2 (Y_q - Y_fp) / max(||Y_fp||^2, 1e-24), float64."""
    yfp, yq = _f64(Yfp_bits), _f64(Yq_bits)
    _, _, den = rel_mse(Yfp_bits, Yq_bits)
    return 2.0 * (yq - yfp) / max(den, DEN_FLOOR)


def add_aux_grad(G_bits, Yfp_bits, Yq_bits, lam: float) -> np.ndarray:
    """bf16 bit patterns of G + lam * d aux / d Y_q (one rounding)."""
    g = _f64(G_bits) + float(lam) * rel_mse_grad(Yfp_bits, Yq_bits)
    return bf16_round(g)
