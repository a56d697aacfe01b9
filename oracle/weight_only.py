"""CPU oracle for the int8 weight-only linear layer (a decode comparison point
beside the W8A8 path).

TEST INFRASTRUCTURE ONLY, like ``oracle.smoothquant``: only ``tests/``,
``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` use it, and it
shares no code with the CUDA library.

Source of truth: the torchao page (``Int8WeightOnlyQuantizedLinearWeight``,
its ``_quantized_op``): the activations stay in floating point, the product
is taken against the int8 weight codes and then multiplied by the
per-output-channel weight scale, and the bias is added:
``y[m][n] = (sum_k x[m][k] * Wq[n][k]) * w_scale[n] + bias[n]``.

Readings:

* The weight is quantised per output channel, symmetric to +-127, by the
  SmoothQuant page's ``quantize_per_channel_symmetric`` (``sq_prepare_weight``
  with s = 1): the quantiser torchao's ``from_float`` calls is imported from a
  module the pages do not print.
* The page computes the product in the activations' dtype (bf16) and rounds
  after each operation; the reading here is the exact value of the formula
  above rounded once to bf16.  The oracle sums in float64 (the products of a
  bf16 value and an int8 code are exact; the float64 sum's error is ~1e-16
  relative, far below a bf16 ulp) and returns that float64 value beside the
  rounded one, so a test can bound an fp32-accumulating kernel's error.
"""
from __future__ import annotations

import numpy as np

from oracle.smoothquant import bf16_round, widen_bf16

__all__ = ["weight_only_linear", "abs_product_sum"]


def weight_only_linear(X_bits, Wq, w_scale, bias_bits=None):
    """``(Y bf16 bits [M,N], y float64 [M,N])`` of the weight-only product."""
    X = widen_bf16(np.asarray(X_bits)).astype(np.float64)
    Q = np.asarray(Wq).astype(np.float64)
    y = (X @ Q.T) * np.asarray(w_scale, dtype=np.float64)[None, :]
    if bias_bits is not None:
        y = y + widen_bf16(np.asarray(bias_bits)).astype(np.float64)[None, :]
    return bf16_round(y), y


def abs_product_sum(X_bits, Wq, w_scale):
    """``sum_k |x[m][k] * Wq[n][k]| * w_scale[n]``: the scale of a summation
    error bound (float64, [M,N])."""
    X = np.abs(widen_bf16(np.asarray(X_bits)).astype(np.float64))
    Q = np.abs(np.asarray(Wq).astype(np.float64))
    return (X @ Q.T) * np.asarray(w_scale, dtype=np.float64)[None, :]
