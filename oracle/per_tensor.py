"""CPU oracle for the per-tensor symmetric W8A8 linear layer (accuracy
baseline beside SmoothQuant).

TEST INFRASTRUCTURE ONLY, like ``oracle.smoothquant``: only ``tests/``,
``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` use it, and it
shares no code with the CUDA library.

Source of truth: the page "quantized_linear.py -- QuantizedLinear + apply_w8a8
(V5 -- bug fix critico)", function ``quantize_tensor`` and
``QuantizedLinear.forward``:

* one scale for the whole tensor: ``scale = max|x| / qmax`` with qmax = 127,
  computed on fp32 tensors (one IEEE binary32 division of the exact maximum);
* a scale below 1e-8 is replaced by 1.0 (the comparison is made in the
  tensor's fp32, so the threshold is the fp32 value nearest 1e-8);
* codes ``round(x / scale)`` (fp32 division, round half to even as
  ``torch.round``) clamped to [qmin, qmax] = [-128, 127];
* ``QuantizedLinear.forward`` multiplies the dequantised tensors
  (``q * scale``): Y = (Xq Wq^T) * (scale_x * scale_w) + bias, computed here
  from the exact integer product in float64 and rounded once to bf16, the
  same reading as the SmoothQuant epilogue.

Since |x| <= max|x| and scale = fl(max|x| / 127), |x / scale| exceeds 127 by
at most one fp32 ulp, so the code -128 never occurs: the lower clamp bound of
the page is never reached.
"""
from __future__ import annotations

import numpy as np

from oracle.smoothquant import dequant_epilogue, int8_gemm, widen_bf16

__all__ = ["QMIN_PT", "QMAX_PT", "SCALE_FLOOR_PT", "tensor_scale", "quantize_per_tensor", "linear_per_tensor"]

QMIN_PT = -128
QMAX_PT = 127
# the page compares an fp32 scale with 1e-8: the threshold is fp32(1e-8)
SCALE_FLOOR_PT = np.float32(1e-8)


def tensor_scale(x_bits) -> np.float32:
    """``scale = max|x| / 127`` in fp32, replaced by 1.0 below 1e-8."""
    x = widen_bf16(np.asarray(x_bits))
    m = np.float32(np.max(np.abs(x))) if x.size else np.float32(0.0)
    scale = np.float32(m / np.float32(QMAX_PT))
    if scale < SCALE_FLOOR_PT:
        scale = np.float32(1.0)
    return scale


def quantize_per_tensor(x_bits):
    """``(q int8 [same shape], scale fp32)``: ``q = clamp(rne(fl(x / scale)), -128, 127)``."""
    x = widen_bf16(np.asarray(x_bits))
    scale = tensor_scale(x_bits)
    v = (x / scale).astype(np.float32)  # one binary32 division per element
    q = np.clip(np.rint(v), QMIN_PT, QMAX_PT).astype(np.int8)
    return q, scale


def linear_per_tensor(X_bits, W_bits, bias_bits=None):
    """``(Y bf16 bits, Xq, scale_x, Wq, scale_w)`` of QuantizedLinear.forward
    with the int8 product made exact."""
    Xq, sx = quantize_per_tensor(X_bits)
    Wq, sw = quantize_per_tensor(W_bits)
    acc = int8_gemm(Xq, Wq)
    xs = np.full(Xq.shape[0], sx, dtype=np.float32)
    ws = np.full(Wq.shape[0], sw, dtype=np.float32)
    return dequant_epilogue(acc, xs, ws, bias_bits), Xq, sx, Wq, sw
