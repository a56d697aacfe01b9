"""Seeded synthetic inputs for the SmoothQuant W8A8 linear layer.

This module only *makes data*: shapes, seeds, the outlier-channel set and the
bf16 encoding of the drawn values.  It holds none of the method's arithmetic
(no max-abs, no smoothing factor, no quantisation), so both the CPU oracle and
the CUDA path can take their inputs from it without sharing any computation.

Workloads follow the layer shapes that the SmoothQuant page's linear layer is
exercised on (``Y = X W^T`` with ``X`` activations carrying a few large input
channels and ``W`` near-uniform weights; w8a8_smoothquant.py, module docstring
"Algoritmo"):

  tiny     X[16 x 256]    W[256 x 256]     bias  alpha 0.5   5 outlier channels x40
  proj     X[512 x 4096]  W[4096 x 4096]   none  alpha 0.5   1% channels x50
  mlp      X[2048 x 4096] W[11008 x 4096]  bias  alpha 0.8   1% channels x60
  prefill  X[8192 x 8192] W[28672 x 8192]  none  alpha 0.5   0.5% channels x100
  decode   X[8 x 8192]    W[8192 x 8192]   none  alpha 0.5   1% channels x50

Recipe (identical on every machine):
  * generator: ``numpy.random.default_rng`` (PCG64), seed ``1000*index + stream``
    with stream 1 = X, 2 = calibration batch C, 3 = W, 4 = bias, 5 = outlier set;
  * outlier channels: ``round_half_even(frac*K)`` distinct columns drawn by
    stream 5 (an explicit count for the tiny layer); the calibration batch and
    the evaluated batch share this set;
  * values drawn in fp32 (X, C ~ N(0,1); W ~ N(0, w_std); bias ~ N(0, 0.01)),
    outlier columns of X and C multiplied by ``outlier_scale`` in fp32, then
    rounded to bf16 (round-to-nearest-even) -- the bf16 bit patterns are what
    both sides consume;
  * alpha is stored as the fp32 value the C ABI receives.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, Optional

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "get",
    "outlier_channels",
    "make_inputs",
    "f32_to_bf16_bits",
    "bf16_bits_to_f32",
    "random_bf16",
]


@dataclass(frozen=True)
class Workload:
    name: str
    index: int          # seed family: seed = 1000*index + stream
    M: int              # tokens (rows of X)
    N: int              # output features (rows of W)
    K: int              # input features (columns of X and W)
    R: int              # rows of the calibration batch
    outliers: int       # number of outlier input channels
    outlier_scale: float
    w_std: float
    has_bias: bool
    alpha_f32: float    # smoothing strength as the fp32 value passed to the ABI

    @property
    def int8_ops(self) -> int:
        """2*M*N*K multiply-adds counted as two operations each."""
        return 2 * self.M * self.N * self.K


def _alpha32(a: float) -> float:
    return float(np.float32(a))


def _count(frac: float, K: int) -> int:
    # round-half-even of frac*K (Python's round is half-even)
    return int(round(frac * K))


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in (
        Workload("tiny", 1, 16, 256, 256, 64, 5, 40.0, 0.02, True, _alpha32(0.5)),
        Workload("proj", 2, 512, 4096, 4096, 512, _count(0.01, 4096), 50.0, 0.02, False, _alpha32(0.5)),
        Workload("mlp", 3, 2048, 11008, 4096, 512, _count(0.01, 4096), 60.0, 0.015, True, _alpha32(0.8)),
        Workload("prefill", 4, 8192, 28672, 8192, 512, _count(0.005, 8192), 100.0, 0.01, False, _alpha32(0.5)),
        Workload("decode", 5, 8, 8192, 8192, 512, _count(0.01, 8192), 50.0, 0.02, False, _alpha32(0.5)),
    )
}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Encode fp32 values as bf16 bit patterns, round-to-nearest-even.

    Input formatting only (the generator draws fp32 and stores bf16).  NaN is
    not expected from the generator and is not special-cased.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Decode bf16 bit patterns to fp32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def outlier_channels(w: Workload) -> np.ndarray:
    rng = np.random.default_rng(1000 * w.index + 5)
    return np.sort(rng.choice(w.K, size=w.outliers, replace=False)).astype(np.int64)


def _activations(w: Workload, rows: int, stream: int) -> np.ndarray:
    rng = np.random.default_rng(1000 * w.index + stream)
    a = rng.standard_normal((rows, w.K), dtype=np.float32)
    cols = outlier_channels(w)
    a[:, cols] *= np.float32(w.outlier_scale)
    return f32_to_bf16_bits(a)


def make_inputs(w: Workload, parts=("X", "C", "W", "bias")) -> Dict[str, Optional[np.ndarray]]:
    """Return the requested bf16 bit arrays (uint16, row-major) of a workload.

    X[M,K], C[R,K] (calibration batch), W[N,K], bias[N] (None when the layer has
    no bias).  Each part has its own seed, so asking for a subset gives the same
    bytes as asking for all of them.
    """
    out: Dict[str, Optional[np.ndarray]] = {}
    for p in parts:
        if p == "X":
            out["X"] = _activations(w, w.M, 1)
        elif p == "C":
            out["C"] = _activations(w, w.R, 2)
        elif p == "W":
            rng = np.random.default_rng(1000 * w.index + 3)
            a = rng.standard_normal((w.N, w.K), dtype=np.float32)
            a *= np.float32(w.w_std)
            out["W"] = f32_to_bf16_bits(a)
        elif p == "bias":
            if w.has_bias:
                rng = np.random.default_rng(1000 * w.index + 4)
                a = rng.standard_normal(w.N, dtype=np.float32) * np.float32(0.01)
                out["bias"] = f32_to_bf16_bits(a)
            else:
                out["bias"] = None
        else:
            raise KeyError(p)
    return out


def random_bf16(shape, seed: int, scale: float = 1.0, outlier_cols=None, outlier_scale: float = 1.0) -> np.ndarray:
    """Ad-hoc seeded bf16 matrix for edge-case tests (ragged shapes and the like)."""
    rng = np.random.default_rng(seed)
    a = rng.standard_normal(shape, dtype=np.float32) * np.float32(scale)
    if outlier_cols is not None and len(outlier_cols):
        a[..., np.asarray(outlier_cols)] *= np.float32(outlier_scale)
    return f32_to_bf16_bits(a)
