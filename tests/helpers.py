"""Helpers for the GPU parity tests: moving bf16 bit arrays to and from the
device, and the comparison rules of the parity bar.

Parity bar (the tolerance the target states, applied element by element):
  * s, x_scale, w_scale: within 2 fp32 ulp of the oracle;
  * int8 codes: bit-exact, except elements within 1e-6 (relative) of a rounding
    tie, which are counted and reported;
  * int32 accumulators: bit-exact for identical codes;
  * Y: within 1 bf16 ulp of the oracle's dequantised result, with an absolute
    floor of 2^-20 * (|acc*xs*ws| + |bias|) where the bias cancels the product
    (the fp32 epilogue's own rounding error relative to its terms).
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import smoothquant as O


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16).cuda()


def host_bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def ulp_f32_diff(a: np.ndarray, b: np.ndarray) -> int:
    """Largest distance in fp32 ulps (representation steps) between a and b."""
    a = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    b = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    return int(np.abs(a - b).max()) if a.size else 0


def assert_scales_close(got: np.ndarray, want: np.ndarray, what: str, max_ulp: int = 2) -> int:
    d = ulp_f32_diff(got, want)
    assert d <= max_ulp, f"{what}: {d} fp32 ulp apart (allowed {max_ulp})"
    return d


def assert_codes(got: np.ndarray, want: np.ndarray, v_pre: np.ndarray, what: str) -> int:
    """Codes equal except within 1e-6 of a tie; returns the number of such exceptions."""
    diff = got != want
    n = int(diff.sum())
    if n:
        assert np.all(np.abs(got[diff].astype(np.int32) - want[diff].astype(np.int32)) == 1), what
        assert np.all(O.near_tie_mask(v_pre[diff], 1e-6)), f"{what}: {n} code mismatches not at ties"
    return n


def bf16_values(bits: np.ndarray) -> np.ndarray:
    return O.widen_bf16(bits).astype(np.float64)


def assert_y_close(y_gpu_bits: np.ndarray, acc: np.ndarray, xs: np.ndarray, ws: np.ndarray,
                   bias_bits, what: str) -> float:
    """Y within 1 bf16 ulp of the oracle's dequantised value (see module doc)."""
    want_bits = O.dequant_epilogue(acc, xs, ws, bias_bits)
    yg = bf16_values(y_gpu_bits)
    yo = bf16_values(want_bits)
    prod = np.abs(acc.astype(np.float64) * xs.astype(np.float64)[:, None] * ws.astype(np.float64)[None, :])
    b = np.abs(bf16_values(bias_bits))[None, :] if bias_bits is not None else 0.0
    _, e = np.frexp(yo)
    ulp = np.ldexp(1.0, e - 8)  # bf16 ulp of |yo| in [2^(e-1), 2^e)
    ulp = np.where(yo == 0, np.ldexp(1.0, -133), ulp)
    tol = np.maximum(ulp, 2.0 ** -20 * (prod + b))
    err = np.abs(yg - yo)
    bad = err > tol
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outputs beyond 1 bf16 ulp; "
                           f"worst {float((err / tol).max()):.3f} x tol")
    return float((err / tol).max()) if err.size else 0.0
