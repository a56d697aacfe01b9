"""Pins of the auxiliary-loss oracle (oracle/aux_loss.py) to facts outside it.

Page: "w8a8_smoothquant.py -- W8A8 com SmoothQuant e alpha APRENDIVEL (V5)",
module docstring (the relative-MSE loss ||Y_fp - Y_q||^2 / ||Y_fp||^2) and
``SmoothQuantW8A8.quantization_error`` (the unsquared ratio, norm floored at
1e-12).  Each ``pin_*`` takes the oracle's three functions ``(loss, grad,
add)`` -- the signatures of ``rel_mse``, ``rel_mse_grad`` and
``add_aux_grad`` -- and raises AssertionError when they disagree with:

* closed forms: Y_q = Y_fp gives 0, Y_q = 0 gives 1, Y_q = c Y_fp (c a power
  of two, so every value is exact) gives (1 - c)^2;
* the page's own metric: the loss is ``quantization_error`` squared (a
  separate code path, norms by ``numpy.linalg.norm``);
* scale invariance: the loss of (k Y_fp, k Y_q) equals the loss of
  (Y_fp, Y_q) for k a power of two;
* PyTorch autograd in float64 of the loss written as tensor operations (the
  derivative computed by a different method than the oracle's formula);
* the floor: Y_fp = 0 divides by 1e-24 = (1e-12)^2;
* the composed gradient: G + lambda * grad rounded once to bf16, lambda = 0
  leaving G unchanged bit for bit.
"""
from __future__ import annotations

import numpy as np
import torch

import workloads
from oracle import smoothquant as SQ


def _bits(x: np.ndarray) -> np.ndarray:
    return workloads.f32_to_bf16_bits(np.asarray(x, np.float32))


def _case(seed=0, shape=(6, 10), scale=1.0):
    rng = np.random.default_rng(seed)
    yfp = _bits(rng.standard_normal(shape) * scale)
    yq = _bits(SQ.widen_bf16(yfp) + rng.standard_normal(shape).astype(np.float32) * np.float32(0.05 * scale))
    return yfp, yq


def pin_closed_forms(loss, grad, add):
    yfp, _ = _case(1)
    assert loss(yfp, yfp)[0] == 0.0
    assert not np.any(grad(yfp, yfp))
    assert loss(yfp, np.zeros_like(yfp))[0] == 1.0
    for c in (0.5, 2.0, 0.25, -1.0):
        yq = _bits(SQ.widen_bf16(yfp) * np.float32(c))
        assert loss(yfp, yq)[0] == (1.0 - c) ** 2, c


def pin_page_metric(loss, grad, add):
    yfp, yq = _case(2, (16, 33))
    e = SQ.quantization_error(SQ.widen_bf16(yfp).astype(np.float64), SQ.widen_bf16(yq).astype(np.float64))
    assert abs(loss(yfp, yq)[0] - e * e) <= 1e-14 * e * e


def pin_scale_invariance(loss, grad, add):
    yfp, yq = _case(3, (8, 12))
    for k in (4.0, 0.125):
        l1 = loss(yfp, yq)[0]
        l2 = loss(_bits(SQ.widen_bf16(yfp) * np.float32(k)), _bits(SQ.widen_bf16(yq) * np.float32(k)))[0]
        assert abs(l1 - l2) <= 1e-15 * l1


def pin_autograd(loss, grad, add):
    yfp, yq = _case(4, (5, 7))
    tf = torch.tensor(SQ.widen_bf16(yfp), dtype=torch.float64)
    tq = torch.tensor(SQ.widen_bf16(yq), dtype=torch.float64, requires_grad=True)
    aux = ((tf - tq) ** 2).sum() / (tf ** 2).sum()
    aux.backward()
    assert abs(aux.item() - loss(yfp, yq)[0]) <= 1e-14 * aux.item()
    np.testing.assert_allclose(grad(yfp, yq), tq.grad.numpy(), rtol=1e-12, atol=0)


def pin_floor(loss, grad, add):
    yfp = np.zeros((3, 4), np.uint16)
    yq = _bits(np.full((3, 4), 2.0 ** -30, np.float32))
    num = 12 * 2.0 ** -60
    assert loss(yfp, yq)[0] == num / 1e-24
    np.testing.assert_array_equal(grad(yfp, yq), np.full((3, 4), 2.0 * 2.0 ** -30 / 1e-24))


def pin_composed(loss, grad, add):
    yfp, yq = _case(5, (9, 11))
    rng = np.random.default_rng(6)
    G = _bits(rng.standard_normal((9, 11)) * 1e-3)
    assert np.array_equal(add(G, yfp, yq, 0.0), G)
    lam = 0.3
    expect = SQ.widen_bf16(G).astype(np.float64) + lam * grad(yfp, yq)
    got = SQ.widen_bf16(add(G, yfp, yq, lam)).astype(np.float64)
    # one rounding to bf16: within half a bf16 ulp of the exact value
    ulp = np.exp2(np.floor(np.log2(np.abs(expect))) - 7)
    assert np.all(np.abs(got - expect) <= 0.5 * ulp)


ALL_PINS = [pin_closed_forms, pin_page_metric, pin_scale_invariance, pin_autograd, pin_floor, pin_composed]
