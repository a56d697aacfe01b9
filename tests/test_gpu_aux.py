"""The relative-MSE auxiliary loss (sq_rel_mse) against the oracle
(oracle/aux_loss.py), through the C ABI.

The loss is a float64 sum of non-negative terms in another order than the
oracle's: its relative error is below n * 2^-53 (n the element count), so
the test allows max(1e-12, n * 2^-52) relative.  The composed gradient is
G_in + lambda * 2 (Y_q - Y_fp) / den in float64, rounded once to bf16 on both
sides; the two float64 values differ only by the last bits of den, so the
bf16 results are equal except where the value sits on a rounding tie (at
most one bf16 ulp apart there; the count is printed)."""
import numpy as np
import pytest
import torch

import workloads
from oracle import aux_loss as A
from oracle import smoothquant as O
from tests.helpers import dev, dev_bf16, host_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import w8a8_smoothquant_int8_sq_b200 as m
    return m


def _check(sq, yfp, yq, G, lam, label):
    n = yfp.size
    loss_o, _, _ = A.rel_mse(yfp, yq)
    loss_g, G_out = sq.sq_rel_mse(dev_bf16(yfp), dev_bf16(yq), lam, G_in=dev_bf16(G) if G is not None else None)
    torch.cuda.synchronize()
    lg = float(loss_g.cpu()[0])
    tol = max(1e-12, n * 2.0 ** -52)
    assert abs(lg - loss_o) <= tol * max(abs(loss_o), 1e-300), f"{label}: loss {lg} vs {loss_o}"
    ties = 0
    if G is not None:
        go = A.add_aux_grad(G, yfp, yq, lam)
        gg = host_bf16_bits(G_out)
        diff = gg != go
        ties = int(diff.sum())
        if ties:
            a = O.widen_bf16(gg[diff]).astype(np.float64)
            b = O.widen_bf16(go[diff]).astype(np.float64)
            ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(b), 1e-300))) - 7)
            assert np.all(np.abs(a - b) <= ulp), f"{label}: G differs by more than one bf16 ulp"
            assert ties <= max(2, n // 100000), f"{label}: {ties} differing elements"
    print(f"\n[aux] {label}: loss {lg:.6e} (oracle {loss_o:.6e}), G elements on a tie: {ties}")
    return lg, G_out


def _rand(shape, seed, noise=0.05):
    rng = np.random.default_rng(seed)
    yfp = workloads.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))
    yq = workloads.f32_to_bf16_bits(O.widen_bf16(yfp) + rng.standard_normal(shape).astype(np.float32)
                                    * np.float32(noise))
    G = workloads.f32_to_bf16_bits((rng.standard_normal(shape) * 1e-3).astype(np.float32))
    return yfp, yq, G


@pytest.mark.parametrize("M,N", [(1, 8), (16, 256), (37, 100), (3, 5), (512, 4096), (2049, 11008)])
def test_random_shapes(sq, M, N):
    yfp, yq, G = _rand((M, N), M * 131 + N)
    _check(sq, yfp, yq, G, 0.25, f"{M}x{N}")
    _check(sq, yfp, yq, None, 0.0, f"{M}x{N} loss only")


def test_w8a8_layer_output(sq):
    """Y_q from the W8A8 forward on the mlp layer's seeded inputs, Y_fp the
    unquantised layer (float64, rounded once to bf16)."""
    wl = workloads.get("mlp")
    inp = workloads.make_inputs(wl)
    Xd, Wd = dev_bf16(inp["X"]), dev_bf16(inp["W"])
    bd = dev_bf16(inp["bias"]) if inp["bias"] is not None else None
    s = sq.sq_calibrate(dev_bf16(inp["C"]), Wd, wl.alpha_f32)
    Wq, ws = sq.sq_prepare_weight(Wd, s)
    yq = host_bf16_bits(sq.sq_forward(Xd, s, Wq, ws, bd))
    yfp = O.bf16_round(O.reference_linear_f64(inp["X"], inp["W"], inp["bias"]))
    G = workloads.random_bf16(yq.shape, seed=77, scale=1e-4)
    loss, _ = _check(sq, yfp, yq, G, 1.0, "mlp layer")
    assert 0.0 < loss < 1e-3  # W8A8 with smoothing: a small relative error


def test_in_place_and_special_cases(sq):
    yfp, yq, G = _rand((64, 200), 5)
    Gd = dev_bf16(G)
    _, G_sep = sq.sq_rel_mse(dev_bf16(yfp), dev_bf16(yq), 0.5, G_in=Gd)
    sq.sq_rel_mse(dev_bf16(yfp), dev_bf16(yq), 0.5, G_in=Gd, G_out=Gd)  # in place
    torch.cuda.synchronize()
    assert torch.equal(G_sep.view(torch.int16), Gd.view(torch.int16))
    # identical outputs: loss 0, G unchanged bit for bit
    loss, G_same = sq.sq_rel_mse(dev_bf16(yfp), dev_bf16(yfp), 3.0, G_in=dev_bf16(G))
    torch.cuda.synchronize()
    assert float(loss.cpu()[0]) == 0.0 and np.array_equal(host_bf16_bits(G_same), G)
    # Y_q = 0: loss exactly 1; Y_fp = 0: the 1e-24 floor
    loss, _ = sq.sq_rel_mse(dev_bf16(yfp), dev_bf16(np.zeros_like(yfp)))
    torch.cuda.synchronize()
    assert float(loss.cpu()[0]) == 1.0
    _check(sq, np.zeros((4, 8), np.uint16), workloads.f32_to_bf16_bits(np.full((4, 8), 2.0 ** -30, np.float32)),
           np.zeros((4, 8), np.uint16), 1e-30, "Y_fp = 0 (floor)")
