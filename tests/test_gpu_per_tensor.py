"""The per-tensor W8A8 baseline on the GPU (through the C ABI) against its CPU
oracle: scales and codes bit for bit, Y within one bf16 ulp, and -- the point
of the baseline -- a larger error than SmoothQuant on the outlier workloads."""
import numpy as np
import pytest
import torch

import workloads
from oracle import per_tensor as PT
from oracle import smoothquant as O
from tests.helpers import assert_y_close, dev_bf16, host, host_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import w8a8_smoothquant_int8_sq_b200 as m
    return m


def _check_quant(sq, A_bits, label):
    Aq_g, sc_g = sq.sq_quantize_per_tensor(dev_bf16(A_bits))
    torch.cuda.synchronize()
    Aq_o, sc_o = PT.quantize_per_tensor(A_bits)
    sc_h = host(sc_g)
    assert np.all(sc_h == sc_o), f"{label}: scale {sc_h[:2]} != {sc_o}"
    assert np.array_equal(host(Aq_g), Aq_o), f"{label}: codes differ"
    return Aq_g, sc_g


@pytest.mark.parametrize("name", ["tiny", "proj", "mlp", "decode"])
def test_per_tensor_linear_parity(sq, name):
    wl = workloads.get(name)
    inp = workloads.make_inputs(wl)
    Xq, xs = _check_quant(sq, inp["X"], f"{name} X")
    Wq, ws = _check_quant(sq, inp["W"], f"{name} W")
    b = dev_bf16(inp["bias"]) if inp["bias"] is not None else None
    Y = sq.sq_linear(Xq, xs, Wq, ws, b)
    torch.cuda.synchronize()
    acc = O.int8_gemm(host(Xq), host(Wq))
    ratio = assert_y_close(host_bf16_bits(Y), acc, host(xs), host(ws), inp["bias"], f"{name}: per-tensor Y")
    print(f"\n[per-tensor parity] {name}: y_tol_ratio {ratio}")


@pytest.mark.parametrize("rows,K", [(1, 16), (3, 48), (130, 4112), (7, 16384)])
def test_per_tensor_ragged(sq, rows, K):
    A = workloads.random_bf16((rows, K), seed=rows * 31 + K, scale=3.0, outlier_cols=[K // 3], outlier_scale=60.0)
    _check_quant(sq, A, f"{rows}x{K}")


def test_per_tensor_zero_and_tiny(sq):
    Z = np.zeros((4, 64), np.uint16)
    Aq, sc = _check_quant(sq, Z, "zeros")
    assert float(host(sc)[0]) == 1.0 and not host(Aq).any()
    T = workloads.random_bf16((4, 64), seed=3, scale=1e-7)   # max / 127 below 1e-8: scale 1
    Aq, sc = _check_quant(sq, T, "tiny values")
    assert float(host(sc)[0]) == 1.0


def test_per_tensor_full_size_weight_sampled(sq):
    wl = workloads.get("prefill")
    W = workloads.make_inputs(wl, ("W",))["W"]
    Wq, ws = sq.sq_quantize_per_tensor(dev_bf16(W))
    torch.cuda.synchronize()
    sc_o = PT.tensor_scale(W)
    assert np.all(host(ws) == sc_o)
    rows = np.sort(np.random.default_rng(9).choice(wl.N, 64, replace=False))
    x = O.widen_bf16(W[rows])
    want = np.clip(np.rint((x / sc_o).astype(np.float32)), -128, 127).astype(np.int8)
    assert np.array_equal(host(Wq[torch.as_tensor(rows, device="cuda")]), want)


def test_per_tensor_is_less_accurate_than_smoothquant(sq):
    for name in ("proj", "mlp"):
        wl = workloads.get(name)
        inp = workloads.make_inputs(wl)
        Xd, Wd = dev_bf16(inp["X"]), dev_bf16(inp["W"])
        b = dev_bf16(inp["bias"]) if inp["bias"] is not None else None
        Y_fp = O.reference_linear_f64(inp["X"], inp["W"], inp["bias"])
        Xq, xs = sq.sq_quantize_per_tensor(Xd)
        Wq, ws = sq.sq_quantize_per_tensor(Wd)
        Y_pt = sq.sq_linear(Xq, xs, Wq, ws, b)
        s = sq.sq_calibrate(dev_bf16(inp["C"]), Wd, wl.alpha_f32)
        Wq_s, ws_s = sq.sq_prepare_weight(Wd, s)
        Y_sq = sq.sq_forward(Xd, s, Wq_s, ws_s, b)
        torch.cuda.synchronize()
        e_pt = O.quantization_error(Y_fp, O.widen_bf16(host_bf16_bits(Y_pt)).astype(np.float64))
        e_sq = O.quantization_error(Y_fp, O.widen_bf16(host_bf16_bits(Y_sq)).astype(np.float64))
        print(f"\n[accuracy] {name}: relative error per-tensor {e_pt:.4g}, SmoothQuant {e_sq:.4g}")
        assert e_pt > 2 * e_sq
