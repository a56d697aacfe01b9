"""The int8 weight-only linear on the GPU (through the C ABI) against its CPU
oracle.  The kernel sums in fp32 in its own order, so the bar is one bf16 ulp
of the exact value plus a first-order bound on the fp32 summation error:
gamma * sum_k |x * q| * w_scale with gamma = (longest sequential chain + 24)
* 2^-24; a thread's chain covers at most 512 columns (an eighth of the 4096
columns a CTA takes), then 8 warp sums and at most 8 K splits are added."""
import numpy as np
import pytest
import torch

import workloads
from oracle import smoothquant as O
from oracle import weight_only as WO
from tests.helpers import dev_bf16, host, host_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import w8a8_smoothquant_int8_sq_b200 as m
    return m


def _ulp_bf16(y):
    a = np.abs(y)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)


def _check(sq, X, W, b, label):
    K = W.shape[1]
    Wd = dev_bf16(W)
    Wq, ws = sq.sq_prepare_weight(Wd, torch.ones(K, dtype=torch.float32, device="cuda"))
    Wq_o, ws_o = O.fold_and_quantize_weight(W, np.ones(K, np.float32))
    assert np.array_equal(host(Wq), Wq_o) and np.array_equal(host(ws), ws_o), f"{label}: weight prep"
    Y = sq.sq_linear_weight_only(dev_bf16(X), Wq, ws, dev_bf16(b) if b is not None else None)
    torch.cuda.synchronize()
    _, y = WO.weight_only_linear(X, Wq_o, ws_o, b)
    S = WO.abs_product_sum(X, Wq_o, ws_o)
    gamma = (min(K, 4096) / 8 + 24) * 2.0 ** -24
    got = O.widen_bf16(host_bf16_bits(Y)).astype(np.float64)
    err = np.abs(got - y)
    bound = _ulp_bf16(y) + gamma * S
    worst = float(np.max(err / bound))
    assert worst <= 1.0, f"{label}: error {worst:.3f} of the bound"
    print(f"\n[weight-only parity] {label}: max error / bound {worst:.3f}")


def test_decode_workload(sq):
    wl = workloads.get("decode")
    inp = workloads.make_inputs(wl, ("X", "W"))
    _check(sq, inp["X"], inp["W"], None, "decode 8x8192x8192")


@pytest.mark.parametrize("M,N,K,with_bias", [
    (1, 256, 256, True),
    (3, 200, 48, False),       # ragged N, K below one CTA eighth
    (13, 1000, 4112, True),    # two token groups, ragged N and K
    (8, 128, 16, True),        # smallest K
    (5, 300, 16384, False),    # largest K: four splits of 4096 columns
])
def test_ragged(sq, M, N, K, with_bias):
    X = workloads.random_bf16((M, K), seed=M * 13 + K, scale=1.0, outlier_cols=[K // 2], outlier_scale=50.0)
    W = workloads.random_bf16((N, K), seed=N + 7, scale=0.02)
    b = workloads.random_bf16((N,), seed=N + 8, scale=0.01) if with_bias else None
    _check(sq, X, W, b, f"{M}x{N}x{K}")
