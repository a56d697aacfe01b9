"""Outputs past 2^31 elements: Y[65536 x 32776] (2.15e9 entries, 4.3 GB of
bf16), K = 256, so every 64-bit index product of the GEMM epilogues, the row
quantiser and the quantising GEMM is exercised.  Sampled blocks of Y --
including the last row and the last (ragged) column -- against the oracle;
the quantising GEMM's Y equal to sq_linear's on the row quantiser's codes,
compared on the same samples and, for equality, over whole rows near the end
of the array."""
import numpy as np
import pytest
import torch

import workloads
from oracle import smoothquant as O
from tests.helpers import assert_codes, assert_y_close, dev, dev_bf16, host, host_bf16_bits

pytestmark = pytest.mark.gpu

M, N, K = 65536, 32776, 256


@pytest.fixture(scope="module")
def sq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import w8a8_smoothquant_int8_sq_b200 as m
    return m


def test_outputs_past_int32_indexing(sq):
    assert M * N > 2 ** 31
    X = workloads.random_bf16((M, K), seed=11)
    W = workloads.random_bf16((N, K), seed=12, scale=0.02)
    s = np.exp(np.random.default_rng(13).uniform(-1.0, 1.0, K)).astype(np.float32)
    Xd, Wd, sd = dev_bf16(X), dev_bf16(W), dev(s)
    Wq, ws = sq.sq_prepare_weight(Wd, sd)
    Xq, xs = sq.sq_quantize_act(Xd, sd)
    Y = sq.sq_linear(Xq, xs, Wq, ws)
    torch.cuda.synchronize()
    rng = np.random.default_rng(14)
    rows = np.sort(np.concatenate([[0, M - 1, M - 2, 2 ** 16 - 256], rng.choice(M, 28, replace=False)]))
    cols = np.sort(np.concatenate([[0, N - 1, N - 2, N - 8], rng.choice(N, 124, replace=False)]))
    rows_t, cols_t = torch.as_tensor(rows, device="cuda"), torch.as_tensor(cols, device="cuda")
    # the quantisers on the sampled rows, against the oracle
    Wq_o, ws_o = O.fold_and_quantize_weight(W[cols], s)
    _, _, vw = O.fold_and_quantize_weight_f64(W[cols], s)
    assert_codes(host(Wq[cols_t]), Wq_o, vw, "Wq sampled rows")
    assert np.array_equal(host(ws)[cols], ws_o)
    Xq_o, xs_o = O.quantize_activation(X[rows], s)
    _, _, vx = O.quantize_activation_f64(X[rows], s)
    assert_codes(host(Xq[rows_t]), Xq_o, vx, "Xq sampled rows")
    assert np.array_equal(host(xs)[rows], xs_o)
    # Y on the sampled block from the GPU's own codes (each output depends only
    # on its row of Xq and of Wq)
    acc_o = O.int8_gemm(host(Xq[rows_t]), host(Wq[cols_t]))
    y = host_bf16_bits(Y[rows_t][:, cols_t])
    assert_y_close(y, acc_o, host(xs)[rows], host(ws)[cols], None, "Y sampled block past 2^31")
    # the GEMM that quantises X itself: the same Y
    Yp = sq.sq_forward_prologue(Xd, sd, Wq, ws)
    torch.cuda.synchronize()
    assert torch.equal(Yp[rows_t][:, cols_t].view(torch.int16), Y[rows_t][:, cols_t].view(torch.int16))
    assert torch.equal(Yp[-4:].view(torch.int16), Y[-4:].view(torch.int16))
    assert sq.sq_device_status() == 0
