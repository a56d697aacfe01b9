"""Device-side failure detection without a GPU fault: every pipeline wait of
the GEMM is bounded.  With the test hook on, the producer never fills the first
stage, the waits give up after 50 ms, the kernel reports bit 0 of the status
word and returns; the context stays usable and the next call is exact."""
import time

import numpy as np
import pytest
import torch

from oracle import smoothquant as O
from tests.helpers import assert_y_close, dev, host, host_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sq():
    assert torch.cuda.is_available(), "GPU test"
    import w8a8_smoothquant_int8_sq_b200 as m
    return m


def test_pipeline_wait_timeout_is_reported_and_the_context_survives(sq):
    rng = np.random.default_rng(99)
    M, N, K = 256, 512, 4096  # general GEMM (M > 32), 32 k-blocks: more than the ring holds
    Xq = rng.integers(-127, 128, (M, K), dtype=np.int64).astype(np.int8)
    Wq = rng.integers(-127, 128, (N, K), dtype=np.int64).astype(np.int8)
    Xq_d, Wq_d = dev(Xq), dev(Wq)
    assert sq.sq_device_status(clear=True) == 0
    try:
        sq.sq_debug_pipeline_stall(True, 50_000_000)
        t0 = time.perf_counter()
        sq.sq_gemm_s32(Xq_d, Wq_d)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        sq.sq_debug_pipeline_stall(False)
    flags = sq.sq_device_status(clear=True)
    assert flags & 1, "the stalled pipeline was not reported"
    assert elapsed < 5.0
    # the context is intact: the same call now returns the exact product
    acc = host(sq.sq_gemm_s32(Xq_d, Wq_d))
    assert np.array_equal(acc.astype(np.int64), O.int8_gemm(Xq, Wq))
    assert sq.sq_device_status() == 0


def test_split_k_wait_timeout_is_reported_and_the_context_survives(sq):
    """The same failure in the split-K GEMM (few 128 x 256 tiles, K split over a
    CTA pair, partial sums exchanged through the workspace): the stalled CTA
    still stores its (zero) partial, so its partner never waits for it."""
    rng = np.random.default_rng(98)
    M, N, K = 256, 512, 4096  # 4 tiles of 128 x 256: split-K when a workspace is given
    Xq = rng.integers(-127, 128, (M, K), dtype=np.int64).astype(np.int8)
    Wq = rng.integers(-127, 128, (N, K), dtype=np.int64).astype(np.int8)
    xs = (rng.random(M, dtype=np.float32) * 1e-3 + 1e-4).astype(np.float32)
    ws = (rng.random(N, dtype=np.float32) * 1e-3 + 1e-4).astype(np.float32)
    assert sq.sq_workspace_bytes(M, N, K) > 0
    args = (dev(Xq), dev(xs), dev(Wq), dev(ws))
    assert sq.sq_device_status(clear=True) == 0
    try:
        sq.sq_debug_pipeline_stall(True, 50_000_000)
        t0 = time.perf_counter()
        sq.sq_linear(*args)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        sq.sq_debug_pipeline_stall(False)
    flags = sq.sq_device_status(clear=True)
    assert flags & 1, "the stalled split-K pipeline was not reported"
    assert elapsed < 5.0
    Y = sq.sq_linear(*args)
    torch.cuda.synchronize()
    assert_y_close(host_bf16_bits(Y), O.int8_gemm(Xq, Wq), xs, ws, None, "split-K after a timeout")
    assert sq.sq_device_status() == 0


def test_cta_pair_wait_timeout_is_reported_and_the_context_survives(sq):
    """The same failure in the CTA-pair GEMM (256 x 256 tiles shared by the two
    CTAs of a cluster): both producers skip their first stage, every wait of
    both CTAs gives up, and the pair meets at its closing cluster barrier."""
    rng = np.random.default_rng(97)
    M, N, K = 2048, 9472, 1024  # 8 x 37 pair tiles: more than one per pair
    Xq = rng.integers(-127, 128, (M, K), dtype=np.int64).astype(np.int8)
    Wq = rng.integers(-127, 128, (N, K), dtype=np.int64).astype(np.int8)
    Xq_d, Wq_d = dev(Xq), dev(Wq)
    assert sq.sq_device_status(clear=True) == 0
    try:
        sq.sq_debug_pipeline_stall(True, 50_000_000)
        t0 = time.perf_counter()
        sq.sq_gemm_s32(Xq_d, Wq_d)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        sq.sq_debug_pipeline_stall(False)
    flags = sq.sq_device_status(clear=True)
    assert flags & 1, "the stalled pair pipeline was not reported"
    assert elapsed < 5.0
    acc = host(sq.sq_gemm_s32(Xq_d, Wq_d))
    assert np.array_equal(acc.astype(np.int64), O.int8_gemm(Xq, Wq))
    assert sq.sq_device_status() == 0


def test_fused_prologue_wait_timeout_is_reported_and_the_context_survives(sq):
    """The same failure in the GEMM that quantises X itself (CTA pairs, 256 x
    512 tiles, converter warps feeding the A operand): the Wq producers skip
    their first stage, so the MMA's first wait gives up; every other wait of
    both CTAs (converters, X producer, epilogue) gives up in turn."""
    rng = np.random.default_rng(96)
    M, N, K = 1024, 4096, 1024  # 4 x 8 pair tiles, 8 k-blocks: more than the ring holds
    X = torch.randn(M, K, device="cuda").to(torch.bfloat16)
    s = (torch.rand(K, device="cuda") + 0.5).float()
    Wq = dev(rng.integers(-127, 128, (N, K), dtype=np.int64).astype(np.int8))
    ws = dev((rng.random(N, dtype=np.float32) * 1e-3 + 1e-4).astype(np.float32))
    assert sq.sq_device_status(clear=True) == 0
    try:
        sq.sq_debug_pipeline_stall(True, 50_000_000)
        t0 = time.perf_counter()
        sq.sq_forward_prologue(X, s, Wq, ws)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        sq.sq_debug_pipeline_stall(False)
    flags = sq.sq_device_status(clear=True)
    assert flags & 1, "the stalled fused-prologue pipeline was not reported"
    assert elapsed < 5.0
    Y = sq.sq_forward_prologue(X, s, Wq, ws)
    Xq, xs = sq.sq_quantize_act(X, s)
    Y_l = sq.sq_linear(Xq, xs, Wq, ws)
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), Y_l.view(torch.int16))
    assert sq.sq_device_status() == 0


def test_few_token_wait_timeout_is_reported_and_the_context_survives(sq):
    """The same failure in the few-token GEMM (decode shape: K split over a
    cluster of 8, partial sums pushed to the reducing rank by st.async and
    counted on its mbarrier): every producer skips its first stage, so the MMA
    waits give up; every rank still sends its (zero) partial sums, so no rank
    waits for another.  Both the quantising forward and the product on
    prequantised codes are stalled, then run again and checked."""
    rng = np.random.default_rng(95)
    M, N, K = 8, 2048, 8192  # 8 row blocks x 8 K ranks, 8 k-blocks each: more than the ring holds
    X = torch.randn(M, K, device="cuda").to(torch.bfloat16)
    s = (torch.rand(K, device="cuda") + 0.5).float()
    Wq_h = rng.integers(-127, 128, (N, K), dtype=np.int64).astype(np.int8)
    ws_h = (rng.random(N, dtype=np.float32) * 1e-3 + 1e-4).astype(np.float32)
    Wq, ws = dev(Wq_h), dev(ws_h)
    Xq, xs = sq.sq_quantize_act(X, s)
    torch.cuda.synchronize()
    assert sq.sq_device_status(clear=True) == 0
    for run in (lambda: sq.sq_forward(X, s, Wq, ws), lambda: sq.sq_linear(Xq, xs, Wq, ws)):
        try:
            sq.sq_debug_pipeline_stall(True, 50_000_000)
            t0 = time.perf_counter()
            run()
            torch.cuda.synchronize()
            elapsed = time.perf_counter() - t0
        finally:
            sq.sq_debug_pipeline_stall(False)
        flags = sq.sq_device_status(clear=True)
        assert flags & 1, "the stalled few-token pipeline was not reported"
        assert elapsed < 5.0
    Y_f = sq.sq_forward(X, s, Wq, ws)
    Y_l = sq.sq_linear(Xq, xs, Wq, ws)
    torch.cuda.synchronize()
    assert torch.equal(Y_f.view(torch.int16), Y_l.view(torch.int16)), "fused forward != quantise + product"
    assert_y_close(host_bf16_bits(Y_l), O.int8_gemm(host(Xq), Wq_h), host(xs), ws_h, None,
                   "few-token GEMM after a timeout")
    assert sq.sq_device_status() == 0


def test_backward_wait_timeout_is_reported_and_the_context_survives(sq):
    """The same failure in the straight-through backward's two tcgen05 GEMMs
    (dX and dW): their producers skip the first stage, the waits give up, the
    kernels report and return; then the whole backward runs again and matches
    its oracle within the derived bounds."""
    from tests.helpers import dev_bf16
    from tests.test_gpu_ste import _inputs, _run
    from oracle import ste_backward as STE
    G, X, W, mx = _inputs(64, 264, 640, seed=7)
    alpha = float(STE.alpha_from_logit(0.5))
    Wd, Xd = dev_bf16(W), dev_bf16(X)
    mx_d = dev(np.asarray(mx, np.float32).copy())
    s = sq.sq_calibrate(None, Wd, alpha, mx_inout=mx_d)
    Wq, ws = sq.sq_prepare_weight(Wd, s)
    Xq, xs = sq.sq_quantize_act(Xd, s)
    torch.cuda.synchronize()
    assert sq.sq_device_status(clear=True) == 0
    try:
        sq.sq_debug_pipeline_stall(True, 50_000_000)
        t0 = time.perf_counter()
        sq.sq_ste_backward(dev_bf16(G), Xd, Wd, s, mx_d, alpha, Xq, xs, Wq, ws)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        sq.sq_debug_pipeline_stall(False)
    flags = sq.sq_device_status(clear=True)
    assert flags & 1, "the stalled backward was not reported"
    assert elapsed < 5.0
    _run(sq, G, X, W, mx, 0.5, "backward after a timeout")


def test_weight_only_wait_timeout_is_reported_and_the_context_survives(sq):
    """The same failure in the int8 weight-only comparison kernel (K split
    over a cluster, partial sums pushed to rank 0): the first stage never
    fills, the waits give up, every CTA lets the copies it issued land and
    still meets its cluster at the reduction; the next call is exact."""
    from tests.helpers import dev_bf16
    from tests.test_gpu_weight_only import _check
    import workloads
    X = workloads.random_bf16((8, 4096), seed=12, scale=1.0)
    W = workloads.random_bf16((1024, 4096), seed=13, scale=0.02)
    Wq, ws = sq.sq_prepare_weight(dev_bf16(W), torch.ones(4096, dtype=torch.float32, device="cuda"))
    Xd = dev_bf16(X)
    torch.cuda.synchronize()
    assert sq.sq_device_status(clear=True) == 0
    try:
        sq.sq_debug_pipeline_stall(True, 50_000_000)
        t0 = time.perf_counter()
        sq.sq_linear_weight_only(Xd, Wq, ws, None)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        sq.sq_debug_pipeline_stall(False)
    flags = sq.sq_device_status(clear=True)
    assert flags & 1, "the stalled weight-only pipeline was not reported"
    assert elapsed < 5.0
    _check(sq, X, W, None, "weight-only after a timeout")
    assert sq.sq_device_status() == 0


def test_calibration_wait_timeout_is_reported_and_the_context_survives(sq):
    """The same failure in the calibration (column max-abs over C and W by a
    TMA ring per block): the first box of every block never fills, the waits
    give up, every block still merges what it has and takes part in its
    stripe's arrival count, so the workspace is left zero; the next call
    equals the oracle's s."""
    from tests.helpers import assert_scales_close, dev_bf16
    import workloads
    C = workloads.random_bf16((512, 4096), seed=21, scale=1.0, outlier_cols=[7, 900], outlier_scale=40.0)
    W = workloads.random_bf16((1024, 4096), seed=22, scale=0.02)
    Cd, Wd = dev_bf16(C), dev_bf16(W)
    torch.cuda.synchronize()
    assert sq.sq_device_status(clear=True) == 0
    try:
        sq.sq_debug_pipeline_stall(True, 50_000_000)
        t0 = time.perf_counter()
        sq.sq_calibrate(Cd, Wd, 0.5)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        sq.sq_debug_pipeline_stall(False)
    flags = sq.sq_device_status(clear=True)
    assert flags & 1, "the stalled calibration was not reported"
    assert elapsed < 5.0
    s = sq.sq_calibrate(Cd, Wd, 0.5)
    torch.cuda.synchronize()
    s_o, _ = O.calibrate(C, W, np.float32(0.5))
    assert_scales_close(host(s), s_o, "calibration after a timeout")
    assert sq.sq_device_status() == 0
