"""sq_calibrate_noalloc: calibration for callers that cannot give the library
device memory (an engine that owns every byte through its own fixed pool, or a
loop where an allocation is not allowed).  It must give the same smoothing
factor as sq_calibrate, which takes a caller workspace, on consecutive calls:
the second call reuses the library's fixed scratch array and must not see the
first call's leftovers.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from tests.helpers import assert_scales_close, dev_bf16, host

pytestmark = pytest.mark.gpu

SQ_OK, SQ_ERR_SHAPE = 0, 2


@pytest.fixture(scope="module")
def sq():
    assert torch.cuda.is_available(), "GPU test"
    import w8a8_smoothquant_int8_sq_b200 as m
    return m


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(sq, C, W, alpha, s, mx=None):
    R = 0 if C is None else C.shape[0]
    N, K = W.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return sq.lib.sq_calibrate_noalloc(_p(C), R, K, _p(W), N, ctypes.c_float(alpha), _p(s), _p(mx), stream)


def test_noalloc_matches_workspace_calibration_on_consecutive_calls(sq):
    wl = workloads.get("proj")
    inp = workloads.make_inputs(wl, ("C", "W"))
    C1, W = dev_bf16(inp["C"]), dev_bf16(inp["W"])
    # second batch: same shape, no outlier channels, so every column max is
    # smaller than in the first -- stale maxima from call 1 would show up in s
    C2 = dev_bf16(workloads.random_bf16((wl.R, wl.K), seed=777))
    K = wl.K
    for C in (C1, C2):                                   # two calls in a row
        s_ref = sq.sq_calibrate(C, W, wl.alpha_f32)      # existing entry point (workspace)
        s = torch.empty(K, dtype=torch.float32, device="cuda")
        assert _noalloc(sq, C, W, wl.alpha_f32, s) == SQ_OK, sq.lib.sq_last_error()
        torch.cuda.synchronize()
        assert_scales_close(host(s), host(s_ref), "sq_calibrate_noalloc vs sq_calibrate")
    # with the running max, twice more (tiny layer, different K)
    wt = workloads.get("tiny")
    it = workloads.make_inputs(wt, ("C", "W"))
    Ct, Wt = dev_bf16(it["C"]), dev_bf16(it["W"])
    mx_a = torch.zeros(wt.K, dtype=torch.float32, device="cuda")
    mx_b = torch.zeros(wt.K, dtype=torch.float32, device="cuda")
    for half in (Ct[:32], Ct[32:]):
        s_ref = sq.sq_calibrate(half, Wt, wt.alpha_f32, mx_inout=mx_a)
        s = torch.empty(wt.K, dtype=torch.float32, device="cuda")
        assert _noalloc(sq, half, Wt, wt.alpha_f32, s, mx_b) == SQ_OK, sq.lib.sq_last_error()
        torch.cuda.synchronize()
        assert_scales_close(host(s), host(s_ref), "noalloc with running max")
        assert np.array_equal(host(mx_a), host(mx_b))


def test_noalloc_rejects_k_beyond_its_scratch(sq):
    K = 16384 + 16
    W = torch.zeros(8, K, dtype=torch.bfloat16, device="cuda")
    C = torch.zeros(4, K, dtype=torch.bfloat16, device="cuda")
    s = torch.empty(K, dtype=torch.float32, device="cuda")
    assert _noalloc(sq, C, W, 0.5, s) == SQ_ERR_SHAPE
    assert b"K <= 16384" in sq.lib.sq_last_error()
