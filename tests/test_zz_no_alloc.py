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
from oracle import smoothquant as O
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
    C2_bits = workloads.random_bf16((wl.R, wl.K), seed=777)
    C2 = dev_bf16(C2_bits)
    K = wl.K
    for C, C_bits in ((C1, inp["C"]), (C2, C2_bits)):   # two calls in a row
        s_ref = sq.sq_calibrate(C, W, wl.alpha_f32)      # existing entry point (workspace)
        s = torch.empty(K, dtype=torch.float32, device="cuda")
        assert _noalloc(sq, C, W, wl.alpha_f32, s) == SQ_OK, sq.lib.sq_last_error()
        torch.cuda.synchronize()
        assert_scales_close(host(s), host(s_ref), "sq_calibrate_noalloc vs sq_calibrate")
        # and against the CPU oracle on the same bf16 inputs
        s_o, _ = O.calibrate(C_bits, inp["W"], wl.alpha_f32)
        assert_scales_close(host(s), s_o, "sq_calibrate_noalloc vs the oracle")
    # with the running max, twice more (tiny layer, different K)
    wt = workloads.get("tiny")
    it = workloads.make_inputs(wt, ("C", "W"))
    Ct, Wt = dev_bf16(it["C"]), dev_bf16(it["W"])
    mx_a = torch.zeros(wt.K, dtype=torch.float32, device="cuda")
    mx_b = torch.zeros(wt.K, dtype=torch.float32, device="cuda")
    mx_o = None
    for half, lo, hi in ((Ct[:32], 0, 32), (Ct[32:], 32, None)):
        s_ref = sq.sq_calibrate(half, Wt, wt.alpha_f32, mx_inout=mx_a)
        s = torch.empty(wt.K, dtype=torch.float32, device="cuda")
        assert _noalloc(sq, half, Wt, wt.alpha_f32, s, mx_b) == SQ_OK, sq.lib.sq_last_error()
        torch.cuda.synchronize()
        assert_scales_close(host(s), host(s_ref), "noalloc with running max")
        assert np.array_equal(host(mx_a), host(mx_b))
        s_o, mx_o = O.calibrate(it["C"][lo:hi], it["W"], wt.alpha_f32, mx_prev=mx_o)
        assert_scales_close(host(s), s_o, "noalloc with running max vs the oracle")
        assert np.array_equal(host(mx_b), mx_o)


def test_noalloc_rejects_k_beyond_its_scratch(sq):
    K = 16384 + 16
    W = torch.zeros(8, K, dtype=torch.bfloat16, device="cuda")
    C = torch.zeros(4, K, dtype=torch.bfloat16, device="cuda")
    s = torch.empty(K, dtype=torch.float32, device="cuda")
    assert _noalloc(sq, C, W, 0.5, s) == SQ_ERR_SHAPE
    assert b"K <= 16384" in sq.lib.sq_last_error()
