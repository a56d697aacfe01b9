"""The C ABI library without a GPU: it loads, exports every symbol that
include/sq.h declares, and rejects bad arguments with status codes before it
touches a device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def sq():
    from w8a8_smoothquant_int8_sq_b200 import build
    build.build()
    import w8a8_smoothquant_int8_sq_b200 as m
    return m


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "sq.h")).read()
    return sorted(set(re.findall(r"SQ_API\s+[\w\s\*]+?\b(sq_\w+)\s*\(", text)))


def test_header_declares_the_path():
    names = declared_symbols()
    for n in ("sq_calibrate", "sq_prepare_weight", "sq_quantize_act", "sq_linear", "sq_forward", "sq_gemm_s32"):
        assert n in names


def test_every_declared_symbol_is_exported(sq):
    lib = ctypes.CDLL(sq.library_path)
    missing = [n for n in declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_has_every_entry_point(sq):
    """The Python binding carries the C names (sq_last_error and
    sq_status_string are surfaced through SqError instead)."""
    missing = [n for n in declared_symbols()
               if n not in ("sq_last_error", "sq_status_string") and not callable(getattr(sq, n, None))]
    assert not missing, missing


def test_version_and_sizes(sq):
    assert sq.sq_version() == 100
    assert sq.sq_calibrate_workspace_bytes(4096) >= 2 * 4096 * 4
    assert sq.sq_forward_workspace_bytes(512, 4096, 4096) >= 512 * 4096 + 512 * 4
    assert sq.lib.sq_status_string(7) == b"SQ_ERR_TIMEOUT"


def test_validation_before_device(sq):
    lib = sq.lib
    a = ctypes.c_void_p(1 << 20)          # 16-byte aligned, never dereferenced
    mis = ctypes.c_void_p((1 << 20) + 4)
    assert lib.sq_quantize_act(None, 4, 64, a, a, a, None) == 1
    assert lib.sq_quantize_act(a, 4, 40, a, a, a, None) == 3
    assert lib.sq_quantize_act(a, 4, 8, a, a, a, None) == 2
    assert lib.sq_quantize_act(a, 0, 64, a, a, a, None) == 2
    assert lib.sq_quantize_act(mis, 4, 64, a, a, a, None) == 3
    assert b"not 16-byte aligned" in lib.sq_last_error()
    assert lib.sq_prepare_weight(a, 4, 64, None, a, a, None) == 1
    assert lib.sq_prepare_weight(a, 4, 32768, a, a, a, None) == 2        # above the on-chip K limit
    assert lib.sq_calibrate(a, 4, 64, a, 8, ctypes.c_float(-0.1), a, None, a, 1024, None) == 4
    assert lib.sq_calibrate(a, 4, 64, a, 8, ctypes.c_float(float("nan")), a, None, a, 1024, None) == 4
    assert lib.sq_calibrate(a, 4, 64, a, 8, ctypes.c_float(0.5), a, None, a, 8, None) == 8
    assert lib.sq_calibrate(None, 0, 64, a, 8, ctypes.c_float(0.5), a, None, a, 1024, None) == 1
    assert lib.sq_linear(a, a, a, a, mis, 4, 8, 64, a, None, 0, None) == 3
    assert lib.sq_linear(a, a, a, a, None, 4, 8, 200000, a, None, 0, None) == 2
    assert lib.sq_forward(a, a, a, a, None, 4, 8, 64, a, a, 16, None) == 8
    assert lib.sq_forward_prologue(a, a, a, a, None, 4, 8, 64, a, a, 16, None) == 8      # workspace too small
    wsb = sq.sq_rel_mse_workspace_bytes()
    assert wsb >= 2 * 8 * 148 * 8
    d = ctypes.c_double
    assert lib.sq_rel_mse(a, a, 4, 8, d(0.5), a, None, a, a, wsb, None) == 4           # G_in without G_out
    assert lib.sq_rel_mse(a, a, 4, 8, d(0.5), None, None, None, a, wsb, None) == 1     # no loss_out
    assert lib.sq_rel_mse(a, mis, 4, 8, d(0.5), None, None, a, a, wsb, None) == 3      # Y_q misaligned
    assert lib.sq_rel_mse(a, a, 4, 8, d(0.5), None, None, a, a, 16, None) == 8         # workspace too small
    assert lib.sq_rel_mse(a, a, 0, 8, d(0.5), None, None, a, a, wsb, None) == 2        # M = 0
    assert lib.sq_rel_mse(a, a, 4, 8, d(float("nan")), None, None, a, a, wsb, None) == 4
    assert lib.sq_forward_prologue(a, mis, a, a, None, 4, 8, 64, a, a, 512, None) == 3   # s misaligned
    assert lib.sq_forward_prologue(a, a, a, a, None, 4, 8, 16400, a, a, 1 << 20, None) == 2  # K above 16384
    assert lib.sq_gemm_s32(a, a, 4, 0, 64, a, None) == 2
    ws = lib.sq_quantize_per_tensor_workspace_bytes()
    assert ws >= 4
    assert lib.sq_quantize_per_tensor(a, 4, 64, a, a, None, 0, None) == 8
    assert lib.sq_quantize_per_tensor(a, 4, 64, a, a, a, ws - 4, None) == 8
    assert lib.sq_quantize_per_tensor(a, 4, 40, a, a, a, ws, None) == 3
    assert lib.sq_quantize_per_tensor(None, 4, 64, a, a, a, ws, None) == 1
    assert lib.sq_quantize_per_tensor(a, 0, 64, a, a, a, ws, None) == 2
    # straight-through backward: N % 8, alpha, NULL, workspace size
    wsb = lib.sq_ste_backward_workspace_bytes(4, 64, 64)
    assert wsb >= 64 * 64 * 2 + 64 * 8 * 2 + 4 * 64 * 8 * 2 + 3 * 64 * 4
    f = ctypes.c_float

    def bwd(G=a, N=64, alpha=0.5, db=None, ds=None, ws=a, nbytes=wsb, K=64):
        return lib.sq_ste_backward(G, a, a, a, a, f(alpha), a, a, a, a, 4, N, K, a, a, db, ds, a, ws, nbytes, None)
    assert bwd(N=60) == 3
    assert bwd(alpha=1.5) == 4
    assert bwd(alpha=float("nan")) == 4
    assert bwd(G=None) == 1
    assert bwd(db=mis) == 3
    assert bwd(ds=mis) == 3
    assert bwd(nbytes=wsb - 1) == 8
    assert bwd(K=40) == 3


def test_valid_call_without_gpu_fails_cleanly(sq):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    a = ctypes.c_void_p(1 << 20)
    st = sq.lib.sq_quantize_act(a, 4, 64, a, a, a, None)
    assert st in (5, 6)          # no sm_100 device: UNSUPPORTED or CUDA error, never a crash
    assert sq.lib.sq_last_error()


def test_binding_refuses_host_tensors(sq):
    """No CPU fallback: every entry point of the binding rejects host tensors
    before calling the library."""
    import torch
    bf = torch.zeros(4, 64, dtype=torch.bfloat16)
    i8 = torch.zeros(4, 64, dtype=torch.int8)
    f1 = torch.zeros(64, dtype=torch.float32)
    f4 = torch.zeros(4, dtype=torch.float32)
    G = torch.zeros(4, 8, dtype=torch.bfloat16)
    W8 = torch.zeros(8, 64, dtype=torch.bfloat16)
    calls = [
        lambda: sq.sq_calibrate(bf, bf, 0.5),
        lambda: sq.sq_prepare_weight(bf, f1),
        lambda: sq.sq_quantize_act(bf, f1),
        lambda: sq.sq_quantize_per_tensor(bf),
        lambda: sq.sq_linear(i8, f4, i8, f4),
        lambda: sq.sq_forward(bf, f1, i8, f4),
        lambda: sq.sq_linear_weight_only(bf, i8, f4),
        lambda: sq.sq_ste_backward(G, bf, W8, f1, f1, 0.5, i8, f4, torch.zeros(8, 64, dtype=torch.int8),
                                   torch.zeros(8, dtype=torch.float32)),
    ]
    for c in calls:
        with pytest.raises(ValueError, match="CUDA tensor"):
            c()
