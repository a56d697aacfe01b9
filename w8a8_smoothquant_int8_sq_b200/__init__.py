"""SmoothQuant W8A8 int8 linear layer on B200 (sm_100a): Python binding of libsq.

This module is argument marshalling only: it checks tensor dtypes, devices and
shapes, allocates output tensors when the caller passes none, and calls the C
ABI declared in ``include/sq.h`` (``libsq.so``, built next to this file by
``build.py``).  Every step of the computation runs in the library's CUDA
kernels; there is no Python or CPU fallback -- importing this package without
the built library raises ImportError.

Tensors: bf16 inputs are ``torch.bfloat16``, codes ``torch.int8``, scales
``torch.float32``; all on the current CUDA device, contiguous, 16-byte aligned.
Work is enqueued on the current torch CUDA stream (or ``stream=``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

__all__ = [
    "SqError", "lib", "library_path",
    "sq_version", "sq_calibrate", "sq_calibrate_workspace_bytes", "sq_calibrate_noalloc", "sq_prepare_weight",
    "sq_quantize_act", "sq_quantize_per_tensor", "sq_quantize_per_tensor_workspace_bytes", "sq_linear_weight_only", "sq_ste_backward",
    "sq_ste_backward_workspace_bytes", "sq_linear", "sq_workspace_bytes", "sq_forward",
    "sq_forward_workspace_bytes", "sq_forward_prologue", "sq_rel_mse", "sq_rel_mse_workspace_bytes", "sq_forward_prologue_workspace_bytes", "sq_gemm_s32", "sq_device_status", "sq_debug_fail_after",
    "sq_debug_pipeline_stall",
    "STATUS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libsq.so")

STATUS = {
    0: "SQ_OK", 1: "SQ_ERR_NULL", 2: "SQ_ERR_SHAPE", 3: "SQ_ERR_ALIGN", 4: "SQ_ERR_ARG",
    5: "SQ_ERR_UNSUPPORTED", 6: "SQ_ERR_CUDA", 7: "SQ_ERR_TIMEOUT", 8: "SQ_ERR_WORKSPACE",
}

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t

# (name, restype, argtypes) of every entry point of include/sq.h
_SIGNATURES = [
    ("sq_version", ctypes.c_int, ()),
    ("sq_last_error", ctypes.c_char_p, ()),
    ("sq_status_string", ctypes.c_char_p, (ctypes.c_int,)),
    ("sq_calibrate_workspace_bytes", _SZ, (_I64,)),
    ("sq_calibrate", ctypes.c_int, (_P, _I64, _I64, _P, _I64, ctypes.c_float, _P, _P, _P, _SZ, _P)),
    ("sq_calibrate_noalloc", ctypes.c_int, (_P, _I64, _I64, _P, _I64, ctypes.c_float, _P, _P, _P)),
    ("sq_prepare_weight", ctypes.c_int, (_P, _I64, _I64, _P, _P, _P, _P)),
    ("sq_quantize_act", ctypes.c_int, (_P, _I64, _I64, _P, _P, _P, _P)),
    ("sq_quantize_per_tensor_workspace_bytes", _SZ, ()),
    ("sq_quantize_per_tensor", ctypes.c_int, (_P, _I64, _I64, _P, _P, _P, _SZ, _P)),
    ("sq_linear_weight_only", ctypes.c_int, (_P, _I64, _P, _P, _P, _I64, _I64, _P, _P)),
    ("sq_ste_backward_workspace_bytes", _SZ, (_I64, _I64, _I64)),
    ("sq_rel_mse_workspace_bytes", _SZ, ()),
    ("sq_rel_mse", ctypes.c_int, (_P, _P, _I64, _I64, ctypes.c_double, _P, _P, _P, _P, _SZ, _P)),
    ("sq_ste_backward", ctypes.c_int, (_P, _P, _P, _P, _P, ctypes.c_float, _P, _P, _P, _P, _I64, _I64, _I64,
                                       _P, _P, _P, _P, _P, _P, _SZ, _P)),
    ("sq_workspace_bytes", _SZ, (_I64, _I64, _I64)),
    ("sq_linear", ctypes.c_int, (_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _SZ, _P)),
    ("sq_forward_workspace_bytes", _SZ, (_I64, _I64, _I64)),
    ("sq_forward", ctypes.c_int, (_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _SZ, _P)),
    ("sq_forward_prologue_workspace_bytes", _SZ, (_I64, _I64)),
    ("sq_forward_prologue", ctypes.c_int, (_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _SZ, _P)),
    ("sq_gemm_s32", ctypes.c_int, (_P, _P, _I64, _I64, _I64, _P, _P)),
    ("sq_device_status", ctypes.c_int, (ctypes.POINTER(ctypes.c_uint32), ctypes.c_int)),
    ("sq_debug_fail_after", None, (ctypes.c_int,)),
    ("sq_debug_pipeline_stall", None, (ctypes.c_int, _I64)),
]

_LIB = None


def _load():
    """Load libsq.so on first use.  There is no fallback: a missing library is an error."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(library_path):
            raise ImportError(
                f"libsq.so not found at {library_path}; build it with "
                "`python -m w8a8_smoothquant_int8_sq_b200.build` (nvcc, sm_100a)")
        handle = ctypes.CDLL(library_path)
        for name, res, args in _SIGNATURES:
            f = getattr(handle, name)
            f.restype = res
            f.argtypes = list(args)
        _LIB = handle
    return _LIB


def __getattr__(name):
    if name == "lib":
        return _load()
    raise AttributeError(name)


class SqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


def _check(st: int) -> None:
    if st != 0:
        msg = _load().sq_last_error()
        raise SqError(st, msg.decode() if msg else "")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _want(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int) -> torch.Tensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _out(t, shape, dtype, device, name):
    if t is None:
        return torch.empty(shape, dtype=dtype, device=device)
    _want(t, name, dtype, len(shape))
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def sq_version() -> int:
    return int(_load().sq_version())


def sq_calibrate_workspace_bytes(K: int) -> int:
    return int(_load().sq_calibrate_workspace_bytes(K))


def sq_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_load().sq_workspace_bytes(M, N, K))


def sq_forward_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_load().sq_forward_workspace_bytes(M, N, K))


def _workspace(ws, nbytes, device):
    if ws is None:
        return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
    if ws.dtype != torch.uint8 or ws.numel() < nbytes:
        raise ValueError(f"workspace must be a uint8 tensor of at least {nbytes} bytes")
    return ws


def sq_calibrate(C: Optional[torch.Tensor], W: torch.Tensor, alpha: float, s: Optional[torch.Tensor] = None,
                 mx_inout: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """Smoothing factor s[K] (fp32) from calibration activations C[R,K] (or
    only the running max ``mx_inout``) and the weight W[N,K]."""
    _want(W, "W", torch.bfloat16, 2)
    N, K = W.shape
    if C is not None:
        _want(C, "C", torch.bfloat16, 2)
        if C.shape[1] != K:
            raise ValueError(f"C has {C.shape[1]} columns, W has {K}")
        R = C.shape[0]
    else:
        R = 0
    if mx_inout is not None:
        _want(mx_inout, "mx_inout", torch.float32, 1)
        if mx_inout.shape[0] != K:
            raise ValueError("mx_inout must have K entries")
    s = _out(s, (K,), torch.float32, W.device, "s")
    ws = _workspace(workspace, sq_calibrate_workspace_bytes(K), W.device)
    _check(_load().sq_calibrate(_ptr(C), R, K, _ptr(W), N, float(alpha), _ptr(s), _ptr(mx_inout), _ptr(ws),
                            ws.numel(), _stream(stream)))
    return s


def sq_calibrate_noalloc(C: Optional[torch.Tensor], W: torch.Tensor, alpha: float,
                         s: Optional[torch.Tensor] = None, mx_inout: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """sq_calibrate without scratch from the caller (K <= 16384): for code that
    cannot give the library device memory.  The library uses a fixed device
    array of its own; calls that overlap on the GPU race (see include/sq.h).
    Only ``s`` is allocated here when the caller passes none."""
    _want(W, "W", torch.bfloat16, 2)
    N, K = W.shape
    R = 0
    if C is not None:
        _want(C, "C", torch.bfloat16, 2)
        if C.shape[1] != K:
            raise ValueError(f"C has {C.shape[1]} columns, W has {K}")
        R = C.shape[0]
    if mx_inout is not None:
        _want(mx_inout, "mx_inout", torch.float32, 1)
    s = _out(s, (K,), torch.float32, W.device, "s")
    _check(_load().sq_calibrate_noalloc(_ptr(C), R, K, _ptr(W), N, float(alpha), _ptr(s), _ptr(mx_inout),
                                    _stream(stream)))
    return s


def sq_prepare_weight(W: torch.Tensor, s: torch.Tensor, Wq: Optional[torch.Tensor] = None,
                      w_scale: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """(Wq[N,K] int8, w_scale[N] fp32) from W[N,K] bf16 and s[K]."""
    _want(W, "W", torch.bfloat16, 2)
    _want(s, "s", torch.float32, 1)
    N, K = W.shape
    if s.shape[0] != K:
        raise ValueError("s must have K entries")
    Wq = _out(Wq, (N, K), torch.int8, W.device, "Wq")
    w_scale = _out(w_scale, (N,), torch.float32, W.device, "w_scale")
    _check(_load().sq_prepare_weight(_ptr(W), N, K, _ptr(s), _ptr(Wq), _ptr(w_scale), _stream(stream)))
    return Wq, w_scale


def sq_quantize_act(X: torch.Tensor, s: torch.Tensor, Xq: Optional[torch.Tensor] = None,
                    x_scale: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """(Xq[M,K] int8, x_scale[M] fp32) from X[M,K] bf16 and s[K]."""
    _want(X, "X", torch.bfloat16, 2)
    _want(s, "s", torch.float32, 1)
    M, K = X.shape
    if s.shape[0] != K:
        raise ValueError("s must have K entries")
    Xq = _out(Xq, (M, K), torch.int8, X.device, "Xq")
    x_scale = _out(x_scale, (M,), torch.float32, X.device, "x_scale")
    _check(_load().sq_quantize_act(_ptr(X), M, K, _ptr(s), _ptr(Xq), _ptr(x_scale), _stream(stream)))
    return Xq, x_scale


def sq_quantize_per_tensor_workspace_bytes() -> int:
    return int(_load().sq_quantize_per_tensor_workspace_bytes())


def sq_quantize_per_tensor(A: torch.Tensor, Aq: Optional[torch.Tensor] = None,
                           scale_rows: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                           stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """(Aq[rows,K] int8, scale_rows[rows] fp32) with one scale for the whole of
    A[rows,K] bf16 -- the per-tensor baseline; feed the pair to sq_linear."""
    _want(A, "A", torch.bfloat16, 2)
    rows, K = A.shape
    Aq = _out(Aq, (rows, K), torch.int8, A.device, "Aq")
    scale_rows = _out(scale_rows, (rows,), torch.float32, A.device, "scale_rows")
    ws = _workspace(workspace, sq_quantize_per_tensor_workspace_bytes(), A.device)
    _check(_load().sq_quantize_per_tensor(_ptr(A), rows, K, _ptr(Aq), _ptr(scale_rows), _ptr(ws), ws.numel(),
                                          _stream(stream)))
    return Aq, scale_rows


def sq_linear_weight_only(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                          bias: Optional[torch.Tensor] = None, Y: Optional[torch.Tensor] = None,
                          stream=None) -> torch.Tensor:
    """Y[M,N] bf16 = bf16((X Wq^T) * w_scale[n] + bias[n]) with X[M,K] bf16 (weight-only int8)."""
    _want(X, "X", torch.bfloat16, 2)
    _want(Wq, "Wq", torch.int8, 2)
    _want(w_scale, "w_scale", torch.float32, 1)
    M, K = X.shape
    N = Wq.shape[0]
    if Wq.shape[1] != K or w_scale.shape[0] != N:
        raise ValueError("inconsistent shapes")
    if bias is not None:
        _want(bias, "bias", torch.bfloat16, 1)
    Y = _out(Y, (M, N), torch.bfloat16, X.device, "Y")
    _check(_load().sq_linear_weight_only(_ptr(X), M, _ptr(Wq), _ptr(w_scale), _ptr(bias), N, K, _ptr(Y),
                                         _stream(stream)))
    return Y


def sq_ste_backward_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_load().sq_ste_backward_workspace_bytes(M, N, K))


def sq_ste_backward(G: torch.Tensor, X: torch.Tensor, W: torch.Tensor, s: torch.Tensor, mx: torch.Tensor,
                    alpha: float, Xq: torch.Tensor, x_scale: torch.Tensor, Wq: torch.Tensor,
                    w_scale: torch.Tensor, with_db: bool = True, with_ds: bool = False,
                    dX: Optional[torch.Tensor] = None, dW: Optional[torch.Tensor] = None,
                    db: Optional[torch.Tensor] = None, ds: Optional[torch.Tensor] = None,
                    d_eta: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                    stream=None):
    """Straight-through backward of the learnable-alpha layer: returns
    ``(dX [M,K] fp32, dW [N,K] fp32, db [N] fp32 or None, ds [K] fp32 or None,
    d_eta [1] fp32)`` from G = dL/dY [M,N] bf16 and the forward's inputs, s,
    running max, alpha, codes and scales."""
    _want(G, "G", torch.bfloat16, 2)
    _want(X, "X", torch.bfloat16, 2)
    _want(W, "W", torch.bfloat16, 2)
    _want(s, "s", torch.float32, 1)
    _want(mx, "mx", torch.float32, 1)
    _want(Xq, "Xq", torch.int8, 2)
    _want(x_scale, "x_scale", torch.float32, 1)
    _want(Wq, "Wq", torch.int8, 2)
    _want(w_scale, "w_scale", torch.float32, 1)
    M, K = X.shape
    N = W.shape[0]
    if (G.shape != (M, N) or W.shape[1] != K or s.shape[0] != K or mx.shape[0] != K or Xq.shape != (M, K)
            or x_scale.shape[0] != M or Wq.shape != (N, K) or w_scale.shape[0] != N):
        raise ValueError("inconsistent shapes")
    dX = _out(dX, (M, K), torch.float32, X.device, "dX")
    dW = _out(dW, (N, K), torch.float32, X.device, "dW")
    if with_db or db is not None:
        db = _out(db, (N,), torch.float32, X.device, "db")
    if with_ds or ds is not None:
        ds = _out(ds, (K,), torch.float32, X.device, "ds")
    d_eta = _out(d_eta, (1,), torch.float32, X.device, "d_eta")
    nbytes = sq_ste_backward_workspace_bytes(M, N, K)
    ws = _workspace(workspace, nbytes, X.device)
    _check(_load().sq_ste_backward(_ptr(G), _ptr(X), _ptr(W), _ptr(s), _ptr(mx), ctypes.c_float(alpha), _ptr(Xq),
                                   _ptr(x_scale), _ptr(Wq), _ptr(w_scale), M, N, K, _ptr(dX), _ptr(dW), _ptr(db),
                                   _ptr(ds), _ptr(d_eta), _ptr(ws), nbytes if workspace is None else ws.numel(),
                                   _stream(stream)))
    return dX, dW, db, ds, d_eta


def sq_linear(Xq: torch.Tensor, x_scale: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
              bias: Optional[torch.Tensor] = None, Y: Optional[torch.Tensor] = None,
              workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Y[M,N] bf16 = bf16((Xq Wq^T) * x_scale[m] * w_scale[n] + bias[n])."""
    _want(Xq, "Xq", torch.int8, 2)
    _want(Wq, "Wq", torch.int8, 2)
    _want(x_scale, "x_scale", torch.float32, 1)
    _want(w_scale, "w_scale", torch.float32, 1)
    M, K = Xq.shape
    N = Wq.shape[0]
    if Wq.shape[1] != K or x_scale.shape[0] != M or w_scale.shape[0] != N:
        raise ValueError("inconsistent shapes")
    if bias is not None:
        _want(bias, "bias", torch.bfloat16, 1)
        if bias.shape[0] != N:
            raise ValueError("bias must have N entries")
    Y = _out(Y, (M, N), torch.bfloat16, Xq.device, "Y")
    nbytes = sq_workspace_bytes(M, N, K)
    ws = _workspace(workspace, nbytes, Xq.device) if nbytes else workspace
    _check(_load().sq_linear(_ptr(Xq), _ptr(x_scale), _ptr(Wq), _ptr(w_scale), _ptr(bias), M, N, K, _ptr(Y),
                         _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))
    return Y


def sq_forward(X: torch.Tensor, s: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
               bias: Optional[torch.Tensor] = None, Y: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Y[M,N] bf16 from X[M,K] bf16: per-token quantisation of X/s, int8 GEMM,
    dequant + bias, all in the library's kernels."""
    _want(X, "X", torch.bfloat16, 2)
    _want(s, "s", torch.float32, 1)
    _want(Wq, "Wq", torch.int8, 2)
    _want(w_scale, "w_scale", torch.float32, 1)
    M, K = X.shape
    N = Wq.shape[0]
    if Wq.shape[1] != K or s.shape[0] != K or w_scale.shape[0] != N:
        raise ValueError("inconsistent shapes")
    if bias is not None:
        _want(bias, "bias", torch.bfloat16, 1)
        if bias.shape[0] != N:
            raise ValueError("bias must have N entries")
    Y = _out(Y, (M, N), torch.bfloat16, X.device, "Y")
    ws = _workspace(workspace, sq_forward_workspace_bytes(M, N, K), X.device)
    _check(_load().sq_forward(_ptr(X), _ptr(s), _ptr(Wq), _ptr(w_scale), _ptr(bias), M, N, K, _ptr(Y), _ptr(ws),
                          ws.numel(), _stream(stream)))
    return Y


def sq_rel_mse_workspace_bytes() -> int:
    return int(_load().sq_rel_mse_workspace_bytes())


def sq_rel_mse(Y_fp: torch.Tensor, Y_q: torch.Tensor, lam: float = 0.0, G_in: Optional[torch.Tensor] = None,
               G_out: Optional[torch.Tensor] = None, loss: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None, stream=None):
    """The relative-MSE auxiliary loss ||Y_fp - Y_q||^2 / ||Y_fp||^2 (a
    float64 tensor of one element, on the device) and, given G_in (bf16
    [M, N]), G_out = bf16(G_in + lam * d aux / d Y_q).  Returns (loss, G_out);
    G_out is None without G_in.  G_out may be G_in (in place)."""
    _want(Y_fp, "Y_fp", torch.bfloat16, 2)
    _want(Y_q, "Y_q", torch.bfloat16, 2)
    M, N = Y_fp.shape
    if tuple(Y_q.shape) != (M, N):
        raise ValueError("Y_fp and Y_q must have the same shape")
    if G_in is not None:
        _want(G_in, "G_in", torch.bfloat16, 2)
        if tuple(G_in.shape) != (M, N):
            raise ValueError("G_in must be [M, N]")
        G_out = _out(G_out, (M, N), torch.bfloat16, Y_fp.device, "G_out")
    elif G_out is not None:
        raise ValueError("G_out without G_in")
    loss = _out(loss, (1,), torch.float64, Y_fp.device, "loss")
    ws = _workspace(workspace, sq_rel_mse_workspace_bytes(), Y_fp.device)
    _check(_load().sq_rel_mse(_ptr(Y_fp), _ptr(Y_q), M, N, float(lam), _ptr(G_in), _ptr(G_out), _ptr(loss),
                          _ptr(ws), ws.numel(), _stream(stream)))
    return loss, G_out


def sq_forward_prologue_workspace_bytes(M: int, K: int) -> int:
    return int(_load().sq_forward_prologue_workspace_bytes(M, K))


def sq_forward_prologue(X: torch.Tensor, s: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                        bias: Optional[torch.Tensor] = None, Y: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Y[M,N] bf16 from X[M,K] bf16 like ``sq_forward``, with the per-token
    quantisation done inside the GEMM (a scale pre-pass, then converter warps
    that write the codes into the tensor core's shared-memory operand).  The
    workspace receives x_scale[M] at offset 0."""
    _want(X, "X", torch.bfloat16, 2)
    _want(s, "s", torch.float32, 1)
    _want(Wq, "Wq", torch.int8, 2)
    _want(w_scale, "w_scale", torch.float32, 1)
    M, K = X.shape
    N = Wq.shape[0]
    if Wq.shape[1] != K or s.shape[0] != K or w_scale.shape[0] != N:
        raise ValueError("inconsistent shapes")
    if bias is not None:
        _want(bias, "bias", torch.bfloat16, 1)
        if bias.shape[0] != N:
            raise ValueError("bias must have N entries")
    Y = _out(Y, (M, N), torch.bfloat16, X.device, "Y")
    ws = _workspace(workspace, sq_forward_prologue_workspace_bytes(M, K), X.device)
    _check(_load().sq_forward_prologue(_ptr(X), _ptr(s), _ptr(Wq), _ptr(w_scale), _ptr(bias), M, N, K, _ptr(Y),
                                   _ptr(ws), ws.numel(), _stream(stream)))
    return Y


def sq_gemm_s32(Xq: torch.Tensor, Wq: torch.Tensor, acc: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """acc[M,N] int32 = Xq Wq^T on the tensor cores (accumulator exposed for tests)."""
    _want(Xq, "Xq", torch.int8, 2)
    _want(Wq, "Wq", torch.int8, 2)
    M, K = Xq.shape
    N = Wq.shape[0]
    if Wq.shape[1] != K:
        raise ValueError("inconsistent K")
    acc = _out(acc, (M, N), torch.int32, Xq.device, "acc")
    _check(_load().sq_gemm_s32(_ptr(Xq), _ptr(Wq), M, N, K, _ptr(acc), _stream(stream)))
    return acc


def sq_device_status(clear: bool = False) -> int:
    """Device status flags (bit 0: a GEMM pipeline wait timed out).  Syncs the device."""
    v = ctypes.c_uint32(0)
    st = _load().sq_device_status(ctypes.byref(v), 1 if clear else 0)
    if st not in (0, 7):
        _check(st)
    return int(v.value)


def sq_debug_fail_after(n: int) -> None:
    """Host-side fault injection: after n more launches, entry points fail with SQ_ERR_CUDA."""
    _load().sq_debug_fail_after(int(n))


def sq_debug_pipeline_stall(enable: bool, timeout_ns: int = 0) -> None:
    """Test hook: the general GEMM skips its first stage and its waits give up
    after timeout_ns, reporting bit 0 of the device status word (no GPU fault)."""
    _load().sq_debug_pipeline_stall(1 if enable else 0, int(timeout_ns))
