"""The GPU backward test's comparison rule, exercised on the CPU: an
emulation of the kernels' arithmetic (exact codes, G times a scale split into
two bf16 halves, fp32 products and sums, X times the rounded reciprocal of
s) passes it, and the same emulation with one planted kernel mistake fails
it.  This shows the bound is neither too tight for a correct kernel nor too
loose to see a wrong one."""
import numpy as np
import pytest
import torch

from oracle import smoothquant as O
from oracle import ste_backward as STE
from tests import test_gpu_ste as T


def _bf16(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def _split(v):
    v = np.asarray(v, np.float32)
    hi = _bf16(v)
    return hi, _bf16((v - hi).astype(np.float32))


def emulate(G, X, W, mx, alpha, mistake=None):
    r = STE.ste_backward(G, X, W, mx, np.float32(alpha))
    s = r["s"]
    Gv = O.widen_bf16(G)
    gh, gl = _split(Gv * r["w_scale"][None, :])
    gth, gtl = _split(Gv * r["x_scale"][:, None])
    Wc, Xc = r["Wq"].astype(np.float32), r["Xq"].astype(np.float32)
    dXs = (gh @ Wc + gl @ Wc).astype(np.float32)
    dWs = (gth.T @ Xc + gtl.T @ Xc).astype(np.float32)
    if mistake == "hi_only":
        dXs = (gh @ Wc).astype(np.float32)
    rs = (np.float32(1) / s).astype(np.float32)
    dX = (dXs * (s if mistake == "dX_times_s" else rs)[None, :]).astype(np.float32)
    dW = (dWs * s[None, :]).astype(np.float32)
    db = Gv.sum(axis=0, dtype=np.float32)
    Xv, Wv = O.widen_bf16(X), O.widen_bf16(W)
    errX = (Xv * rs[None, :]).astype(np.float32) - Xc * r["x_scale"][:, None]
    errW = (Wv * s[None, :]).astype(np.float32) - Wc * r["w_scale"][:, None]
    tx = (dXs * errX).sum(axis=0, dtype=np.float32)
    tw = (dWs * errW).sum(axis=0, dtype=np.float32)
    if mistake == "ds_sign":
        tx = -tx
    mw = np.abs(Wv).max(axis=0)
    raw, mxc, mwc = STE.raw_smoothing(mx, mw, alpha)
    ds = (tw.astype(np.float64) - tx) / s
    L = np.log(mxc) + np.log(mwc)
    if mistake == "no_clamp_mask":
        keep = np.ones_like(raw, dtype=bool)
    else:
        keep = raw >= float(O.CLAMP_FLOOR)
    d_eta = float(np.float32(alpha * (1 - alpha) * np.sum(np.where(keep, ds * raw * L, 0.0))))
    return r, dX, dW, db, ds.astype(np.float32), d_eta


def _case(clamped=False):
    G, X, W, mx = T._inputs(24, 64, 96, seed=777)
    if clamped:
        from tests.oracle_pins import bits
        Wv = O.widen_bf16(W)
        Wv[:, 9] *= 2.0 ** 40
        W = bits(Wv)
        mx = mx.copy()
        mx[9] = 0.0
    return G, X, W, mx, float(STE.alpha_from_logit(0.3))


def test_emulated_kernel_passes():
    for clamped in (False, True):
        G, X, W, mx, alpha = _case(clamped)
        r, dX, dW, db, ds, d_eta = emulate(G, X, W, mx, alpha)
        T.compare(G, X, W, mx, alpha, r, dX, dW, db, ds, d_eta, "emulated")


@pytest.mark.parametrize("mistake", ["hi_only", "dX_times_s", "ds_sign", "no_clamp_mask"])
def test_planted_kernel_mistake_fails(mistake):
    G, X, W, mx, alpha = _case(clamped=mistake == "no_clamp_mask")
    r, dX, dW, db, ds, d_eta = emulate(G, X, W, mx, alpha, mistake)
    with pytest.raises(AssertionError):
        T.compare(G, X, W, mx, alpha, r, dX, dW, db, ds, d_eta, mistake)
