"""The learnable-alpha straight-through backward on the GPU (through the C
ABI) against its CPU oracle.

The forward values (s, codes, scales) come from the library's own forward
calls, which other tests hold bit-exact to the oracle; here they must equal
the oracle's again, and the gradients must lie within the error bound the
kernels' arithmetic allows.  The two products take the codes as exact bf16
operands and G times a scale split into two bf16 halves (2^-16 relative, after
the scale's own fp32 product), accumulated in fp32 over 2C products (at most
2C * 2^-22 of the sum of absolute products, a worst-case bound that allows
round-toward-zero accumulation), then one fp32 product (dW) or a product with the rounded reciprocal of s (dX).
ds_k s_k is formed from the quantisation errors, so its bound is that
relative error times sum |dWs| |W s - Wdq| + sum |dXs| |X/s - Xdq|, plus the
fp32 rounding of W s and X / s and the fp32 sums of N and M such terms.
d eta is checked twice: against the oracle under the propagated bound, and
against alpha (1 - alpha) sum ds raw (ln mx + ln mw) evaluated in float64
from the kernel's own ds (the reduction alone, within fp32 rounding)."""
import numpy as np
import pytest
import torch

import workloads
from oracle import smoothquant as O
from oracle import ste_backward as STE
from tests.helpers import dev, dev_bf16, host

pytestmark = pytest.mark.gpu

OPERAND = 2.0 ** -16 + 2.0 ** -23   # hi + lo of an fp32-rounded product of the dequantised code (after its fp32 product)


@pytest.fixture(scope="module")
def sq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import w8a8_smoothquant_int8_sq_b200 as m
    return m


def _run(sq, G, X, W, mx, eta, label, with_db=True):
    M, K = X.shape
    N = W.shape[0]
    alpha = float(STE.alpha_from_logit(eta))
    Wd, Xd = dev_bf16(W), dev_bf16(X)
    mx_d = dev(np.asarray(mx, np.float32).copy())
    s = sq.sq_calibrate(None, Wd, alpha, mx_inout=mx_d)
    Wq, ws = sq.sq_prepare_weight(Wd, s)
    Xq, xs = sq.sq_quantize_act(Xd, s)
    dX, dW, db, ds, d_eta = sq.sq_ste_backward(dev_bf16(G), Xd, Wd, s, mx_d, alpha, Xq, xs, Wq, ws, with_db=with_db,
                                               with_ds=True)
    torch.cuda.synchronize()
    assert sq.sq_device_status() == 0
    r = STE.ste_backward(G, X, W, mx, np.float32(alpha))
    assert np.array_equal(host(s), r["s"]), f"{label}: s"
    assert np.array_equal(host(Wq), r["Wq"]) and np.array_equal(host(ws), r["w_scale"]), f"{label}: weight codes"
    assert np.array_equal(host(Xq), r["Xq"]) and np.array_equal(host(xs), r["x_scale"]), f"{label}: act codes"
    compare(G, X, W, mx, alpha, r, host(dX), host(dW), None if db is None else host(db), host(ds),
            float(host(d_eta)[0]), label, with_db)


def compare(G, X, W, mx, alpha, r, dX, dW, db, ds, d_eta, label, with_db=True):
    """Element-wise comparison of a backward's results with the oracle's
    ``r`` under the bound described in the module docstring."""
    M, K = X.shape
    N = W.shape[0]
    e = STE.ste_error_scales(G, X, W, r)
    s64 = r["s"].astype(np.float64)
    gx = OPERAND + 2 * N * 2.0 ** -22 * (1 + 2.0 ** -7)   # contraction over N (hi and lo products)
    gw = OPERAND + 2 * M * 2.0 ** -22 * (1 + 2.0 ** -7)   # contraction over M
    worst = {}

    def check(name, got, ref, bound):
        ratio = np.abs(np.asarray(got, np.float64) - ref) / np.maximum(bound, 1e-300)
        worst[name] = float(ratio.max()) if ratio.size else 0.0
        assert worst[name] <= 1.0, f"{label}: {name} error {worst[name]:.3f} of the bound"

    # dX = dXs * RN(1/s): two roundings after the product
    check("dX", dX, r["dX"], gx * e["aXs"] / s64[None, :] * (1 + 2.0 ** -22) + 2.0 ** -22 * np.abs(r["dX"]))
    check("dW", dW, r["dW"], gw * e["aWs"] * s64[None, :] + 2.0 ** -24 * np.abs(r["dW"]))
    if with_db:
        Ga = np.abs(O.widen_bf16(G).astype(np.float64)).sum(axis=0)
        check("db", db, r["db"], (M + 2) * 2.0 ** -24 * Ga + 1e-30)
    else:
        assert db is None
    Xv = O.widen_bf16(X).astype(np.float64)
    Wv = O.widen_bf16(W).astype(np.float64)
    # bound of T_k = ds_k s_k: product errors times the quantisation errors, the
    # fp32 rounding of W*s and X/s, and the fp32 sums over N and M terms
    round_terms = (e["aWs"] * np.abs(Wv) * s64[None, :]).sum(axis=0) + (e["aXs"] * np.abs(Xv) / s64[None, :]).sum(axis=0)
    aT_w = (e["aWs"] * np.abs(e["dW_q"])).sum(axis=0)
    aT_x = (e["aXs"] * np.abs(e["dX_q"])).sum(axis=0)
    # (X/s is formed as X * RN(1/s): two roundings, hence 2^-22 on the X terms)
    bT = gw * aT_w + gx * aT_x + 2.0 ** -22 * round_terms + (N + M + 4) * 2.0 ** -24 * (aT_w + aT_x)
    check("ds", ds, r["ds"], bT / s64 + 2.0 ** -23 * np.abs(r["ds"]))
    raw, mxc, mwc = STE.raw_smoothing(mx, r["mw"], alpha)
    Ls = np.log(mxc) + np.log(mwc)
    L = np.abs(Ls)
    b_eta = alpha * (1 - alpha) * np.sum(np.where(r["passes"], bT / s64 * raw * L, 0.0))
    check("d_eta", d_eta, r["deta"], b_eta + 2.0 ** -23 * abs(r["deta"]))
    # the reduction alone, from the kernel's ds (rounded to fp32 on output)
    terms = np.where(r["passes"], ds.astype(np.float64) * raw * Ls, 0.0)
    own = alpha * (1 - alpha) * terms.sum()
    check("d_eta_sum", d_eta, own, 2.0 ** -23 * (abs(own) + alpha * (1 - alpha) * np.abs(terms).sum()) + 1e-38)
    print(f"\n[ste backward] {label}: error / bound " + ", ".join(f"{k} {v:.3f}" for k, v in worst.items())
          + f"; d_eta {d_eta:.6g} (oracle {r['deta']:.6g}, relative error {abs(d_eta - r['deta']) / max(abs(r['deta']), 1e-30):.2e})")


def _inputs(M, N, K, seed, outliers=True):
    X = workloads.random_bf16((M, K), seed=seed, scale=1.0, outlier_cols=[K // 3] if outliers else None,
                              outlier_scale=40.0)
    W = workloads.random_bf16((N, K), seed=seed + 1, scale=0.02)
    C = workloads.random_bf16((max(M, 8), K), seed=seed + 2, scale=1.0,
                              outlier_cols=[K // 3] if outliers else None, outlier_scale=40.0)
    G = workloads.random_bf16((M, N), seed=seed + 3, scale=1e-3)
    mx = O.column_max_abs(O.widen_bf16(C))
    return G, X, W, mx


def test_tiny_workload(sq):
    wl = workloads.get("tiny")
    inp = workloads.make_inputs(wl, ("X", "C", "W"))
    G = workloads.random_bf16((wl.M, wl.N), seed=wl.index * 1000 + 9, scale=1e-3)
    mx = O.column_max_abs(O.widen_bf16(inp["C"]))
    _run(sq, G, inp["X"], inp["W"], mx, 0.0, "tiny 16x256x256")


def test_proj_workload(sq):
    wl = workloads.get("proj")
    inp = workloads.make_inputs(wl, ("X", "C", "W"))
    G = workloads.random_bf16((wl.M, wl.N), seed=wl.index * 1000 + 9, scale=1e-3)
    mx = O.column_max_abs(O.widen_bf16(inp["C"]))
    _run(sq, G, inp["X"], inp["W"], mx, 0.4, "proj 512x4096x4096")


@pytest.mark.parametrize("M,N,K,eta,with_db", [
    (1, 8, 16, 0.0, True),          # one token, the smallest N and K
    (3, 200, 48, -1.2, False),      # ragged everything, no db
    (130, 136, 4112, 0.7, True),    # tile overhangs in k, m and n
    (64, 264, 640, 2.0, True),      # alpha near 0.88
])
def test_ragged(sq, M, N, K, eta, with_db):
    G, X, W, mx = _inputs(M, N, K, seed=M * 7 + N + K)
    _run(sq, G, X, W, mx, eta, f"{M}x{N}x{K}", with_db=with_db)


def test_clamped_channel(sq):
    """A channel whose s sits on the 1e-8 clamp contributes nothing to d eta."""
    M, N, K = 5, 64, 32
    G, X, W, mx = _inputs(M, N, K, seed=4242)
    Wv = O.widen_bf16(W)
    Wv[:, 9] *= 2.0 ** 40
    from tests.oracle_pins import bits
    W = bits(Wv)
    mx = mx.copy()
    mx[9] = 0.0
    r = STE.ste_backward(G, X, W, mx, STE.alpha_from_logit(0.3))
    assert not r["passes"][9]
    _run(sq, G, X, W, mx, 0.3, "clamped channel")
