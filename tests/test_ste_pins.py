"""The learnable-alpha backward oracle against its pins, and planted mistakes
that the pins must catch."""
import numpy as np
import pytest

from oracle import smoothquant as SQ
from oracle import ste_backward as STE
from tests import ste_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(STE.ste_backward)


def test_sigmoid():
    P.pin_sigmoid()


# --------------------------------------------------------------- planted mistakes
def _mutant(kind):
    """ste_backward with one step changed."""
    def bwd(G_bits, X_bits, W_bits, mx, alpha):
        r = dict(STE.ste_backward(G_bits, X_bits, W_bits, mx, alpha))
        G = SQ.widen_bf16(np.asarray(G_bits)).astype(np.float64)
        X = SQ.widen_bf16(np.asarray(X_bits)).astype(np.float64)
        W = SQ.widen_bf16(np.asarray(W_bits)).astype(np.float64)
        s = r["s"].astype(np.float64)
        Xdq = r["Xq"].astype(np.float64) * r["x_scale"].astype(np.float64)[:, None]
        dXs, dWs = r["dXs"], r["dWs"]
        if kind == "dX_times_s":
            r["dX"] = dXs * s[None, :]
        if kind == "dW_over_s":
            r["dW"] = dWs / s[None, :]
        if kind == "dWs_from_unquantised_X":
            dWs = G.T @ (X / s[None, :])
            r["dW"] = dWs * s[None, :]
        if kind == "db_over_rows_of_G_T":
            r["db"] = G.sum(axis=1)[: G.shape[1]] if G.shape[0] >= G.shape[1] else np.resize(G.sum(axis=1), G.shape[1])
        pw = (dWs * W).sum(axis=0)
        px = (dXs * X).sum(axis=0)
        ds = pw - px / (s * s)
        if kind == "ds_sign":
            ds = pw + px / (s * s)
        if kind == "ds_over_s":
            ds = pw - px / s
        r["ds"] = ds
        raw, mxc, mwc = STE.raw_smoothing(mx, r["mw"], alpha)
        L = np.log(mxc) + np.log(mwc)
        if kind == "drop_ln_mw":
            L = np.log(mxc)
        passes = raw >= float(SQ.CLAMP_FLOOR)
        if kind == "no_clamp_mask":
            passes = np.ones_like(passes)
        dalpha = float(np.sum(np.where(passes, ds * raw * L, 0.0)))
        a = float(alpha)
        r["dalpha"] = dalpha
        r["deta"] = dalpha if kind == "no_sigmoid_factor" else a * (1.0 - a) * dalpha
        return r
    return bwd


MUTANTS = ["dX_times_s", "dW_over_s", "dWs_from_unquantised_X", "db_over_rows_of_G_T", "ds_sign", "ds_over_s",
           "drop_ln_mw", "no_clamp_mask", "no_sigmoid_factor"]


def test_unmutated_harness_passes():
    for pin in P.ALL_PINS:
        pin(_mutant("none"))


@pytest.mark.parametrize("kind", MUTANTS)
def test_mutant_is_caught(kind):
    caught = []
    for pin in P.ALL_PINS:
        try:
            pin(_mutant(kind))
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches {kind}"
