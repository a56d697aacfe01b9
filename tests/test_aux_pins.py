"""The auxiliary-loss oracle against its pins, and planted mistakes that the
pins must catch."""
import numpy as np
import pytest

from oracle import aux_loss as A
from oracle import smoothquant as SQ
from tests import aux_pins as P

ORACLE = (A.rel_mse, A.rel_mse_grad, A.add_aux_grad)


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(*ORACLE)


def _mutant(kind):
    """The oracle with one step changed."""
    def loss(yfp_bits, yq_bits):
        l, num, den = A.rel_mse(yfp_bits, yq_bits)
        if kind == "unsquared":
            l = np.sqrt(num) / max(np.sqrt(den), 1e-12)
        if kind == "den_of_y_q":
            yq = SQ.widen_bf16(yq_bits).astype(np.float64)
            l = num / max(float(np.sum(yq * yq)), A.DEN_FLOOR)
        if kind == "floor_on_norm_unsquared":
            l = num / max(den, 1e-12)
        return l, num, den

    def grad(yfp_bits, yq_bits):
        g = A.rel_mse_grad(yfp_bits, yq_bits)
        if kind == "grad_sign":
            g = -g
        if kind == "grad_without_2":
            g = g / 2.0
        if kind == "floor_on_norm_unsquared":
            yfp = SQ.widen_bf16(yfp_bits).astype(np.float64)
            yq = SQ.widen_bf16(yq_bits).astype(np.float64)
            g = 2.0 * (yq - yfp) / max(float(np.sum(yfp * yfp)), 1e-12)
        return g

    def add(G_bits, yfp_bits, yq_bits, lam):
        g = SQ.widen_bf16(G_bits).astype(np.float64) + lam * grad(yfp_bits, yq_bits)
        if kind == "drops_G":
            g = lam * grad(yfp_bits, yq_bits)
        return SQ.bf16_round(g)

    return loss, grad, add


def test_unmutated_harness_passes():
    for pin in P.ALL_PINS:
        pin(*_mutant("none"))


@pytest.mark.parametrize("kind", ["unsquared", "den_of_y_q", "floor_on_norm_unsquared", "grad_sign",
                                  "grad_without_2", "drops_G"])
def test_mutant_is_caught(kind):
    caught = False
    for pin in P.ALL_PINS:
        try:
            pin(*_mutant(kind))
        except AssertionError:
            caught = True
    assert caught, kind
