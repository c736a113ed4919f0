"""Plants plausible mistakes in a copy of the backward oracle (on the CPU) and
checks that the pins of test_oracle_backward.py catch each of them."""
import inspect
import types

import numpy as np
import pytest

import oracle.rglru_backward as bwd_mod
import tests.test_oracle_backward as pins

MUTANTS = {
    "drops the g path of d la": ("(C_DECAY * sp) * (a * a) * (1.0 - r) * d_g * r_over_g", "0.0"),
    "sign of d Lambda": ("dLambda = d_sp * (-sigmoid(-L))", "dLambda = d_sp * sigmoid(-L)"),
    "reverse scan uses a_{t-1}": ("carry = a[:, t, :] * carry", "carry = a[:, max(t - 1, 0), :] * carry"),
    "d h_prev uses h_t": ("d_a = G * h_prev", "d_a = G * h"),
    "gate W not transposed in d u": ("W.transpose(0, 2, 1)", "W"),
    "conv taps reversed in d x": ("dxp[:, k:k + T, :] += w64[k]", "dxp[:, k:k + T, :] += w64[3 - k]"),
    "d i misses u": ("d_i = d_beta * g * u", "d_i = d_beta * g"),
}


def _mutant(old, new):
    src = inspect.getsource(bwd_mod)
    assert src.count(old) >= 1, old
    mod = types.ModuleType("mutant_bwd")
    mod.__dict__["__package__"] = "oracle"
    exec(compile(src.replace(old, new), "mutant_bwd", "exec"), mod.__dict__)
    return mod.rglru_bwd


def _pins_pass(fn):
    orig = pins.rglru_bwd
    pins.rglru_bwd = fn
    try:
        for name in sorted(pins.GRAD_OF):
            pins.test_directional_finite_differences(name, 0)
        pins.test_r_zero_holds_the_state()
        pins.test_constant_gate_dh0_closed_form()
        pins.test_linear_in_output_gradients()
        return True
    except AssertionError:
        return False
    finally:
        pins.rglru_bwd = orig


def test_pins_pass_on_the_oracle():
    assert _pins_pass(bwd_mod.rglru_bwd)


@pytest.mark.parametrize("label", sorted(MUTANTS))
def test_pins_catch_mutant(label):
    old, new = MUTANTS[label]
    assert not _pins_pass(_mutant(old, new)), label
