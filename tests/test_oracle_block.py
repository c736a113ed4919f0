"""Pins of the recurrent-block oracle (oracle/block_oracle.py) by facts that do
not come from it: values of the standard normal distribution function, GeLU's
odd-part identity and a brute-force integral of the normal density; a zero
gate weight; reduction to the separately pinned layer oracle when both
projections are identities; linearity in the output projection. Each pin is
also run against planted mistakes (on the CPU) that it must catch.
"""
import numpy as np
import pytest

from gated_linear_recurrence_rglru_b200.workloads import WORKLOADS, generate_block
from oracle import block_oracle as bo
from oracle import rglru_oracle as ro

# Phi(v) of the standard normal distribution (tables of the normal integral)
PHI = {0.0: 0.5, 1.0: 0.8413447460685429, -1.0: 0.15865525393145707, 2.0: 0.9772498680518208,
       -2.0: 0.022750131948179195, 0.5: 0.6914624612740131}


def _params(Dm, D, H, T=40, B=2, seed=5):
    wl = WORKLOADS["tiny_f32"].with_shape(B=B, T=T, D=D, H=H, h0_var=0.5, bias_std=0.3, seed=seed)
    return generate_block(wl, Dm)


def _layer_args(t):
    return [t[k] for k in ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")]


# ---- pins, each a function of (gelu, block) so that mutants can be run through them ----

def pin_gelu_values(gelu, block):
    for v, phi in PHI.items():
        assert abs(gelu(v) - v * phi) <= 1e-15 * max(1.0, abs(v)), v


def pin_gelu_odd_part(gelu, block):
    v = np.linspace(-6, 6, 101)
    assert np.allclose(gelu(v) - gelu(-v), v, rtol=0, atol=1e-14)


def pin_gelu_integral(gelu, block):
    # Phi(v) as the integral of the density from -12 (Simpson, fine grid)
    for v in (-1.7, -0.3, 0.4, 1.3, 2.6):
        s = np.linspace(-12.0, v, 20001)
        f = np.exp(-0.5 * s * s) / np.sqrt(2 * np.pi)
        h = s[1] - s[0]
        phi = h / 3 * (f[0] + f[-1] + 4 * f[1:-1:2].sum() + 2 * f[2:-1:2].sum())
        assert abs(gelu(v) - v * phi) < 1e-10, v


def pin_zero_gate(gelu, block):
    t = _params(16, 32, 2)
    out, _, _ = block(t["x"], t["W_in"], 0 * t["W_gate"], t["W_out"], *_layer_args(t),
                      h0=t["h0"])
    assert np.all(out == 0.0)


def pin_identity_projections(gelu, block):
    D = 32
    t = _params(D, D, 2)
    eye = np.eye(D)
    out, hT, cs = block(t["x"], eye, t["W_gate"], eye, *_layer_args(t), h0=t["h0"])
    y, hT_ref, cs_ref = ro.rglru_fwd(t["x"], *_layer_args(t), h0=t["h0"])
    x64 = ro.as_f64(t["x"])
    g = x64 @ ro.as_f64(t["W_gate"])
    # with the gate pinned above: out = layer(x) * v Phi(v), Phi from the table-free erf of scipy
    from scipy.stats import norm
    assert np.allclose(out, y * g * norm.cdf(g), rtol=1e-12, atol=1e-12)
    assert np.allclose(hT, hT_ref, rtol=1e-12, atol=0)


def pin_output_linearity(gelu, block):
    Dm, D = 24, 32
    t = _params(Dm, D, 2)
    rng = np.random.default_rng(3)
    M = rng.standard_normal((D, Dm))
    eye_out = np.eye(D)
    pre, _, _ = block(t["x"], t["W_in"], t["W_gate"], eye_out, *_layer_args(t), h0=t["h0"])
    out, _, _ = block(t["x"], t["W_in"], t["W_gate"], M, *_layer_args(t), h0=t["h0"])
    assert np.allclose(out, pre @ M, rtol=1e-12, atol=1e-12)


PINS = [pin_gelu_values, pin_gelu_odd_part, pin_gelu_integral, pin_zero_gate,
        pin_identity_projections, pin_output_linearity]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_block_oracle_pins(pin):
    pin(bo.gelu, bo.block_fwd)


# ---- planted mistakes ----

def _gelu_tanh(v):
    v = np.asarray(v, dtype=np.float64)
    return 0.5 * v * (1 + np.tanh(np.sqrt(2 / np.pi) * (v + 0.044715 * v ** 3)))


def _block_with(gelu=bo.gelu, swap_branches=False, gate_before_layer=False, transpose_out=False):
    def block(x, W_in, W_gate, W_out, conv_w, W_a, b_a, W_x, b_x, Lambda, h0=None,
              conv_state=None):
        x64 = ro.as_f64(x)
        Wi, Wg, Wo = ro.as_f64(W_in), ro.as_f64(W_gate), ro.as_f64(W_out)
        if swap_branches:
            Wi, Wg = Wg, Wi
        g = gelu(x64 @ Wg)
        v = x64 @ Wi
        if gate_before_layer:
            y, hT, cs = ro.rglru_fwd(v * g, conv_w, W_a, b_a, W_x, b_x, Lambda, h0=h0)
            pre = y
        else:
            y, hT, cs = ro.rglru_fwd(v, conv_w, W_a, b_a, W_x, b_x, Lambda, h0=h0)
            pre = y * g
        Wo2 = Wo.T if transpose_out and Wo.shape[0] == Wo.shape[1] else Wo
        if transpose_out and Wo.shape[0] != Wo.shape[1]:
            Wo2 = Wo[::-1]                              # a wrong row order of W_out
        return pre @ Wo2, hT, cs
    return block


MUTANTS = {
    "tanh_gelu": (_gelu_tanh, _block_with(gelu=_gelu_tanh)),
    "swapped_branches": (bo.gelu, _block_with(swap_branches=True)),
    "gate_before_layer": (bo.gelu, _block_with(gate_before_layer=True)),
    "wrong_output_projection": (bo.gelu, _block_with(transpose_out=True)),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_block_mutants_are_caught(name):
    gelu, block = MUTANTS[name]
    caught = 0
    for pin in PINS:
        try:
            pin(gelu, block)
        except AssertionError:
            caught += 1
    assert caught > 0, name


def test_block_oracle_runs_the_workload_recipe_shapes():
    t = _params(16, 32, 2, T=9)
    out, hT, cs = bo.block_fwd(t["x"], t["W_in"], t["W_gate"], t["W_out"], *_layer_args(t),
                               h0=t["h0"])
    assert out.shape == (2, 9, 16) and hT.shape == (2, 32) and cs.shape == (2, 3, 32)
    assert np.all(np.isfinite(out))
