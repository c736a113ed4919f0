"""Plants plausible mistakes in (a copy of) the oracle on the CPU and checks that
the pins in test_oracle.py catch each of them. A pin set that a mutant survives
would not be pinning the oracle."""
import numpy as np
import pytest

from oracle import rglru_oracle as orc
import tests.test_oracle as pins


def _flip_taps(x, conv_w, conv_state=None):
    return orc_conv4(x, conv_w[::-1], conv_state)


def _transposed_gate(u, W, b):
    return orc_gate(u, np.swapaxes(W, 1, 2), b)


def _softplus_wrong_sign(r, Lambda):
    return -orc.C_DECAY * r * orc.softplus(Lambda)[None, None, :]


def _c_is_4(r, Lambda):
    return -4.0 * r * orc.softplus(-Lambda)[None, None, :]


def _sqrt_one_minus_a(log_a, i, u):
    return np.sqrt(-np.expm1(log_a)) * (i * u)


def _drop_u(log_a, i, u):
    return np.sqrt(-np.expm1(2.0 * log_a)) * i


def _scan_off_by_one(a, beta, h0=None):
    B, T, D = a.shape
    h = np.zeros((B, D)) if h0 is None else np.array(h0, dtype=np.float64)
    out = np.empty((B, T, D))
    for t in range(T):
        h = a[:, max(t - 1, 0), :] * h + beta[:, t, :]
        out[:, t, :] = h
    return out


def _ring_rotated_wrong(ring, pos):
    ring = orc.as_f64(ring)
    return ring[:, [(pos + 1 + k) % 3 for k in range(3)], :]


def _decode_writes_wrong_slot(x_t, ring, pos, h, conv_w, W_a, b_a, W_x, b_x, Lambda,
                              gate_operand=None):
    y, h_new, ring_new = orc_decode(x_t, ring, pos, h, conv_w, W_a, b_a, W_x, b_x, Lambda,
                                    gate_operand)
    ring_new = orc.as_f64(ring).copy()
    ring_new[:, (pos + 1) % 3, :] = orc.as_f64(x_t)
    return y, h_new, ring_new


orc_conv4 = orc.conv4
orc_gate = orc.gate_preacts
orc_decode = orc.rglru_decode_step

MUTANTS = {
    "conv taps reversed": ("conv4", _flip_taps),
    "gate weight transposed": ("gate_preacts", _transposed_gate),
    "softplus(+Lambda)": ("log_decay", _softplus_wrong_sign),
    "c = 4": ("log_decay", _c_is_4),
    "sqrt(1 - a) normaliser": ("gated_input", _sqrt_one_minus_a),
    "input term drops u": ("gated_input", _drop_u),
    "scan uses a_{t-1}": ("linear_scan", _scan_off_by_one),
    "decode ring read in the wrong order": ("ring_to_chronological", _ring_rotated_wrong),
    "decode overwrites the wrong ring slot": ("rglru_decode_step", _decode_writes_wrong_slot),
}

PIN_TESTS = [
    lambda: pins.test_conv4_matches_torch_conv1d(True),
    pins.test_gate_orientation_not_transposed,
    pins.test_gates_match_dense_block_diagonal,
    pins.test_full_gate_gives_a_to_the_c,
    pins.test_a_sixteenth_closed_form,
    pins.test_constant_gates_geometric_sum,
    pins.test_scan_bruteforce_unrolled,
    lambda: pins.test_chunked_and_sequential_scans_agree(7),
    pins.test_second_moment_is_preserved,
    pins.test_stationary_worst_case_bound,
    lambda: pins.test_decode_steps_compose_with_fwd(0),
    lambda: pins.test_decode_steps_compose_with_fwd(3),
]


def test_pins_pass_on_the_unchanged_oracle():
    for pin in PIN_TESTS:
        pin()


@pytest.mark.parametrize("name", ["decode ring read in the wrong order",
                                  "decode overwrites the wrong ring slot"])
def test_decode_pin_alone_catches_ring_mutants(name, monkeypatch):
    """The fwd/decode composition pin on its own catches both ring mistakes."""
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(orc, attr, fn)
    with pytest.raises(AssertionError):
        pins.test_decode_steps_compose_with_fwd(3)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(orc, attr, fn)
    caught = 0
    for pin in PIN_TESTS:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin caught the mutant '{name}'"
