"""Pins for the float64 oracle (CPU only).

Each test checks the oracle against something that does not come from the
oracle itself: a library routine (torch Conv1D, torch.block_diag matmul,
numpy logaddexp), a closed form, a brute-force unrolled sum, an invariant of
the recurrence, or a composition of two of its own entry points along
different routes. Each is chosen so that a plausible slip (a dropped term, a
flipped sign, a shifted tap, a transposed weight) fails at least one test.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from gated_linear_recurrence_rglru_b200.workloads import WORKLOADS, generate, lambda_from_ac
from oracle import rglru_oracle as orc
from oracle.compare import FLOOR, max_rel_err

RNG = np.random.default_rng(1234)


def rand(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


def small_params(B=2, T=9, D=12, H=3, bias=0.3):
    bw = D // H
    return dict(
        x=rand(B, T, D), conv_w=rand(4, D, scale=0.5),
        W_a=rand(H, bw, bw, scale=1 / math.sqrt(bw)), b_a=rand(D, scale=bias),
        W_x=rand(H, bw, bw, scale=1 / math.sqrt(bw)), b_x=rand(D, scale=bias),
        Lambda=rand(D, scale=2.0) + 3.0)


# ---------------------------------------------------------------- conv4 ----

@pytest.mark.parametrize("with_state", [False, True])
def test_conv4_matches_torch_conv1d(with_state):
    B, T, D = 3, 17, 10
    x, w = rand(B, T, D), rand(4, D)
    state = rand(B, 3, D) if with_state else None
    u = orc.conv4(x, w, state)
    # torch conv1d is a cross-correlation: out[t] = sum_k weight[k] * in[t + k].
    hist = torch.zeros(B, D, 3, dtype=torch.float64) if state is None else \
        torch.from_numpy(state).permute(0, 2, 1)
    inp = torch.cat([hist, torch.from_numpy(x).permute(0, 2, 1)], dim=2)
    ref = F.conv1d(inp, torch.from_numpy(w).T.unsqueeze(1).contiguous(), groups=D)
    np.testing.assert_allclose(u, ref.permute(0, 2, 1).numpy(), rtol=0, atol=1e-13)


def test_conv4_identity_taps():
    x = rand(2, 5, 4)
    w = np.zeros((4, 4)); w[3] = 1.0
    np.testing.assert_array_equal(orc.conv4(x, w), x)
    w = np.zeros((4, 4)); w[0] = 1.0          # pure 3-step delay
    u = orc.conv4(x, w)
    np.testing.assert_array_equal(u[:, 3:], x[:, :-3])
    np.testing.assert_array_equal(u[:, :3], 0.0)


# ---------------------------------------------------------------- gates ----

def test_gates_match_dense_block_diagonal():
    B, T, D, H = 2, 5, 12, 3
    bw = D // H
    u, W, b = rand(B, T, D), rand(H, bw, bw), rand(D)
    dense = torch.block_diag(*[torch.from_numpy(W[h]) for h in range(H)]).numpy()
    ref = u @ dense + b
    np.testing.assert_allclose(orc.gate_preacts(u, W, b), ref, rtol=0, atol=1e-12)


def test_gate_orientation_not_transposed():
    # One nonzero weight W[0, i=0, j=1]: input channel 0 must drive output channel 1 only.
    u = np.zeros((1, 1, 4)); u[0, 0, 0] = 2.0
    W = np.zeros((1, 4, 4)); W[0, 0, 1] = 3.0
    z = orc.gate_preacts(u, W, np.zeros(4))
    np.testing.assert_array_equal(z[0, 0], [0.0, 6.0, 0.0, 0.0])


def test_sigmoid_softplus_library_values():
    v = np.array([-800.0, -30.0, -1.0, 0.0, 1e-9, 2.5, 40.0, 800.0])
    np.testing.assert_allclose(orc.softplus(v), np.logaddexp(0.0, v), rtol=1e-15, atol=0)
    assert orc.softplus(np.array([0.0]))[0] == pytest.approx(math.log(2.0), rel=1e-16)
    assert orc.sigmoid(np.array([0.0]))[0] == 0.5
    # sigmoid via a different library route: tanh identity
    z = np.linspace(-8, 8, 33)                # (cancellation in 1 + tanh limits the range)
    np.testing.assert_allclose(orc.sigmoid(z), 0.5 * (1 + np.tanh(z / 2)), rtol=1e-12)
    assert orc.sigmoid(np.array([-1e4]))[0] == 0.0 and orc.sigmoid(np.array([1e4]))[0] == 1.0


# ---------------------------------------------------------------- decay ----

def test_full_gate_gives_a_to_the_c():
    """r_t = 1 must give a_t = sigmoid(Lambda)^8 (the 'a^c' of the method, c = 8)."""
    D = 6
    s = torch.tensor([0.9, 0.95, 0.99, 0.999, 0.9999, 0.5], dtype=torch.float64)
    Lam = lambda_from_ac(s).double().numpy()
    r = np.ones((1, 1, D))
    a = np.exp(orc.log_decay(r, Lam))[0, 0]
    sig = 1.0 / (1.0 + np.exp(-Lam))
    np.testing.assert_allclose(a, sig ** 8, rtol=1e-13)
    np.testing.assert_allclose(a, s.numpy(), rtol=2e-6)   # Lambda is stored in fp32


def test_a_sixteenth_closed_form():
    """Lambda = 0 (a = 1/2), z = 0 (r = i = 1/2): a_t = 2^-4, beta = sqrt(255/256) * u / 2."""
    B, T, D, H = 1, 8, 4, 2
    bw = D // H
    x = np.full((B, T, D), 2.0)
    w = np.zeros((4, D)); w[3] = 1.0
    Z = np.zeros((H, bw, bw))
    h0 = np.array([[1.0, -3.0, 0.0, 0.5]])
    y, hT, _ = orc.rglru_fwd(x, w, Z, np.zeros(D), Z, np.zeros(D), np.zeros(D), h0=h0)
    a = 1.0 / 16.0
    beta = math.sqrt(255.0) / 16.0          # sqrt(1 - 1/256) * (1/2) * 2
    t = np.arange(1, T + 1)[:, None]
    ref = a ** t * h0 + beta * (1 - a ** t) / (1 - a)
    np.testing.assert_allclose(y[0], ref, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(hT, ref[-1:], rtol=1e-14)


def test_zero_recurrence_gate_holds_state():
    """r_t = 0 => a_t = 1 and sqrt(1 - a_t^2) = 0: h_t = h0 exactly, whatever x."""
    p = small_params()
    D = p["x"].shape[2]
    p["b_a"] = np.full(D, -1e4)
    p["W_a"] = np.zeros_like(p["W_a"])
    h0 = rand(2, D)
    y, hT, _ = orc.rglru_fwd(h0=h0, **p)
    np.testing.assert_array_equal(y, np.broadcast_to(h0[:, None, :], y.shape))
    np.testing.assert_array_equal(hT, h0)


def test_constant_gates_geometric_sum():
    B, T, D, H = 2, 40, 6, 2
    bw = D // H
    c = rand(B, 1, D)
    x = np.repeat(c, T, axis=1)
    w = np.zeros((4, D)); w[3] = 1.0
    Z = np.zeros((H, bw, bw))
    b_a, b_x, Lam = rand(D), rand(D), rand(D) + 2.0
    h0 = rand(B, D)
    y, _, _ = orc.rglru_fwd(x, w, Z, b_a, Z, b_x, Lam, h0=h0)
    r = 1 / (1 + np.exp(-b_a)); i = 1 / (1 + np.exp(-b_x))
    a = (1 / (1 + np.exp(-Lam))) ** (8 * r)           # a^(c r) with a = sigmoid(Lambda)
    beta = np.sqrt(1 - a * a) * i * c[:, 0, :]
    t = np.arange(1, T + 1)[None, :, None]
    ref = a ** t * h0[:, None, :] + beta[:, None, :] * (1 - a ** t) / (1 - a)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- scan -----

def test_scan_bruteforce_unrolled():
    p = small_params(B=2, T=14, D=8, H=2)
    h0 = rand(2, 8)
    it = orc.intermediates(**p)
    a, beta = it["a"], it["beta"]
    y = orc.linear_scan(a, beta, h0)
    B, T, D = a.shape
    for b in range(B):
        for d in range(D):
            for t in range(T):
                tot = math.prod(a[b, j, d] for j in range(t + 1)) * h0[b, d]
                for k in range(t + 1):
                    tot += math.prod(a[b, j, d] for j in range(k + 1, t + 1)) * beta[b, k, d]
                assert y[b, t, d] == pytest.approx(tot, rel=1e-12, abs=1e-14)


def _chunked_scan(a, beta, h0, L):
    """Two-level scan: per-chunk (prod a, local h) aggregates, carried across chunks."""
    B, T, D = a.shape
    out = np.empty_like(a)
    h_in = h0.copy()
    for s in range(0, T, L):
        A = np.ones((B, D)); Hl = np.zeros((B, D))
        loc, P = [], []
        for t in range(s, min(s + L, T)):
            Hl = a[:, t] * Hl + beta[:, t]
            A = A * a[:, t]
            loc.append(Hl.copy()); P.append(A.copy())
        for k, t in enumerate(range(s, min(s + L, T))):
            out[:, t] = loc[k] + P[k] * h_in            # fix-up with the carried state
        h_in = A * h_in + Hl                            # (A1,H1) o (A2,H2) combine
    return out


@pytest.mark.parametrize("L", [1, 2, 3, 7, 64])
def test_chunked_and_sequential_scans_agree(L):
    B, T, D = 2, 64, 5
    a = RNG.uniform(0.5, 1.0, (B, T, D)); beta = rand(B, T, D); h0 = rand(B, D)
    np.testing.assert_allclose(_chunked_scan(a, beta, h0, L), orc.linear_scan(a, beta, h0),
                               rtol=1e-13, atol=1e-13)


def test_second_moment_is_preserved():
    """a_t^2 + (1 - a_t^2) = 1: with iid unit-variance i*u, E h_t^2 = 1 - a^(2(t+1)) from h0 = 0."""
    B, T, D = 1, 60, 40000
    x = rand(B, T, D)
    w = np.zeros((4, D)); w[3] = 1.0                 # u = x
    Z = np.zeros((D, 1, 1))                          # H = D heads of width 1
    b_a = np.zeros(D)                                # r = 1/2
    b_x = np.full(D, 1e4)                            # i = 1
    s = torch.full((D,), 0.81, dtype=torch.float64)  # sigmoid(Lambda)^8 = 0.81 => a_t = 0.9
    Lam = lambda_from_ac(s).double().numpy()
    y, _, _ = orc.rglru_fwd(x, w, Z, b_a, Z, b_x, Lam)
    a = 0.81 ** 0.5
    t = np.arange(1, T + 1)
    ref = 1 - a ** (2 * t)
    got = (y[0] ** 2).mean(axis=1)
    np.testing.assert_allclose(got, ref, rtol=0.03)


def test_stationary_worst_case_bound():
    """beta~ = i*u = 1 for all t with constant a: h -> sqrt((1 + a) / (1 - a)) from below."""
    B, T, D = 1, 4000, 3
    x = np.ones((B, T, D))
    w = np.zeros((4, D)); w[3] = 1.0
    Z = np.zeros((1, D, D))
    b_a = np.full(D, 1e4)                            # r = 1 => a_t = sigmoid(Lambda)^8
    b_x = np.full(D, 1e4)                            # i = 1
    s = torch.tensor([0.5, 0.9, 0.99], dtype=torch.float64)
    Lam = lambda_from_ac(s).double().numpy()
    y, _, _ = orc.rglru_fwd(x, w, Z, b_a, Z, b_x, Lam)
    a = (1 / (1 + np.exp(-Lam))) ** 8
    lim = np.sqrt((1 + a) / (1 - a))
    assert np.all(y[0] <= lim * (1 + 1e-12))
    np.testing.assert_allclose(y[0, -1], lim, rtol=1e-9)


def test_per_step_bound_holds():
    p = small_params(B=3, T=50, D=16, H=4, bias=2.0)
    p["x"] *= 3
    it = orc.intermediates(**p)
    y = orc.linear_scan(it["a"], it["beta"])
    hprev = np.concatenate([np.zeros_like(y[:, :1]), y[:, :-1]], axis=1)
    bound = it["a"] * np.abs(hprev) + np.sqrt(1 - it["a"] ** 2) * np.abs(it["i"] * it["u"])
    assert np.all(np.abs(y) <= bound * (1 + 1e-12) + 1e-300)


# --------------------------------------------------- composition / decode --

def test_fwd_split_composition():
    p = small_params(B=2, T=20, D=8, H=2)
    h0 = rand(2, 8)
    y, hT, cs = orc.rglru_fwd(h0=h0, **p)
    for T1 in (1, 2, 3, 11):
        q = dict(p); q["x"] = p["x"][:, :T1]
        y1, h1, c1 = orc.rglru_fwd(h0=h0, **q)
        q["x"] = p["x"][:, T1:]
        y2, h2, c2 = orc.rglru_fwd(h0=h1, conv_state=c1, **q)
        np.testing.assert_allclose(np.concatenate([y1, y2], axis=1), y, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(h2, hT, rtol=1e-12, atol=1e-13)
        np.testing.assert_array_equal(c2, cs)


@pytest.mark.parametrize("T1", [0, 1, 3, 12])
def test_decode_steps_compose_with_fwd(T1):
    p = small_params(B=3, T=13, D=8, H=2)
    h0 = rand(3, 8)
    y, hT, cs = orc.rglru_fwd(h0=h0, **p)
    x = p["x"]
    w = {k: p[k] for k in ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")}
    if T1:
        _, h, ring = orc.rglru_fwd(x[:, :T1], h0=h0, **w)
    else:
        h, ring = h0, np.zeros((3, 3, 8))
    for k, t in enumerate(range(T1, x.shape[1])):
        y_t, h, ring = orc.rglru_decode_step(x[:, t], ring, k, h, **w)
        np.testing.assert_allclose(y_t, y[:, t], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(h, hT, rtol=1e-12, atol=1e-13)
    # after the last step the ring, read at the next position, is the chronological state
    np.testing.assert_array_equal(orc.ring_to_chronological(ring, x.shape[1] - T1), cs)


def test_conv_state_after_short_sequences():
    x = rand(1, 2, 3)
    cs = orc.conv_state_after(x)
    np.testing.assert_array_equal(cs[0, 0], 0.0)
    np.testing.assert_array_equal(cs[0, 1:], x[0])


# ----------------------------------------------------- workloads / metric --

def test_workload_recipe_statistics():
    wl = WORKLOADS["hawk_block"].with_shape(B=1, T=512, D=1024)
    t = generate(wl)
    assert t["x"].dtype == torch.bfloat16 and t["Lambda"].dtype == torch.float32
    assert abs(t["x"].float().std().item() - 1.0) < 0.01
    assert abs(t["W_a"].float().var().item() - 1 / 64) < 1e-3
    assert abs(t["conv_w"].float().var().item() - 1 / 4) < 0.03
    ac = torch.sigmoid(t["Lambda"].double()) ** 8
    assert ac.min() >= 0.9 - 1e-6 and ac.max() <= 0.999 + 1e-6
    assert t["h0"] is None and torch.all(t["b_a"] == 0)
    again = generate(wl)
    assert torch.equal(again["x"], t["x"]) and torch.equal(again["Lambda"], t["Lambda"])


def test_max_rel_err_measure():
    o = np.array([[[1.0, -2.0], [0.0, 2.0]]])             # (B=1, T=2, D=2)
    g = o.copy()
    assert max_rel_err(g, o) == 0.0
    g[0, 1, 0] = 0.1                                      # error at a zero of o: floored by channel rms
    rms0 = math.sqrt((1.0 + 0.0) / 2)
    assert max_rel_err(g, o) == pytest.approx(0.1 / (FLOOR * rms0))
    assert max_rel_err(g, o, floor=1.0) == pytest.approx(0.1 / rms0)
    g = o * 1.01
    assert max_rel_err(g, o) == pytest.approx(0.01)
    g[0, 0, 0] = np.nan
    assert max_rel_err(g, o) == float("inf")


def test_oracle_regression_fixture():
    """The oracle still reproduces the frozen fixture written by tests/golden/make_golden.py."""
    import os
    import sys
    sys.path.insert(0, os.path.join(os.path.dirname(__file__), "golden"))
    import make_golden
    t = make_golden.case_inputs()
    y, hT, _ = orc.rglru_fwd(t["x"], t["conv_w"], t["W_a"], t["b_a"], t["W_x"], t["b_x"],
                             t["Lambda"], h0=t["h0"])
    rows = np.loadtxt(os.path.join(os.path.dirname(__file__), "golden", "oracle_regression.txt"))
    B, T = make_golden.CASE["B"], make_golden.CASE["T"]
    np.testing.assert_allclose(y.reshape(B * T, -1), rows[:B * T], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(hT, rows[B * T:], rtol=1e-13, atol=1e-15)
