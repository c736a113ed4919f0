"""Pins of the backward oracle (oracle/rglru_backward.py) against facts that do
not come from it: central finite differences of the forward oracle along random
directions, the r = 0 closed form, the constant-gate closed form of d h0, and
linearity in (dy, dh_T)."""
import numpy as np
import pytest

from oracle import rglru_oracle as orc
from oracle.rglru_backward import rglru_bwd

B, T, D, H = 2, 9, 8, 2
BW = D // H


def _inputs(seed, r_zero=False):
    rng = np.random.default_rng(seed)
    p = dict(
        x=rng.normal(size=(B, T, D)),
        conv_w=rng.normal(size=(4, D)) * 0.5,
        W_a=rng.normal(size=(H, BW, BW)) * 0.4,
        b_a=rng.normal(size=D) * 0.3,
        W_x=rng.normal(size=(H, BW, BW)) * 0.4,
        b_x=rng.normal(size=D) * 0.3,
        Lambda=rng.uniform(1.0, 5.0, size=D),
        h0=rng.normal(size=(B, D)),
        conv_state=rng.normal(size=(B, 3, D)),
    )
    if r_zero:
        p["W_a"] = np.zeros((H, BW, BW))
        p["b_a"] = np.full(D, -1e4)
    dy = rng.normal(size=(B, T, D))
    dh_T = rng.normal(size=(B, D))
    return p, dy, dh_T


def _loss(p, dy, dh_T):
    y, hT, _ = orc.rglru_fwd(p["x"], p["conv_w"], p["W_a"], p["b_a"], p["W_x"], p["b_x"],
                             p["Lambda"], h0=p["h0"], conv_state=p["conv_state"])
    return float(np.sum(dy * y) + np.sum(dh_T * hT))


def _bwd(p, dy, dh_T):
    return rglru_bwd(p["x"], p["conv_w"], p["W_a"], p["b_a"], p["W_x"], p["b_x"], p["Lambda"],
                     dy, h0=p["h0"], conv_state=p["conv_state"], dh_T=dh_T)


GRAD_OF = {"x": "dx", "conv_w": "dconv_w", "W_a": "dW_a", "b_a": "db_a", "W_x": "dW_x",
           "b_x": "db_x", "Lambda": "dLambda", "h0": "dh0", "conv_state": "dconv_state"}


@pytest.mark.parametrize("name", sorted(GRAD_OF))
@pytest.mark.parametrize("seed", [0, 1])
def test_directional_finite_differences(name, seed):
    p, dy, dh_T = _inputs(seed)
    g = _bwd(p, dy, dh_T)[GRAD_OF[name]]
    rng = np.random.default_rng(100 + seed)
    v = rng.normal(size=p[name].shape)
    eps = 1e-6
    pp, pm = dict(p), dict(p)
    pp[name] = p[name] + eps * v
    pm[name] = p[name] - eps * v
    fd = (_loss(pp, dy, dh_T) - _loss(pm, dy, dh_T)) / (2 * eps)
    an = float(np.sum(g * v))
    assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_r_zero_holds_the_state():
    """r = 0: a = 1 and beta = 0, so y_t = h0 for every t: d h0 = sum_t dy_t + dh_T
    and no other input influences L."""
    p, dy, dh_T = _inputs(3, r_zero=True)
    g = _bwd(p, dy, dh_T)
    np.testing.assert_allclose(g["dh0"], dy.sum(axis=1) + dh_T, rtol=1e-14, atol=1e-14)
    for k in ("dx", "dconv_w", "dW_a", "db_a", "dW_x", "db_x", "dLambda", "dconv_state"):
        assert np.all(g[k] == 0.0), k


def test_constant_gate_dh0_closed_form():
    """W_a = 0 makes r = sigmoid(b_a) and a constant per channel; then
    d h0 = sum_t a^(t+1) dy_t + a^T dh_T (geometric weights)."""
    p, dy, dh_T = _inputs(4)
    p["W_a"] = np.zeros((H, BW, BW))
    g = _bwd(p, dy, dh_T)
    r = 1.0 / (1.0 + np.exp(-p["b_a"]))
    a = np.exp(-8.0 * r * np.log1p(np.exp(-p["Lambda"])))
    pw = a[None, :] ** np.arange(1, T + 1)[:, None]            # (T, D): a^(t+1)
    want = np.einsum("btd,td->bd", dy, pw) + dh_T * a[None, :] ** T
    np.testing.assert_allclose(g["dh0"], want, rtol=1e-12, atol=1e-12)


def test_linear_in_output_gradients():
    p, dy, dh_T = _inputs(5)
    rng = np.random.default_rng(6)
    dy2, dh2 = rng.normal(size=dy.shape), rng.normal(size=dh_T.shape)
    g1, g2 = _bwd(p, dy, dh_T), _bwd(p, dy2, dh2)
    g12 = _bwd(p, dy + 2.0 * dy2, dh_T + 2.0 * dh2)
    for k in g12:
        np.testing.assert_allclose(g12[k], g1[k] + 2.0 * g2[k], rtol=1e-10, atol=1e-10)
