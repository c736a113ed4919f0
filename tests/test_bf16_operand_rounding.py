"""Where the parity floor comes from (CPU): the designed arithmetic of a bf16
tensor-core gate contraction, run against the exact float64 oracle.

The tensor-core kernels round one thing that the definition keeps exact: the
Conv1D output u where it enters the gate contraction (a bf16 MMA operand), and
they store y in bf16. oracle.rglru_fwd(..., gate_operand="bf16") applies that
one rounding and keeps everything else in float64. These tests

  1. pin that rounding (off = the oracle; exact when u is already a bf16
     value; the contraction's error within the rounding bound), and
  2. measure, on the shapes of the GPU parity cases, what the designed
     arithmetic scores under the candidate floors of oracle/compare.py: the
     floor 1e-3 * RMS cannot be met by it at all, a per-row RMS floor needs a
     factor above 1 on a short decode case, and the floor used (the channel's
     RMS over all rows and steps) is met with a margin of at least 1.2.
"""
import numpy as np
import pytest
import torch

from gated_linear_recurrence_rglru_b200.workloads import WORKLOADS, generate
from oracle import rglru_oracle as orc
from oracle.compare import FLOOR, TIGHT_FLOOR, channel_rms, max_rel_err, row_rms

BAR = 2e-2


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).bfloat16().double().numpy()


def _args(t):
    return [t[k] for k in ("x", "conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")]


# ---------------------------------------------------- pins of the rounding --

def test_rounding_off_is_the_oracle():
    wl = WORKLOADS["hawk_block"].with_shape(B=2, T=40, D=128, H=2, h0_var=0.5, bias_std=0.5,
                                            seed=101)
    t = generate(wl)
    y0, h0, c0 = orc.rglru_fwd(*_args(t), h0=t["h0"])
    y1, h1, c1 = orc.rglru_fwd(*_args(t), h0=t["h0"], gate_operand=None)
    assert np.array_equal(y0, y1) and np.array_equal(h0, h1) and np.array_equal(c0, c1)
    with pytest.raises(ValueError):
        orc.rglru_fwd(*_args(t), gate_operand="fp8")


def test_rounding_is_exact_on_bf16_values():
    """conv_w = tap 3 only, x stored in bf16: u = x is already a bf16 value."""
    wl = WORKLOADS["hawk_block"].with_shape(B=2, T=30, D=128, H=2, bias_std=0.5, seed=102)
    t = generate(wl)
    t["conv_w"] = torch.zeros_like(t["conv_w"])
    t["conv_w"][3] = 1.0
    y0, _, _ = orc.rglru_fwd(*_args(t))
    y1, _, _ = orc.rglru_fwd(*_args(t), gate_operand="bf16")
    assert np.array_equal(y0, y1)


def test_contraction_error_within_the_rounding_bound():
    """|z(bf16 u) - z(u)| <= 2^-8 sum_i |u_i W_ij| (round to nearest: |du| <= 2^-8 |u|
    for bf16's 8-bit significand, counting the fp32 step before it)."""
    rng = np.random.default_rng(7)
    u = rng.standard_normal((3, 17, 64)) * 3.0
    W = rng.standard_normal((2, 32, 32)) / 8
    b = np.zeros(64)
    ub = orc.round_gate_operand(u, "bf16")
    assert np.all(np.abs(ub - u) <= 2.0 ** -8 * np.abs(u))
    assert np.any(ub != u)
    dz = np.abs(orc.gate_preacts(ub, W, b) - orc.gate_preacts(u, W, b))
    bound = orc.gate_preacts(np.abs(u), np.abs(W), b) * 2.0 ** -8
    assert np.all(dz <= bound * (1 + 1e-12))


# ------------------------------------------------- the floor, measured ----

FWD_CASES = [
    WORKLOADS["hawk_block"].with_shape(B=2, T=300, D=256, H=4, h0_var=0.5, bias_std=0.5, seed=31),
    WORKLOADS["hawk_block"].with_shape(B=3, T=129, D=256, H=2, seed=32),
    WORKLOADS["hawk_block"].with_shape(B=1, T=200, D=512, H=2, h0_var=0.1, seed=33),
    WORKLOADS["long_context"].with_shape(B=1, T=5000, D=256, H=2, seed=35),
    WORKLOADS["long_context"].with_shape(B=1, T=1000, D=512, H=2, seed=36),
    WORKLOADS["long_context"].with_shape(B=1, T=2000, D=512, H=2, seed=35),
    WORKLOADS["griffin2b"].with_shape(B=3, T=100, D=768, H=3, bias_std=0.5, seed=37),
    WORKLOADS["hawk_block"].with_shape(B=2, T=300, D=256, H=4, ac_lo=0.05, ac_hi=0.85, seed=81),
]
DEC_CASES = [  # (workload, steps): the GPU decode parity shapes
    (WORKLOADS["decode_batch"].with_shape(B=33, D=256, H=2, decode_steps=5, bias_std=0.3,
                                          seed=86), 5),
    (WORKLOADS["decode_batch"].with_shape(B=70, D=256, H=4, decode_steps=5, bias_std=0.3,
                                          seed=123), 5),
    (WORKLOADS["decode_batch"].with_shape(B=37, D=256, H=4, decode_steps=7, bias_std=0.3,
                                          seed=51), 7),
    (WORKLOADS["decode_batch"].with_shape(B=64, D=256, H=2, decode_steps=8, bias_std=0.3,
                                          ac_lo=0.05, ac_hi=0.85, seed=90), 8),
]


def _fwd_pair(wl):
    t = generate(wl)
    yo, _, _ = orc.rglru_fwd(*_args(t), h0=t["h0"])
    ye, _, _ = orc.rglru_fwd(*_args(t), h0=t["h0"], gate_operand="bf16")
    return _bf16(ye), yo, 1


def _dec_pair(wl, steps):
    t = generate(wl)
    w = {k: t[k] for k in ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")}
    ho = he = orc.as_f64(t["h"])
    ro = re = orc.as_f64(t["conv_state"])
    yo, ye = [], []
    for s in range(steps):
        y, ho, ro = orc.rglru_decode_step(t["x_steps"][s], ro, s, ho, **w)
        yo.append(y)
        y, he, re = orc.rglru_decode_step(t["x_steps"][s], re, s, he, gate_operand="bf16", **w)
        ye.append(_bf16(y))
    return np.stack(ye), np.stack(yo), 0


def _min_factor(err, o, scale):
    """Smallest floor factor f with max err / max(|o|, f scale) <= BAR (bisection)."""
    lo, hi = 1e-4, 10.0
    for _ in range(50):
        mid = (lo * hi) ** 0.5
        if (err / np.maximum(np.abs(o), mid * scale)).max() <= BAR:
            hi = mid
        else:
            lo = mid
    return hi


@pytest.fixture(scope="module")
def measured():
    rows = []
    for wl in FWD_CASES:
        rows.append(("fwd", wl) + _fwd_pair(wl))
    for wl, steps in DEC_CASES:
        rows.append(("decode", wl) + _dec_pair(wl, steps))
    out = []
    for kind, wl, ye, yo, tax in rows:
        err = np.abs(ye - yo)
        out.append(dict(kind=kind, wl=wl,
                        at_floor=max_rel_err(ye, yo, time_axis=tax),
                        at_tight_floor=max_rel_err(ye, yo, time_axis=tax, floor=TIGHT_FLOOR),
                        f_pooled=_min_factor(err, yo, channel_rms(yo, tax)),
                        f_row=_min_factor(err, yo, row_rms(yo, tax))))
    return out


def test_tight_floor_is_out_of_reach_of_bf16_operands(measured):
    """Under 1e-3 * RMS the designed arithmetic itself is far above the bar."""
    worst = max(m["at_tight_floor"] for m in measured)
    assert worst > 50 * BAR, worst
    assert sum(m["at_tight_floor"] > BAR for m in measured) >= len(measured) - 1


def test_row_rms_floor_needs_a_factor_above_one(measured):
    """The 33-row, 5-step decode case: per-row RMS would need a factor > 1."""
    dec = [m for m in measured if m["kind"] == "decode"]
    assert max(m["f_row"] for m in dec) > 1.0


def test_chosen_floor_is_met_with_margin(measured):
    for m in measured:
        assert m["at_floor"] <= BAR / 1.2, (m["wl"], m["at_floor"])
    worst_f = max(m["f_pooled"] for m in measured)
    assert worst_f < FLOOR / 1.2, worst_f
    assert worst_f > 0.8 * FLOOR, worst_f          # and it is the tightest round factor


def test_long_memory_channels_set_the_floor(measured):
    """The long-memory case (a^8 up to 0.9999) needs more than 0.75 of the RMS."""
    lc = [m for m in measured if m["wl"].name == "long_context" and m["wl"].T == 2000]
    assert lc and lc[0]["f_pooled"] > 0.75
