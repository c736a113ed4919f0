"""GPU parity on the edges of the gate math, through the C ABI, against the oracle.

* The general gate branch. The tensor-core kernels take a shorter form of the
  decay when c * softplus(-Lambda) <= 1/8 for every channel a warp holds
  (a^8 >= 0.8825) and a general form otherwise; a^8 ~ U[0.05, 0.85] sends every
  warp down the general branch, U[0.85, 0.92] mixes both within a call.
* A closed recurrence gate: with b_a = -30 the gate r is about 1e-13, so a_t
  rounds to 1 in fp32 and sqrt(1 - a_t^2) is about 1e-6: the state holds h0
  ("the RG-LRU's gating does not depend on the recurrent state": "Beyond
  Transformer Architecture: Griffin and Google RecurrentGemma", "Core
  Components of Griffin", 1. RG-LRU; with the recurrence gate shut, a_t = 1
  and the input term vanishes).
* Saturated gates: |z| of 20 to 30, where sigmoid is 0 or 1 to fp32 precision.
* The designed arithmetic: the tensor-core path rounds the Conv1D output to
  bf16 where it enters the gate contraction. Against the oracle with that
  same rounding (oracle gate_operand="bf16") it must agree far more tightly
  than against the exact oracle: what remains is the output's own bf16
  rounding (at most the bf16 unit roundoff 2^-8 of the value) and fp32
  arithmetic (h_T, stored in fp32, agrees to 1e-4 of the floor).
Every output buffer starts as NaN.
"""
import numpy as np
import pytest
import torch

import gated_linear_recurrence_rglru_b200 as rg
from gated_linear_recurrence_rglru_b200.workloads import WORKLOADS, generate
from oracle import rglru_oracle as orc
from oracle.compare import channel_rms, max_rel_err

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
KEYS = ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")


def _dev(t, dev):
    return {k: (v.to(dev) if v is not None else None) for k, v in t.items()}


def _run_fwd(t, wl, dev, algo):
    if rg.fwd_launches(wl.B, wl.T, wl.D, wl.H, wl.dtype, algo) == 0:
        pytest.skip(f"{algo} does not cover {wl}")
    g = _dev(t, dev)
    y = torch.full_like(g["x"], float("nan"))
    hT = torch.full((wl.B, wl.D), float("nan"), device=dev)
    cs = torch.full((wl.B, 3, wl.D), float("nan"), device=dev, dtype=wl.dtype)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    rg.rglru_fwd(g["x"], *[g[k] for k in KEYS], h0=g["h0"], algo=algo, y=y, h_T=hT,
                 conv_state_out=cs, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return y.float().cpu().numpy(), hT.cpu().numpy(), cs.float().cpu().numpy()


def _oracle(t, gate_operand=None):
    return orc.rglru_fwd(t["x"], *[t[k] for k in KEYS], h0=t["h0"], gate_operand=gate_operand)


def _check(t, wl, dev, algo):
    yg, hg, cg = _run_fwd(t, wl, dev, algo)
    yo, ho, co = _oracle(t)
    e_y = max_rel_err(yg, yo)
    e_h = max_rel_err(hg, ho, scale=channel_rms(yo, 1)[:, 0, :])
    assert np.array_equal(cg, co)
    assert e_y <= TOL[wl.io] and e_h <= TOL[wl.io], (wl, algo, e_y, e_h)
    return yg, hg, yo, ho


GENERAL = [
    WORKLOADS["hawk_block"].with_shape(B=2, T=300, D=256, H=4, h0_var=0.5, bias_std=0.5,
                                       ac_lo=0.05, ac_hi=0.85, seed=81),
    WORKLOADS["hawk_block"].with_shape(B=2, T=150, D=256, H=2, ac_lo=0.05, ac_hi=0.85, seed=82),
    WORKLOADS["griffin2b"].with_shape(B=2, T=100, D=512, H=2, h0_var=0.1, bias_std=0.5,
                                      ac_lo=0.05, ac_hi=0.85, seed=83),
    WORKLOADS["hawk_block"].with_shape(B=3, T=129, D=256, H=4, ac_lo=0.85, ac_hi=0.92, seed=84),
    WORKLOADS["long_context"].with_shape(B=1, T=700, D=512, H=2, ac_lo=0.85, ac_hi=0.92,
                                         seed=85),
    WORKLOADS["tiny_f32"].with_shape(B=2, T=100, D=128, H=2, ac_lo=0.05, ac_hi=0.85, seed=86),
]


@pytest.mark.parametrize("algo", ["generic", "tensor"])
@pytest.mark.parametrize("idx", range(len(GENERAL)))
def test_general_gate_branch(cuda_device, algo, idx):
    wl = GENERAL[idx]
    _check(generate(wl), wl, cuda_device, algo)


def _closed_gate_inputs(wl):
    t = generate(wl)
    t["b_a"] = torch.full((wl.D,), -30.0).to(wl.dtype)
    return t


@pytest.mark.parametrize("algo", ["generic", "tensor"])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_closed_recurrence_gate_holds_the_state(cuda_device, algo, io):
    wl = WORKLOADS["hawk_block"].with_shape(B=2, T=200, D=256, H=2, io=io, h0_var=1.0, seed=87)
    t = _closed_gate_inputs(wl)
    yg, hg, yo, ho = _check(t, wl, cuda_device, algo)
    h0 = t["h0"].numpy().astype(np.float64)
    drift = np.abs(ho - h0)                       # the oracle's own drift: sum of ~1e-6 inputs
    assert drift.max() < 1e-3
    assert np.all(np.abs(hg - h0) <= 2 * drift + 1e-6 * np.abs(h0) + 1e-7)
    # y_t stays at h0 too: within the oracle's drift and the output rounding
    ulp = 2.0 ** -8 if io == "bf16" else 2.0 ** -23
    assert np.all(np.abs(yg - h0[:, None, :]) <= 2e-3 + ulp * np.abs(h0[:, None, :]))


@pytest.mark.parametrize("algo", ["generic", "tensor"])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_saturated_gates(cuda_device, algo, io):
    wl = WORKLOADS["hawk_block"].with_shape(B=2, T=130, D=256, H=4, io=io, h0_var=0.5, seed=88)
    t = generate(wl)
    g = torch.Generator().manual_seed(88)
    levels = torch.tensor([-30.0, -20.0, 20.0, 30.0])
    t["b_a"] = levels[torch.randint(0, 4, (wl.D,), generator=g)].to(wl.dtype)
    t["b_x"] = levels[torch.randint(0, 4, (wl.D,), generator=g)].to(wl.dtype)
    _check(t, wl, cuda_device, algo)


DESIGNED = [
    WORKLOADS["hawk_block"].with_shape(B=2, T=300, D=256, H=4, h0_var=0.5, bias_std=0.5, seed=31),
    WORKLOADS["long_context"].with_shape(B=1, T=2000, D=512, H=2, seed=35),
    WORKLOADS["griffin2b"].with_shape(B=3, T=100, D=768, H=3, bias_std=0.5, seed=37),
    WORKLOADS["hawk_block"].with_shape(B=2, T=300, D=256, H=4, ac_lo=0.05, ac_hi=0.85, seed=81),
]
# The bf16 unit roundoff (the output's own rounding) plus fp32 arithmetic.
DESIGNED_TOL_Y = 2.0 ** -8 + 1e-4
DESIGNED_TOL_H = 1e-4


@pytest.mark.parametrize("idx", range(len(DESIGNED)))
def test_tensor_path_is_the_designed_arithmetic(cuda_device, idx):
    wl = DESIGNED[idx]
    t = generate(wl)
    yg, hg, _ = _run_fwd(t, wl, cuda_device, "tensor")
    ye, he, _ = _oracle(t, gate_operand="bf16")
    yo, ho, _ = _oracle(t)
    e_design = max_rel_err(yg, ye)
    h_design = max_rel_err(hg, he, scale=channel_rms(ye, 1)[:, 0, :])
    h_exact = max_rel_err(hg, ho, scale=channel_rms(yo, 1)[:, 0, :])
    assert e_design <= DESIGNED_TOL_Y and h_design <= DESIGNED_TOL_H, (e_design, h_design)
    # the operand rounding explains the error: h_T (fp32, no output rounding)
    # is far closer to the designed arithmetic than to the exact oracle
    assert h_design < h_exact / 10, (h_design, h_exact)
