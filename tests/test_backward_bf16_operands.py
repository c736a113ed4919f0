"""Why the B = 2, T = 1 bf16 backward parity case is an expected failure (CPU).

The tensor-core backward rounds two MMA operands to bf16: u for z = u W, and d z
for d z W^T. This test applies the chain rule of the backward oracle in float64
with exactly those two roundings (and dx stored in bf16), on the inputs of that
parity case. Scored with the parity test's measure (per-channel RMS floor: two
samples per channel at B*T = 2), the designed arithmetic itself exceeds the 2e-2
bar on dx. Without the roundings the same computation stays well inside it, so
the rounding is the cause and no term or index is.
"""
import numpy as np
import torch

import oracle.rglru_oracle as ro
from gated_linear_recurrence_rglru_b200.workloads import WORKLOADS, generate
from oracle.compare import max_rel_err
from oracle.rglru_backward import rglru_bwd as bwd_oracle


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).double().numpy()


def _dx_with_operand_rounding(x, conv_w, W_a, b_a, W_x, b_x, Lambda, dy, h0, rounding):
    """dx of the layer's gradient, the chain rule of oracle.rglru_backward, with u and d z
    rounded to bf16 as MMA operands when `rounding`."""
    x64, w64 = ro.as_f64(x), ro.as_f64(conv_w)
    Wa, Wx, L = ro.as_f64(W_a), ro.as_f64(W_x), ro.as_f64(Lambda)
    dy = ro.as_f64(dy)
    B, T, D = x64.shape
    H, bw, _ = Wa.shape
    u = ro.conv4(x64, w64)
    ue = _bf16(u) if rounding else u
    za = ro.gate_preacts(ue, Wa, ro.as_f64(b_a))
    zx = ro.gate_preacts(ue, Wx, ro.as_f64(b_x))
    r, i = ro.sigmoid(za), ro.sigmoid(zx)
    la = ro.log_decay(r, L)
    a = np.exp(la)
    g = np.sqrt(-np.expm1(2 * la))
    h0v = ro.as_f64(h0)
    h = ro.linear_scan(a, g * i * u, h0v)
    hp = np.concatenate([h0v[:, None], h[:, :-1]], axis=1)
    G = np.empty_like(h)
    c = np.zeros((B, D))
    for t in range(T - 1, -1, -1):
        c = c + dy[:, t]
        G[:, t] = c
        c = a[:, t] * c
    da, dg, di = G * hp, G * i * u, G * g * u
    du = G * g * i
    sp = ro.softplus(-L)[None, None]
    C = ro.C_DECAY
    rog = np.where(g > 0, r / np.where(g > 0, g, 1.0), 0.0)
    dza = -C * sp * da * a * r * (1 - r) + C * sp * a * a * (1 - r) * dg * rog
    dzx = di * i * (1 - i)
    if rounding:
        dza, dzx = _bf16(dza), _bf16(dzx)

    def back(dz, W):
        dzh = dz.reshape(B * T, H, bw).transpose(1, 0, 2)
        return np.matmul(dzh, W.transpose(0, 2, 1)).transpose(1, 0, 2).reshape(B, T, D)

    du = du + back(dza, Wa) + back(dzx, Wx)
    xp = np.concatenate([np.zeros((B, 3, D)), x64], axis=1)
    dxp = np.zeros_like(xp)
    for k in range(4):
        dxp[:, k:k + T] += w64[k][None, None] * du
    return dxp[:, 3:]


def test_bf16_operands_exceed_the_bar_at_two_samples_per_channel():
    wl = WORKLOADS["hawk_block"].with_shape(B=2, T=1, D=128, H=2, h0_var=1.0, seed=51)
    t = generate(wl)
    dy = torch.randn(wl.B, wl.T, wl.D,
                     generator=torch.Generator().manual_seed(wl.seed + 1000)).to(wl.dtype)
    args = [t[k] for k in ("x", "conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")]
    ref = bwd_oracle(*args, dy, h0=t["h0"])["dx"]
    exact = _dx_with_operand_rounding(*args, dy, t["h0"], rounding=False)
    rounded = _bf16(_dx_with_operand_rounding(*args, dy, t["h0"], rounding=True))
    assert max_rel_err(exact, ref) < 1e-9            # the restatement is the oracle's chain rule
    assert max_rel_err(_bf16(exact), ref) < 1e-2      # bf16 storage of dx alone is inside the bar
    assert max_rel_err(rounded, ref) > 2e-2           # the operand roundings are not


def test_backward_floor_factor_is_derived_from_its_operand_roundings():
    """The floor of the backward's sequence gradients (BWD_FLOOR): its designed
    arithmetic needs a factor of about 0.79 on the B=2 T=2048 D=1024 H=16 case
    (the GPU read 0.0211 under 0.75 there, exactly this emulation's figure), so
    0.75 is too tight for it and 1.0 leaves a margin."""
    from oracle.compare import BWD_FLOOR, channel_rms
    wl = WORKLOADS["hawk_block"].with_shape(B=2, T=2048, D=1024, H=16, h0_var=0.1, seed=48)
    t = generate(wl)
    dy = torch.randn(wl.B, wl.T, wl.D,
                     generator=torch.Generator().manual_seed(wl.seed + 1000)).to(wl.dtype)
    args = [t[k] for k in ("x", "conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")]
    ref = bwd_oracle(*args, dy, h0=t["h0"])["dx"]
    em = _bf16(_dx_with_operand_rounding(*args, dy, t["h0"], rounding=True))
    assert max_rel_err(em, ref, floor=0.75) > 2e-2
    assert max_rel_err(em, ref, floor=BWD_FLOOR) <= 2e-2 / 1.2
    err, rms = np.abs(em - ref), channel_rms(ref, 1)
    assert (err / np.maximum(np.abs(ref), 0.7 * rms)).max() > 2e-2          # f* is above 0.7
