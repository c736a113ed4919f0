"""Float64 CPU oracle for the gradient of the RG-LRU layer.

TEST INFRASTRUCTURE ONLY, like rglru_oracle (whose forward intermediates it
uses): only tests/ and bench.py's CPU-baseline leg may call it. It shares no
code with the CUDA library.

What it computes: the exact gradient of the scalar
    L = sum_{b,t,d} dy[b,t,d] * y[b,t,d] + sum_{b,d} dh_T[b,d] * h_T[b,d]
with respect to every input of the forward layer (x, the conv taps, both gate
weights and biases, Lambda, h0 and the conv history), i.e. the vector-Jacobian
product of the layer as defined in rglru_oracle (the layer's definition; the
pages print no equation for it). The sources give no
backward pass; this is the plain chain rule through the forward definition, in
reverse order of its steps:

  scan       h_t = a_t h_{t-1} + beta_t        (reverse-time scan)
             G_t  = dy_t + a_{t+1} G_{t+1},  G_{T-1} = dy_{T-1} + dh_T
             d a_t = G_t h_{t-1},  d beta_t = G_t,  d h0 = a_0 G_0
  input      beta = g i u,  g = sqrt(1 - a^2) = sqrt(-expm1(2 log a))
             d g = d beta i u,  d i = d beta g u,  d u += d beta g i
  decay      a = exp(la),  dg/dla = -a^2 / g
             d la = d a * a + d g * (-a^2 / g)
             la = -c r sp,  sp = softplus(-Lambda)
             d r = d la (-c sp),  d sp = sum_{b,t} d la (-c r)
             (the g path is grouped as r / g, finite as r -> 0)
             d Lambda = d sp * (-sigmoid(-Lambda))
  gates      r = sigmoid(z_a),  i = sigmoid(z_x)
             d z_a = d r r (1 - r),  d z_x = d i i (1 - i)
             z = u_head W + b:  d u_head += d z W^T,  d W = u_head^T d z,  d b = sum d z
  conv       u_t = sum_k w[k] x_{t-3+k}:
             d x_{t-3+k} += w[k] d u_t,  d w[k] = sum_{b,t} x_{t-3+k} d u_t

Pinned in tests/test_oracle_backward.py by central finite differences of the
forward oracle along random directions, by closed forms (r = 0 holds the state,
so d h0 = sum_t dy_t + dh_T and every input gradient vanishes) and by
linearity in (dy, dh_T).
"""
from __future__ import annotations

import numpy as np

from .rglru_oracle import C_DECAY, as_f64, intermediates, linear_scan, sigmoid, softplus


def rglru_bwd(x, conv_w, W_a, b_a, W_x, b_x, Lambda, dy, h0=None, conv_state=None, dh_T=None):
    """Gradients of L (module docstring) for one forward call.

    Inputs as for rglru_oracle.rglru_fwd, plus dy (B, T, D) and dh_T (B, D) or
    None. Returns a dict of float64 arrays: dx (B,T,D), dconv_w (4,D),
    dW_a, dW_x (H,bw,bw), db_a, db_x (D), dLambda (D), dh0 (B,D) and
    dconv_state (B,3,D) (the gradient with respect to the conv history; zero
    history when none was passed).
    """
    x64, w64 = as_f64(x), as_f64(conv_w)
    Wa, Wx, L = as_f64(W_a), as_f64(W_x), as_f64(Lambda)
    dy = as_f64(dy)
    B, T, D = x64.shape
    H, bw, _ = Wa.shape
    it = intermediates(x, conv_w, W_a, b_a, W_x, b_x, Lambda, conv_state)
    u, r, i, la, a = it["u"], it["r"], it["i"], it["log_a"], it["a"]
    h0v = np.zeros((B, D)) if h0 is None else as_f64(h0)
    h = linear_scan(a, it["beta"], h0v)
    h_prev = np.concatenate([h0v[:, None, :], h[:, :-1, :]], axis=1)

    # reverse-time scan of the state gradient
    G = np.empty((B, T, D))
    carry = np.zeros((B, D)) if dh_T is None else as_f64(dh_T).copy()
    for t in range(T - 1, -1, -1):
        carry = carry + dy[:, t, :]
        G[:, t, :] = carry
        carry = a[:, t, :] * carry
    dh0 = carry

    d_a = G * h_prev
    d_beta = G
    g = np.sqrt(-np.expm1(2.0 * la))
    d_g = d_beta * i * u
    d_i = d_beta * g * u
    d_u = d_beta * g * i
    # d la = d a * a + d g * (-a^2 / g); it reaches r through la = -c r sp and
    # z_a through r (1 - r). The g path carries r / g, which tends to 0 with r
    # (1 - a^2 ~ 2 c sp r), so it is formed as that ratio (0 where r = g = 0)
    # instead of as (1 / g) * r, which is 0 * inf there.
    sp = softplus(-L)[None, None, :]
    with np.errstate(divide="ignore", invalid="ignore"):
        r_over_g = np.where(g > 0.0, r / np.where(g > 0.0, g, 1.0), 0.0)
    d_za = (-C_DECAY * sp) * (d_a * a * r * (1.0 - r)) + (C_DECAY * sp) * (a * a) * (1.0 - r) * d_g * r_over_g
    d_sp = np.sum((-C_DECAY) * d_a * a * r + C_DECAY * (a * a) * d_g * r_over_g, axis=(0, 1))
    dLambda = d_sp * (-sigmoid(-L))
    d_zx = d_i * i * (1.0 - i)

    def gate_back(dz, W):
        uh = u.reshape(B * T, H, bw).transpose(1, 0, 2)       # (H, N, bw_in)
        dzh = dz.reshape(B * T, H, bw).transpose(1, 0, 2)     # (H, N, bw_out)
        du_h = np.matmul(dzh, W.transpose(0, 2, 1))           # d u_i = sum_j d z_j W[i, j]
        dW = np.matmul(uh.transpose(0, 2, 1), dzh)            # d W[i, j] = sum_n u_i d z_j
        return du_h.transpose(1, 0, 2).reshape(B, T, D), dW, dz.sum(axis=(0, 1))

    du_a, dW_a, db_a = gate_back(d_za, Wa)
    du_x, dW_x, db_x = gate_back(d_zx, Wx)
    d_u = d_u + du_a + du_x

    hist = np.zeros((B, 3, D)) if conv_state is None else as_f64(conv_state)
    xp = np.concatenate([hist, x64], axis=1)                   # xp[:, t + 3] = x_t
    dxp = np.zeros_like(xp)
    dconv_w = np.zeros((4, D))
    for k in range(4):                                         # tap k reads xp[:, t + k]
        dxp[:, k:k + T, :] += w64[k][None, None, :] * d_u
        dconv_w[k] = np.sum(xp[:, k:k + T, :] * d_u, axis=(0, 1))
    return dict(dx=dxp[:, 3:, :], dconv_w=dconv_w, dW_a=dW_a, db_a=db_a, dW_x=dW_x,
                db_x=db_x, dLambda=dLambda, dh0=dh0, dconv_state=dxp[:, :3, :])
