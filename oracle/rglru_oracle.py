"""Float64 CPU oracle for the RG-LRU layer (conv4 -> gates -> log-space decay -> scan).

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module:
only tests/, the smoke check in __graft_entry__ and bench.py's CPU-baseline
leg may call it. It shares no code with the CUDA library; it receives the same
seeded input tensors (as stored: bf16- or fp32-rounded values) and upcasts
them to float64.

What it computes, step by step, in the order the method states it.
The source pages describe the layer's parts but print no formula for it; the
equations below are the layer's definition as this library states it (the
same text heads include/rglru.h). What the pages do say, and where:
  [DE]   S. De's thread on Griffin ("how we got there", muskviewer page): the
         RG-LRU is the LRU (a diagonal recurrence) with a recurrent gate added;
         a temporal Conv1D sits in the simple recurrent block; the layer is
         memory-bound and its kernel is a linear scan, not a parallel one.
  [RG]   "Beyond Transformer Architecture: Griffin and Google RecurrentGemma",
         "Core Components of Griffin", 1. RG-LRU: the gates do not depend on
         the recurrent state; "Key Strengths of RecurrentGemma", 1. Reduced
         Memory Usage: the recurrent state has a fixed size (decoding).
The equations:
  u_t  = sum_{k=0..3} w[k] * x_{t-3+k}            causal depthwise Conv1D, width 4
  r_t  = sigmoid(W_a u_t + b_a)                    recurrence gate, block-diagonal per head
  i_t  = sigmoid(W_x u_t + b_x)                    input gate, block-diagonal per head
  log a_t = -c * r_t * softplus(-Lambda),  c = 8   (a = sigmoid(Lambda), a_t = a^(c r_t))
  h_t  = a_t * h_{t-1} + sqrt(1 - a_t^2) * (i_t * u_t)
  y_t  = h_t
Readings where the definition and the pages are silent (each listed in the
design notes):
  * tap order: w[3] multiplies the current input, w[0] the input three steps back;
  * no conv bias; history before t = 0 is zeros unless a conv state is passed;
  * block-diagonal gate: z[b, t, h*bw + j] = sum_i u[b, t, h*bw + i] * W[h, i, j];
  * sqrt(1 - a_t^2) is formed as sqrt(-expm1(2 log a_t)), the same number;
  * conv state (B, 3, D) is chronological: slot 0 holds the oldest input.
Decode ring: slot (pos % 3) holds x_{pos-3}, slot ((pos+1) % 3) holds
x_{pos-2}, slot ((pos+2) % 3) holds x_{pos-1}; after the step slot (pos % 3)
holds the new input. A chronological conv state is the ring at pos = 0.

Every function is pinned in tests/test_oracle.py by facts that do not come
from this file: a library Conv1D, a dense block-diagonal matmul, closed forms
(r = 0, constant gates, a = 1/16), a brute-force unrolled sum, reordering
invariance, second-moment preservation and fwd/decode composition.

gate_operand="bf16" (off by default) rounds the Conv1D output to bfloat16
before the gate contraction only, as a bf16 tensor-core contraction rounds
its operand (u is formed in fp32, then rounded to nearest even); everything
else stays float64. It is not the definition: it is the designed arithmetic
of a bf16-operand contraction, used to show how far from the exact result
such a contraction lands (tests/test_bf16_operand_rounding.py).
"""
from __future__ import annotations

import numpy as np

C_DECAY = 8.0  # the constant c in log a_t = -c * r_t * softplus(-Lambda)


def as_f64(t):
    """Upcast a tensor as stored (torch bf16/fp32, numpy, or None) to float64 numpy."""
    if t is None:
        return None
    if hasattr(t, "detach"):
        return t.detach().to("cpu").double().numpy()
    return np.asarray(t, dtype=np.float64)


def conv4(x, conv_w, conv_state=None):
    """Causal depthwise Conv1D of width 4 ([DE]: the temporal Conv1D of the recurrent block).

    x: (B, T, D); conv_w: (4, D); conv_state: (B, 3, D) chronological history
    (x_{-3}, x_{-2}, x_{-1}) or None for zeros. Returns u (B, T, D).
    """
    B, T, D = x.shape
    hist = np.zeros((B, 3, D)) if conv_state is None else conv_state
    xp = np.concatenate([hist, x], axis=1)           # xp[:, t + 3] = x_t
    u = np.zeros((B, T, D))
    for k in range(4):                               # tap k reads x_{t-3+k} = xp[:, t + k]
        u += conv_w[k][None, None, :] * xp[:, k:k + T, :]
    return u


def gate_preacts(u, W, b):
    """Block-diagonal per-head affine map (the gates of the definition; [DE]: a gate added to the LRU).

    u: (B, T, D); W: (H, bw, bw) with z[j] = sum_i u[i] W[i, j]; b: (D,).
    """
    B, T, D = u.shape
    H, bw, bw2 = W.shape
    assert bw == bw2 and H * bw == D
    uh = u.reshape(B * T, H, bw).transpose(1, 0, 2)      # (H, B*T, bw): head h's inputs
    z = np.matmul(uh, W)                                  # z[h, n, j] = sum_i u[n, h*bw+i] W[h, i, j]
    return z.transpose(1, 0, 2).reshape(B, T, D) + b[None, None, :]


def sigmoid(z):
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def softplus(v):
    """log(1 + e^v), written so that it neither overflows nor cancels."""
    return np.maximum(v, 0.0) + np.log1p(np.exp(-np.abs(v)))


def log_decay(r, Lambda):
    """log a_t = -c * r_t * softplus(-Lambda), c = 8 (the definition)."""
    return -C_DECAY * r * softplus(-Lambda)[None, None, :]


def gated_input(log_a, i, u):
    """sqrt(1 - a_t^2) * (i_t * u_t), with 1 - a_t^2 = -expm1(2 log a_t) (the definition)."""
    return np.sqrt(-np.expm1(2.0 * log_a)) * (i * u)


def linear_scan(a, beta, h0=None):
    """h_t = a_t * h_{t-1} + beta_t, sequential in t [DE: diagonal recurrence, linear scan].

    a, beta: (B, T, D); h0: (B, D) or None (zeros). Returns all h_t (B, T, D).
    """
    B, T, D = a.shape
    h = np.zeros((B, D)) if h0 is None else np.array(h0, dtype=np.float64)
    out = np.empty((B, T, D))
    for t in range(T):
        h = a[:, t, :] * h + beta[:, t, :]
        out[:, t, :] = h
    return out


def round_gate_operand(u, gate_operand):
    """The gate contraction's view of u: u itself (None), or u formed in fp32 and
    rounded to the nearest bfloat16 ("bf16"), as a bf16 tensor-core operand."""
    if gate_operand is None:
        return u
    if gate_operand != "bf16":
        raise ValueError(f"unknown gate operand rounding {gate_operand!r}")
    import torch
    return torch.from_numpy(np.asarray(u, dtype=np.float32)).bfloat16().double().numpy()


def intermediates(x, conv_w, W_a, b_a, W_x, b_x, Lambda, conv_state=None, gate_operand=None):
    """u, r, i, log a, a, beta of the layer (all float64, (B, T, D))."""
    x, conv_w, W_a, b_a, W_x, b_x, Lambda, conv_state = map(
        as_f64, (x, conv_w, W_a, b_a, W_x, b_x, Lambda, conv_state))
    u = conv4(x, conv_w, conv_state)
    ug = round_gate_operand(u, gate_operand)
    r = sigmoid(gate_preacts(ug, W_a, b_a))
    i = sigmoid(gate_preacts(ug, W_x, b_x))
    la = log_decay(r, Lambda)
    a = np.exp(la)
    beta = gated_input(la, i, u)
    return dict(u=u, r=r, i=i, log_a=la, a=a, beta=beta)


def conv_state_after(x, conv_state=None):
    """The last three inputs of (history ++ x), chronological (B, 3, D)."""
    x = as_f64(x)
    B, T, D = x.shape
    hist = np.zeros((B, 3, D)) if conv_state is None else as_f64(conv_state)
    return np.concatenate([hist, x], axis=1)[:, -3:, :].copy()


def rglru_fwd(x, conv_w, W_a, b_a, W_x, b_x, Lambda, h0=None, conv_state=None,
              gate_operand=None):
    """The layer over a whole sequence. Returns (y (B,T,D), h_T (B,D), conv_state_out (B,3,D))."""
    it = intermediates(x, conv_w, W_a, b_a, W_x, b_x, Lambda, conv_state, gate_operand)
    y = linear_scan(it["a"], it["beta"], as_f64(h0))
    return y, y[:, -1, :].copy(), conv_state_after(x, conv_state)


def ring_to_chronological(ring, pos):
    """Decode ring (B, 3, D) at step pos -> chronological (x_{pos-3}, x_{pos-2}, x_{pos-1})."""
    ring = as_f64(ring)
    idx = [(pos + k) % 3 for k in range(3)]
    return ring[:, idx, :]


def rglru_decode_step(x_t, ring, pos, h, conv_w, W_a, b_a, W_x, b_x, Lambda, gate_operand=None):
    """One decode step ([RG]: a fixed-size state; the same layer with T = 1).

    x_t: (B, D); ring: (B, 3, D) at step pos; h: (B, D).
    Returns (y_t (B,D), h_new (B,D), ring_new (B,3,D)).
    """
    x_t = as_f64(x_t)
    hist = ring_to_chronological(ring, pos)
    y, h_new, _ = rglru_fwd(x_t[:, None, :], conv_w, W_a, b_a, W_x, b_x, Lambda,
                            h0=as_f64(h), conv_state=hist, gate_operand=gate_operand)
    ring_new = as_f64(ring).copy()
    ring_new[:, pos % 3, :] = x_t
    return y[:, 0, :], h_new, ring_new
