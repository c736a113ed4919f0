"""Float64 CPU oracle for the recurrent block around the RG-LRU layer.

TEST INFRASTRUCTURE ONLY, like rglru_oracle (whose layer it calls): only
tests/ and the bench's CPU legs may call it. It shares no code with the CUDA
library.

Sources: S. De's thread on Griffin (a simple recurrent block with a temporal
Conv1D around the RG-LRU; gated MLP blocks) and "Beyond Transformer
Architecture: Griffin and Google RecurrentGemma", "Core Components of Griffin",
3. Architecture Design (the gated MLP is GeGeLU-like). The pages name the parts but print no equation for the block; the
plainest reading, used here and listed in the design notes:
  g   = GeLU(x W_gate)          the gate branch (GeLU gating)
  v   = x W_in                  the recurrent branch's input projection
  y   = layer(v)                Conv1D, gates, decay and scan (rglru_oracle)
  out = (y * g) W_out           the output projection
with GeLU(v) = v * Phi(v) = v * (1 + erf(v / sqrt 2)) / 2, the exact form (the
pages fix neither the exact nor the tanh form; the exact one is the
definition). x is (B, T, Dm); W_in, W_gate are (Dm, D); W_out is (D, Dm).

Pinned in tests/test_oracle_block.py: GeLU against values of the normal
distribution function and its odd-part identity; a zero gate weight gives a
zero output; with Dm = D, W_in = W_out = I the output divided by the gate is
the (separately pinned) layer; linearity in W_out; mutants of the block.
"""
from __future__ import annotations

import numpy as np
from scipy.special import erf

from .rglru_oracle import as_f64, rglru_fwd


def gelu(v):
    """GeLU(v) = v * Phi(v), Phi the standard normal distribution function."""
    v = np.asarray(v, dtype=np.float64)
    return 0.5 * v * (1.0 + erf(v / np.sqrt(2.0)))


def block_fwd(x, W_in, W_gate, W_out, conv_w, W_a, b_a, W_x, b_x, Lambda, h0=None,
              conv_state=None):
    """(out, h_T, conv_state_out) of the block for x (B, T, Dm); the state and
    conv history are the layer's (over D channels)."""
    x64 = as_f64(x)
    v = x64 @ as_f64(W_in)
    g = gelu(x64 @ as_f64(W_gate))
    y, h_T, cs = rglru_fwd(v, conv_w, W_a, b_a, W_x, b_x, Lambda, h0=h0, conv_state=conv_state)
    out = (y * g) @ as_f64(W_out)
    return out, h_T, cs
