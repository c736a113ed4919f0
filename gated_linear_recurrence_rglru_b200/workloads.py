"""Seeded synthetic workloads for the RG-LRU layer.

This module only draws random inputs. It holds none of the layer's
arithmetic and is the one module that the CUDA path's callers (tests, bench,
smoke) and the float64 oracle share: both sides receive the very same tensors.

The five named workloads are the Griffin / Hawk recurrent-core shapes this
library is measured on (the RG-LRU layer with the temporal Conv1D of its
recurrent block, S. De's thread on Griffin; training sequences of 2048 tokens
and extrapolation to longer ones, "Beyond Transformer Architecture: Griffin and
Google RecurrentGemma", "Technical Foundations of RecurrentGemma"):

  tiny_f32       B=1    T=256    D=256  H=4   fp32 I/O        a^8 ~ U[0.9, 0.999]
  hawk_block     B=8    T=2048   D=1024 H=16  bf16 I/O        a^8 ~ U[0.9, 0.999]
  griffin2b      B=16   T=4096   D=2560 H=10  bf16 I/O        a^8 ~ U[0.9, 0.999], h0 ~ N(0, 0.1)
  long_context   B=1    T=131072 D=4096 H=16  bf16 I/O        a^8 ~ U[0.99, 0.9999]
  decode_batch   B=1024 D=4096   H=16, 256 decode steps, bf16 x_t and conv ring, fp32 state

Recipe (every workload, in this draw order from one torch CPU generator):
  x      ~ N(0, 1)                    stored in the I/O dtype
  conv_w ~ N(0, 1/4)  (variance)      shape (4, D), tap k multiplies x[t-3+k]
  W_a    ~ N(0, 1/64) (variance)      shape (H, bw, bw), z[j] = sum_i u[i] W[i, j]
  W_x    ~ N(0, 1/64) (variance)
  s      ~ U[lo, hi] per channel; a = s**(1/8); Lambda = log(a / (1 - a))
         (so sigmoid(Lambda) = a and a**8 = s: the "a^c" spread of the workload)
  h0     ~ N(0, var) when var > 0, else absent (zeros)
  b_a = b_x = 0     (parity cases may instead draw them last, ~ N(0, bias_std^2))
Lambda, h0 and every recurrent state are fp32 whatever the I/O dtype.
The decode workload then draws h ~ N(0, 1), the conv ring ~ N(0, 1) and the
256 per-step inputs x_t ~ N(0, 1).
The recurrent block around the layer (generate_block) adds, from a second
generator, the block input x (B, T, Dm) ~ N(0, 1) and its projections W_in,
W_gate (Dm, D) ~ N(0, 1/Dm) and W_out (D, Dm) ~ N(0, 1/D).
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    D: int
    H: int
    io: str                 # "f32" or "bf16"
    seed: int
    ac_lo: float            # a^8 ~ U[ac_lo, ac_hi] per channel
    ac_hi: float
    h0_var: float = 0.0
    w_var: float = 1.0 / 64.0
    conv_var: float = 0.25
    decode_steps: int = 0   # > 0 marks a decode workload (T is then 1 per step)
    bias_std: float = 0.0   # > 0 draws b_a, b_x ~ N(0, bias_std^2) last (parity cases only)

    @property
    def bw(self) -> int:
        return self.D // self.H

    @property
    def dtype(self) -> torch.dtype:
        return torch.float32 if self.io == "f32" else torch.bfloat16

    def with_shape(self, **kw) -> "Workload":
        """Same recipe and seed, different sizes (parity cases at small sizes)."""
        return dataclasses.replace(self, **kw)

    def channel_tokens(self) -> int:
        if self.decode_steps:
            return self.B * self.D * self.decode_steps
        return self.B * self.T * self.D


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", B=1, T=256, D=256, H=4, io="f32", seed=0,
                         ac_lo=0.9, ac_hi=0.999),
    "hawk_block": Workload("hawk_block", B=8, T=2048, D=1024, H=16, io="bf16", seed=1,
                           ac_lo=0.9, ac_hi=0.999),
    "griffin2b": Workload("griffin2b", B=16, T=4096, D=2560, H=10, io="bf16", seed=2,
                          ac_lo=0.9, ac_hi=0.999, h0_var=0.1),
    "long_context": Workload("long_context", B=1, T=131072, D=4096, H=16, io="bf16", seed=3,
                             ac_lo=0.99, ac_hi=0.9999),
    "decode_batch": Workload("decode_batch", B=1024, T=1, D=4096, H=16, io="bf16", seed=4,
                             ac_lo=0.9, ac_hi=0.999, decode_steps=256),
}


def _normal(gen: torch.Generator, shape, std: float, dtype: torch.dtype) -> torch.Tensor:
    t = torch.randn(shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def lambda_from_ac(s: torch.Tensor) -> torch.Tensor:
    """Lambda with sigmoid(Lambda)**8 == s, built in float64, stored fp32."""
    a = s.double() ** (1.0 / 8.0)
    return (torch.log(a) - torch.log1p(-a)).float()


def generate(wl: Workload) -> dict:
    """Draw the layer's parameters and inputs (CPU tensors) for a workload."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(wl.seed)
    B, T, D, H = wl.B, wl.T, wl.D, wl.H
    if D % H:
        raise ValueError("D must be a multiple of H")
    bw = D // H
    dt = wl.dtype
    out = {}
    if wl.decode_steps:
        out["x_steps"] = _normal(gen, (wl.decode_steps, B, D), 1.0, dt)
    else:
        out["x"] = _normal(gen, (B, T, D), 1.0, dt)
    out["conv_w"] = _normal(gen, (4, D), math.sqrt(wl.conv_var), dt)
    out["W_a"] = _normal(gen, (H, bw, bw), math.sqrt(wl.w_var), dt)
    out["W_x"] = _normal(gen, (H, bw, bw), math.sqrt(wl.w_var), dt)
    out["b_a"] = torch.zeros(D, dtype=dt)
    out["b_x"] = torch.zeros(D, dtype=dt)
    s = torch.rand(D, generator=gen, dtype=torch.float64) * (wl.ac_hi - wl.ac_lo) + wl.ac_lo
    out["Lambda"] = lambda_from_ac(s)
    if wl.decode_steps:
        out["h"] = _normal(gen, (B, D), 1.0, torch.float32)
        out["conv_state"] = _normal(gen, (B, 3, D), 1.0, dt)
    else:
        out["h0"] = (_normal(gen, (B, D), math.sqrt(wl.h0_var), torch.float32)
                     if wl.h0_var > 0 else None)
    if wl.bias_std > 0:
        out["b_a"] = _normal(gen, (D,), wl.bias_std, dt)
        out["b_x"] = _normal(gen, (D,), wl.bias_std, dt)
    return out


def generate_block(wl: Workload, Dm: int) -> dict:
    """Inputs of the recurrent block around the layer: the layer's parameters of
    generate(wl) (its x unused), the block input x (B, T, Dm) ~ N(0, 1) and the
    projections W_in, W_gate (Dm, D) ~ N(0, 1/Dm), W_out (D, Dm) ~ N(0, 1/D)
    (variance 1/fan-in), drawn in that order from a second generator seeded
    with seed + 7919."""
    out = generate(wl)
    out.pop("x", None)
    gen = torch.Generator(device="cpu")
    gen.manual_seed(wl.seed + 7919)
    B, T, D = wl.B, wl.T, wl.D
    dt = wl.dtype
    out["x"] = _normal(gen, (B, T, Dm), 1.0, dt)
    out["W_in"] = _normal(gen, (Dm, D), 1.0 / math.sqrt(Dm), dt)
    out["W_gate"] = _normal(gen, (Dm, D), 1.0 / math.sqrt(Dm), dt)
    out["W_out"] = _normal(gen, (D, Dm), 1.0 / math.sqrt(D), dt)
    return out

