"""Time-sharded forward of the layer over ranks (torch.distributed).

A sequence too long for one GPU is cut along time: rank r holds tokens
[t_r, t_{r+1}) of every batch row. The layer's state is the only thing that
crosses a cut, plus the Conv1D's last three inputs:

  1. halo: each rank gathers the last (up to) three inputs of every rank and
     builds its Conv1D history from its predecessors (and the caller's
     conv_state_in before rank 0), so a segment shorter than three tokens is
     handled too;
  2. segment aggregates: the layer is affine in its initial state, h_T(h0) =
     A h0 + H with A = prod of a_t over the segment and H the state reached
     from zero (the two-level scan of the carry: (A1, H1) o (A2, H2) =
     (A1 A2, A2 H1 + H2)). H is the final state of a forward from h0 = 0; A is
     the final state of a forward from h0 = 1 with the input gate shut
     (b_x = -1e4 makes i = sigmoid(z_x) exactly 0, so the input term vanishes
     while a_t, which reads only the recurrence gate, is unchanged);
  3. one all-gather of (A, H), 8 bytes per channel per rank, and an exclusive
     scan over ranks in order from the caller's h0 gives each rank its
     entering state h_in;
  4. the rank's forward from h_in gives its part of y.

This is the exchange step that sharding over time needs ("Beyond Transformer
Architecture: Griffin and Google RecurrentGemma", "Key Strengths of
RecurrentGemma", 1. Reduced Memory Usage: the state has a fixed size, so the
exchange is independent of the sequence length). The per-rank forward is the
library's rglru_fwd by default; `fwd` may name another implementation of the
same call (tests pass a CPU one). Each rank runs three forwards of its segment:
the two state-only ones of step 2 and the final one.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

GATE_SHUT = -1.0e4   # b_x that makes the input gate exactly 0


def _default_fwd():
    from . import _abi
    return _abi.rglru_fwd


def _gather(t: torch.Tensor, group) -> list:
    """all_gather of a small tensor: on the device under NCCL, through host copies
    under a CPU backend (gloo), returned on t's device either way."""
    ws = dist.get_world_size(group)
    on_host = t.is_cuda and dist.get_backend(group) != "nccl"
    src = t.cpu() if on_host else t
    out = [torch.empty_like(src) for _ in range(ws)]
    dist.all_gather(out, src.contiguous(), group=group)
    return [o.to(t.device) for o in out] if on_host else out


def conv_history(x_local: torch.Tensor, conv_state_in, group=None) -> torch.Tensor:
    """This rank's chronological Conv1D history (B, 3, D): the three inputs before
    its first token, taken from the preceding ranks' segments (and conv_state_in,
    the history before rank 0's first token, zeros if None)."""
    rank = dist.get_rank(group)
    B, T, D = x_local.shape
    tail = torch.zeros(B, 3, D, dtype=x_local.dtype, device=x_local.device)
    n = min(T, 3)
    if n:
        tail[:, 3 - n:] = x_local[:, T - n:]
    lengths = _gather(torch.tensor([T], dtype=torch.int64, device=x_local.device), group)
    tails = _gather(tail, group)
    hist = (torch.zeros(B, 3, D, dtype=x_local.dtype, device=x_local.device)
            if conv_state_in is None else conv_state_in.clone())
    for r in range(rank):                     # walk the earlier ranks in time order
        k = min(int(lengths[r].item()), 3)
        if k:
            hist = torch.cat([hist, tails[r][:, 3 - k:]], dim=1)[:, -3:]
    return hist.contiguous()


def entering_states(A: torch.Tensor, H: torch.Tensor, h0, group=None):
    """Exclusive scan of the segment aggregates over ranks: the state entering
    this rank's segment and the state after the last rank's (both (B, D) fp32)."""
    rank = dist.get_rank(group)
    As, Hs = _gather(A, group), _gather(H, group)
    h = torch.zeros_like(H) if h0 is None else h0.to(H.dtype).clone()
    h_in = None
    for r in range(len(As)):
        if r == rank:
            h_in = h.clone()
        h = As[r] * h + Hs[r]
    return h_in, h


def rglru_fwd_tsharded(x_local, conv_w, W_a, b_a, W_x, b_x, Lambda, h0=None,
                       conv_state_in=None, *, group=None, fwd=None):
    """Forward of the layer over a sequence cut along time across the ranks of
    `group`; this rank holds x_local (B, T_r, D). Returns (y_local, h_T), h_T
    being the state after the whole sequence (the same on every rank).

    h0 and conv_state_in are the states before the whole sequence (rank 0's
    segment); every rank passes the same ones (or None)."""
    fwd = fwd or _default_fwd()
    B, T, D = x_local.shape
    hist = conv_history(x_local, conv_state_in, group)
    zeros = torch.zeros(B, D, dtype=torch.float32, device=x_local.device)
    ones = torch.ones(B, D, dtype=torch.float32, device=x_local.device)
    shut = torch.full_like(b_x, GATE_SHUT)
    w = (conv_w, W_a, b_a, W_x)
    _, H, _ = fwd(x_local, *w, b_x, Lambda, h0=zeros, conv_state_in=hist)
    _, A, _ = fwd(x_local, *w, shut, Lambda, h0=ones, conv_state_in=hist)
    h_in, h_T = entering_states(A, H, h0, group)
    y, _, _ = fwd(x_local, *w, b_x, Lambda, h0=h_in, conv_state_in=hist)
    return y, h_T
