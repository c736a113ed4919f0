"""Error measure used to compare a result with the float64 oracle (test infrastructure).

max relative error = max_i |g_i - o_i| / max(|o_i|, s_i), where s_i is the
root-mean-square of the oracle's output over every batch row and time (or
decode) step of the element's own channel. A pure elementwise relative error
is undefined where h_t crosses zero; the floor at the channel's RMS keeps the
measure relative to the scale of that channel's state, so a wrong term, sign
or index still shows up as an O(1) error while a correct bf16 pipeline, whose
absolute error is a small fraction of the channel's scale, does not. (One
batch row's RMS alone is too small a floor for a few decode steps from a state
that happens to be near zero: the step's increment then dominates the error.)
"""
from __future__ import annotations

import numpy as np

TINY = 1e-30


def channel_rms(o: np.ndarray, time_axis: int = 1) -> np.ndarray:
    """RMS of o per channel (last axis) over all other axes; keepdims.

    time_axis is accepted for call sites that name it; every non-channel axis
    (batch rows and time or decode steps) enters the RMS.
    """
    o = np.asarray(o, dtype=np.float64)
    axes = tuple(range(o.ndim - 1))
    return np.sqrt(np.mean(o * o, axis=axes, keepdims=True))


def max_rel_err(g, o, scale=None, time_axis: int = 1) -> float:
    """max |g - o| / max(|o|, scale); scale defaults to the per-channel RMS of o."""
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    if g.shape != o.shape:
        raise ValueError(f"shape mismatch {g.shape} vs {o.shape}")
    if o.size == 0:
        return 0.0
    if scale is None:
        scale = channel_rms(o, time_axis)
    den = np.maximum(np.maximum(np.abs(o), scale), TINY)
    err = np.abs(g - o) / den
    if not np.all(np.isfinite(g)):
        return float("inf")
    return float(err.max())


def normwise_err(g, o) -> float:
    """||g - o||_inf / ||o||_inf (reported beside the max relative error)."""
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    if o.size == 0:
        return 0.0
    return float(np.abs(g - o).max() / max(np.abs(o).max(), TINY))
