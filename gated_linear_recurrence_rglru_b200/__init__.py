"""B200-native (sm_100a) RG-LRU: the recurrent core of Griffin / Hawk.

The layer ("Griffin: Mixing Gated Linear Recurrences with Local Attention for
Efficient Language Models", section "Model Architecture"): a width-4 causal
Conv1D, block-diagonal sigmoid gates, a log-space decay a_t = a^(8 r_t) and the
diagonal recurrence h_t = a_t h_{t-1} + sqrt(1 - a_t^2) (i_t u_t), computed by
hand-written CUDA kernels behind a C ABI (include/rglru.h). This package is the
thin Python binding of that library; see _abi.py. rglru_block_fwd adds the
recurrent block around the layer (input and gate projections, GeLU gating,
output projection).
"""
from ._abi import (ALGO_AUTO, ALGO_GENERIC, ALGO_TENSOR, LIB_PATH, FwdOptions,  # noqa: F401
                   RGLRUError, block_fwd_workspace_bytes, bwd_launches, bwd_workspace_bytes,
                   decode_launches, fwd_launches, fwd_workspace_bytes, rglru_block_fwd, rglru_bwd,
                   rglru_decode_step, rglru_fwd, rglru_fwd_noalloc, status_str, version)

__all__ = ["rglru_fwd", "rglru_fwd_noalloc", "rglru_decode_step", "rglru_bwd", "rglru_block_fwd",
           "fwd_workspace_bytes", "bwd_workspace_bytes", "block_fwd_workspace_bytes",
           "fwd_launches", "bwd_launches", "decode_launches", "FwdOptions", "RGLRUError",
           "status_str", "version", "LIB_PATH"]
