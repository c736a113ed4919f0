"""B200-native (sm_100a) RG-LRU: the recurrent core of Griffin / Hawk.

The layer: a width-4 causal Conv1D, block-diagonal sigmoid gates, a
log-space decay a_t = a^(8 r_t) and the diagonal recurrence
h_t = a_t h_{t-1} + sqrt(1 - a_t^2) (i_t u_t) (the definition stated in
include/rglru.h; the pages describe the parts: a recurrent gate added to the
LRU and a temporal Conv1D in the recurrent block, S. De's thread on Griffin;
gates that do not read the state, "Beyond Transformer Architecture: Griffin
and Google RecurrentGemma", "Core Components of Griffin", 1. RG-LRU). It is
computed by hand-written CUDA kernels behind a C ABI; this package is the thin
Python binding of that library (_abi.py). rglru_block_fwd adds the recurrent
block around the layer (input and gate projections, GeLU gating, output
projection).

The library is loaded on first use of any binding name below, and that use
raises ImportError if the library is missing (there is no CPU path).
Importing the package, or its `workloads` module (seeded synthetic inputs
only), loads nothing.
"""
__all__ = ["rglru_fwd", "rglru_fwd_noalloc", "rglru_decode_step", "rglru_bwd", "rglru_block_fwd",
           "fwd_workspace_bytes", "bwd_workspace_bytes", "block_fwd_workspace_bytes",
           "fwd_launches", "bwd_launches", "decode_launches", "FwdOptions", "RGLRUError",
           "status_str", "version", "LIB_PATH", "ALGO_AUTO", "ALGO_GENERIC", "ALGO_TENSOR"]


def __getattr__(name):
    if name in __all__:
        from . import _abi
        return getattr(_abi, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")


def __dir__():
    return sorted(list(globals()) + __all__)
