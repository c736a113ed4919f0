"""ctypes binding of librglru_b200.so (argument marshalling only).

Every step of the layer runs in the library's CUDA kernels. This module turns
torch CUDA tensors into device pointers, allocates outputs and workspace
through torch (device memory is PyTorch's job here), passes the current torch
stream, and raises RGLRUError on any nonzero status. If the library is
missing, importing this module fails: there is no CPU path.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librglru_b200.so")

IO_F32, IO_BF16 = 0, 1
ALGO_AUTO, ALGO_GENERIC, ALGO_TENSOR = 0, 1, 2
ALGOS = {"auto": ALGO_AUTO, "generic": ALGO_GENERIC, "tensor": ALGO_TENSOR}

EXPORTED = (
    "rglru_status_str", "rglru_version", "rglru_fwd_workspace_bytes", "rglru_fwd",
    "rglru_fwd_algo", "rglru_decode_step", "rglru_decode_step_algo", "rglru_fwd_launches",
    "rglru_fwd_noalloc", "rglru_decode_launches", "rglru_fwd_ex", "rglru_bwd",
    "rglru_bwd_workspace_bytes", "rglru_bwd_launches", "rglru_block_fwd",
    "rglru_block_fwd_workspace_bytes",
)


class FwdOptions(ctypes.Structure):
    """rglru_fwd_options of include/rglru.h."""
    _fields_ = [("wait_limit_ns", ctypes.c_ulonglong), ("fault_unpublished_tile", ctypes.c_int),
                ("kernel_begin_event", ctypes.c_void_p), ("kernel_end_event", ctypes.c_void_p)]
NOALLOC_SCRATCH_BYTES = 2 << 20  # RGLRU_NOALLOC_SCRATCH_BYTES in include/rglru.h


class RGLRUError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status)} (status {status})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python gated_linear_recurrence_rglru_b200/build.py` (there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, fp, ip, i32, sz = (ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                           ctypes.c_size_t)
    lib.rglru_status_str.restype = ctypes.c_char_p
    lib.rglru_status_str.argtypes = [i32]
    lib.rglru_version.restype = i32
    lib.rglru_version.argtypes = []
    lib.rglru_fwd_workspace_bytes.restype = sz
    lib.rglru_fwd_workspace_bytes.argtypes = [i32] * 5
    lib.rglru_fwd_launches.restype = i32
    lib.rglru_fwd_launches.argtypes = [i32] * 6
    lib.rglru_decode_launches.restype = i32
    lib.rglru_decode_launches.argtypes = [i32] * 5
    fwd_args = [vp] * 6 + [fp, fp, vp, vp, fp, vp] + [i32] * 5 + [vp, sz, ip, vp]
    lib.rglru_fwd.restype = i32
    lib.rglru_fwd.argtypes = fwd_args
    lib.rglru_fwd_algo.restype = i32
    lib.rglru_fwd_algo.argtypes = fwd_args + [i32]
    lib.rglru_fwd_ex.restype = i32
    lib.rglru_fwd_ex.argtypes = fwd_args + [i32, ctypes.POINTER(FwdOptions)]
    lib.rglru_fwd_noalloc.restype = i32
    lib.rglru_fwd_noalloc.argtypes = [vp] * 6 + [fp, fp, vp, vp, fp, vp] + [i32] * 5 + [vp]
    dec_args = [vp, vp, i32, fp, vp] + [vp] * 5 + [fp] + [i32] * 4 + [vp]
    lib.rglru_decode_step.restype = i32
    lib.rglru_decode_step.argtypes = dec_args
    lib.rglru_decode_step_algo.restype = i32
    lib.rglru_decode_step_algo.argtypes = dec_args + [i32]
    lib.rglru_bwd_workspace_bytes.restype = sz
    lib.rglru_bwd_workspace_bytes.argtypes = [i32] * 5
    lib.rglru_bwd_launches.restype = i32
    lib.rglru_bwd_launches.argtypes = [i32] * 5
    lib.rglru_bwd.restype = i32
    lib.rglru_bwd.argtypes = ([vp] * 6 + [fp, fp, vp, vp, fp, vp] + [fp] * 8 + [i32] * 5
                              + [vp, sz, vp])
    lib.rglru_block_fwd_workspace_bytes.restype = sz
    lib.rglru_block_fwd_workspace_bytes.argtypes = [i32] * 6
    lib.rglru_block_fwd.restype = i32
    lib.rglru_block_fwd.argtypes = ([vp] * 9 + [fp, fp, vp, vp, fp, vp] + [i32] * 6
                                    + [vp, sz, ip, vp])
    return lib


LIB = _load()


def status_str(status: int) -> str:
    return LIB.rglru_status_str(int(status)).decode()


def version() -> int:
    return LIB.rglru_version()


def _io_of(dtype: torch.dtype) -> int:
    if dtype == torch.float32:
        return IO_F32
    if dtype == torch.bfloat16:
        return IO_BF16
    raise TypeError(f"unsupported I/O dtype {dtype} (float32 or bfloat16)")


def _ptr(t, name, dtype=None, shape=None, optional=False):
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr()


def _stream_handle(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def fwd_workspace_bytes(B: int, T: int, D: int, H: int, dtype=torch.bfloat16) -> int:
    return int(LIB.rglru_fwd_workspace_bytes(B, T, D, H, _io_of(dtype)))


def fwd_launches(B: int, T: int, D: int, H: int, dtype=torch.bfloat16, algo="auto") -> int:
    """Kernel launches that one rglru_fwd call with these sizes issues."""
    return int(LIB.rglru_fwd_launches(B, T, D, H, _io_of(dtype),
                                      ALGOS[algo] if isinstance(algo, str) else int(algo)))


def decode_launches(B: int, D: int, H: int, dtype=torch.bfloat16, algo="auto") -> int:
    """Kernel launches that one rglru_decode_step call with these sizes issues."""
    return int(LIB.rglru_decode_launches(B, D, H, _io_of(dtype),
                                         ALGOS[algo] if isinstance(algo, str) else int(algo)))


def rglru_fwd(x, conv_w, W_a, b_a, W_x, b_x, Lambda, h0=None, conv_state_in=None, *,
              y=None, h_T=None, conv_state_out=None, workspace=None, dev_status=None,
              stream=None, algo="auto", want_state=True, options=None):
    """Forward of the layer over (B, T, D). Returns (y, h_T, conv_state_out).

    h_T / conv_state_out are None when want_state is False and no buffer is given.
    """
    if x.dim() != 3:
        raise ValueError("x must be (B, T, D)")
    B, T, D = x.shape
    H = W_a.shape[0]
    bw = D // H if H else 0
    dt = x.dtype
    io = _io_of(dt)
    dev = x.device
    if y is None:
        y = torch.empty_like(x)
    if want_state and h_T is None:
        h_T = torch.empty(B, D, device=dev, dtype=torch.float32)
    if want_state and conv_state_out is None:
        conv_state_out = torch.empty(B, 3, D, device=dev, dtype=dt)
    need = fwd_workspace_bytes(B, T, D, H, dt)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=dev, dtype=torch.uint8)
    args = (
        _ptr(x, "x", dt), _ptr(conv_w, "conv_w", dt, (4, D)),
        _ptr(W_a, "W_a", dt, (H, bw, bw)), _ptr(b_a, "b_a", dt, (D,)),
        _ptr(W_x, "W_x", dt, (H, bw, bw)), _ptr(b_x, "b_x", dt, (D,)),
        _ptr(Lambda, "Lambda", torch.float32, (D,)),
        _ptr(h0, "h0", torch.float32, (B, D), optional=True),
        _ptr(conv_state_in, "conv_state_in", dt, (B, 3, D), optional=True),
        _ptr(y, "y", dt, (B, T, D)),
        _ptr(h_T, "h_T", torch.float32, (B, D), optional=True),
        _ptr(conv_state_out, "conv_state_out", dt, (B, 3, D), optional=True),
        B, T, D, H, io,
        _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _ptr(dev_status, "dev_status", torch.int32, optional=True),
        _stream_handle(stream), ALGOS[algo] if isinstance(algo, str) else int(algo),
    )
    st = (LIB.rglru_fwd_ex(*args, ctypes.byref(options)) if options is not None
          else LIB.rglru_fwd_algo(*args))
    if st != 0:
        raise RGLRUError(st, "rglru_fwd")
    return y, h_T, conv_state_out


def rglru_fwd_noalloc(x, conv_w, W_a, b_a, W_x, b_x, Lambda, h0=None, conv_state_in=None, *,
                      y, h_T=None, conv_state_out=None, stream=None):
    """rglru_fwd without a workspace: the library's static device scratch is used.

    For callers that cannot allocate device memory while they run, so every
    output buffer is the caller's: y (B, T, D) is required; h_T and
    conv_state_out are written when given. The call runs with x's device
    current and, unless `stream` is given, on that device's current stream.
    Returns (y, h_T, conv_state_out).
    """
    B, T, D = x.shape
    H = W_a.shape[0]
    bw = D // H if H else 0
    dt = x.dtype
    with torch.cuda.device(x.device):
        st = LIB.rglru_fwd_noalloc(
            _ptr(x, "x", dt), _ptr(conv_w, "conv_w", dt, (4, D)),
            _ptr(W_a, "W_a", dt, (H, bw, bw)), _ptr(b_a, "b_a", dt, (D,)),
            _ptr(W_x, "W_x", dt, (H, bw, bw)), _ptr(b_x, "b_x", dt, (D,)),
            _ptr(Lambda, "Lambda", torch.float32, (D,)),
            _ptr(h0, "h0", torch.float32, (B, D), optional=True),
            _ptr(conv_state_in, "conv_state_in", dt, (B, 3, D), optional=True),
            _ptr(y, "y", dt, (B, T, D)),
            _ptr(h_T, "h_T", torch.float32, (B, D), optional=True),
            _ptr(conv_state_out, "conv_state_out", dt, (B, 3, D), optional=True),
            B, T, D, H, _io_of(dt),
            (stream if stream is not None else torch.cuda.current_stream(x.device)).cuda_stream)
    if st != 0:
        raise RGLRUError(st, "rglru_fwd_noalloc")
    return y, h_T, conv_state_out


def rglru_decode_step(x_t, conv_state, pos, h, conv_w, W_a, b_a, W_x, b_x, Lambda, *,
                      y_t=None, stream=None, algo="auto"):
    """One decode step: updates h and conv_state in place, returns y_t (B, D)."""
    if x_t.dim() != 2:
        raise ValueError("x_t must be (B, D)")
    B, D = x_t.shape
    H = W_a.shape[0]
    bw = D // H if H else 0
    dt = x_t.dtype
    if y_t is None:
        y_t = torch.empty_like(x_t)
    st = LIB.rglru_decode_step_algo(
        _ptr(x_t, "x_t", dt), _ptr(conv_state, "conv_state", dt, (B, 3, D)), int(pos),
        _ptr(h, "h", torch.float32, (B, D)), _ptr(y_t, "y_t", dt, (B, D)),
        _ptr(conv_w, "conv_w", dt, (4, D)), _ptr(W_a, "W_a", dt, (H, bw, bw)),
        _ptr(b_a, "b_a", dt, (D,)), _ptr(W_x, "W_x", dt, (H, bw, bw)),
        _ptr(b_x, "b_x", dt, (D,)), _ptr(Lambda, "Lambda", torch.float32, (D,)),
        B, D, H, _io_of(dt), _stream_handle(stream),
        ALGOS[algo] if isinstance(algo, str) else int(algo))
    if st != 0:
        raise RGLRUError(st, "rglru_decode_step")
    return y_t


def bwd_workspace_bytes(B: int, T: int, D: int, H: int, dtype=torch.bfloat16) -> int:
    return int(LIB.rglru_bwd_workspace_bytes(B, T, D, H, _io_of(dtype)))


def bwd_launches(B: int, T: int, D: int, H: int, dtype=torch.bfloat16) -> int:
    """Kernel launches that one rglru_bwd call with these sizes issues."""
    return int(LIB.rglru_bwd_launches(B, T, D, H, _io_of(dtype)))


def rglru_bwd(x, conv_w, W_a, b_a, W_x, b_x, Lambda, dy, h0=None, conv_state_in=None,
              dh_T=None, *, want_dh0=True, want_dconv_state=False, workspace=None, out=None,
              stream=None):
    """Backward of the layer: gradients of <dy, y> + <dh_T, h_T> with respect to the
    forward inputs (include/rglru.h, rglru_bwd). Returns a dict with dx (the I/O
    dtype), dconv_w, dW_a, db_a, dW_x, db_x, dLambda (fp32), and dh0 / dconv_state
    (fp32, or None when not wanted). `out` may hold preallocated outputs by name."""
    B, T, D = x.shape
    H = W_a.shape[0]
    bw = D // H
    dt = x.dtype
    dev = x.device
    f32 = torch.float32
    o = dict(out or {})

    def buf(name, shape, dtype):
        t = o.get(name)
        return t if t is not None else torch.empty(shape, device=dev, dtype=dtype)

    g = dict(dx=buf("dx", (B, T, D), dt), dconv_w=buf("dconv_w", (4, D), f32),
             dW_a=buf("dW_a", (H, bw, bw), f32), db_a=buf("db_a", (D,), f32),
             dW_x=buf("dW_x", (H, bw, bw), f32), db_x=buf("db_x", (D,), f32),
             dLambda=buf("dLambda", (D,), f32),
             dh0=buf("dh0", (B, D), f32) if want_dh0 else None,
             dconv_state=buf("dconv_state", (B, 3, D), f32) if want_dconv_state else None)
    if workspace is None:
        workspace = torch.empty(max(bwd_workspace_bytes(B, T, D, H, dt), 256), device=dev,
                                dtype=torch.uint8)
    st = LIB.rglru_bwd(
        _ptr(x, "x", dt, (B, T, D)), _ptr(conv_w, "conv_w", dt, (4, D)),
        _ptr(W_a, "W_a", dt, (H, bw, bw)), _ptr(b_a, "b_a", dt, (D,)),
        _ptr(W_x, "W_x", dt, (H, bw, bw)), _ptr(b_x, "b_x", dt, (D,)),
        _ptr(Lambda, "Lambda", f32, (D,)), _ptr(h0, "h0", f32, (B, D), optional=True),
        _ptr(conv_state_in, "conv_state_in", dt, (B, 3, D), optional=True),
        _ptr(dy, "dy", dt, (B, T, D)), _ptr(dh_T, "dh_T", f32, (B, D), optional=True),
        _ptr(g["dx"], "dx", dt, (B, T, D)), _ptr(g["dconv_w"], "dconv_w", f32, (4, D)),
        _ptr(g["dW_a"], "dW_a", f32, (H, bw, bw)), _ptr(g["db_a"], "db_a", f32, (D,)),
        _ptr(g["dW_x"], "dW_x", f32, (H, bw, bw)), _ptr(g["db_x"], "db_x", f32, (D,)),
        _ptr(g["dLambda"], "dLambda", f32, (D,)),
        _ptr(g["dh0"], "dh0", f32, (B, D), optional=True),
        _ptr(g["dconv_state"], "dconv_state", f32, (B, 3, D), optional=True),
        B, T, D, H, _io_of(dt), _ptr(workspace, "workspace"), workspace.numel(),
        _stream_handle(stream))
    if st != 0:
        raise RGLRUError(st, "rglru_bwd")
    return g


def block_fwd_workspace_bytes(B: int, T: int, Dm: int, D: int, H: int,
                              dtype=torch.bfloat16) -> int:
    """Workspace of rglru_block_fwd (include/rglru.h)."""
    n = LIB.rglru_block_fwd_workspace_bytes(B, T, Dm, D, H, _io_of(dtype))
    if n == 0:
        raise RGLRUError(1, "rglru_block_fwd_workspace_bytes")
    return n


def rglru_block_fwd(x, W_in, W_gate, W_out, conv_w, W_a, b_a, W_x, b_x, Lambda, h0=None,
                    conv_state_in=None, *, out=None, h_T=None, conv_state_out=None,
                    workspace=None, dev_status=None, stream=None, want_state=True):
    """Recurrent block around the layer (include/rglru.h, rglru_block_fwd):
    out = (layer(x W_in) * GeLU(x W_gate)) W_out over x (B, T, Dm).
    Returns (out, h_T, conv_state_out) of the layer inside."""
    if x.dim() != 3:
        raise ValueError("x must be (B, T, Dm)")
    B, T, Dm = x.shape
    D = W_in.shape[1]
    H = W_a.shape[0]
    bw = D // H if H else 0
    dt = x.dtype
    io = _io_of(dt)
    dev = x.device
    if out is None:
        out = torch.empty_like(x)
    if want_state and h_T is None:
        h_T = torch.empty(B, D, device=dev, dtype=torch.float32)
    if want_state and conv_state_out is None:
        conv_state_out = torch.empty(B, 3, D, device=dev, dtype=dt)
    if workspace is None:
        workspace = torch.empty(block_fwd_workspace_bytes(B, T, Dm, D, H, dt), device=dev,
                                dtype=torch.uint8)
    st = LIB.rglru_block_fwd(
        _ptr(x, "x", dt), _ptr(W_in, "W_in", dt, (Dm, D)), _ptr(W_gate, "W_gate", dt, (Dm, D)),
        _ptr(W_out, "W_out", dt, (D, Dm)), _ptr(conv_w, "conv_w", dt, (4, D)),
        _ptr(W_a, "W_a", dt, (H, bw, bw)), _ptr(b_a, "b_a", dt, (D,)),
        _ptr(W_x, "W_x", dt, (H, bw, bw)), _ptr(b_x, "b_x", dt, (D,)),
        _ptr(Lambda, "Lambda", torch.float32, (D,)),
        _ptr(h0, "h0", torch.float32, (B, D), optional=True),
        _ptr(conv_state_in, "conv_state_in", dt, (B, 3, D), optional=True),
        _ptr(out, "out", dt, (B, T, Dm)),
        _ptr(h_T, "h_T", torch.float32, (B, D), optional=True),
        _ptr(conv_state_out, "conv_state_out", dt, (B, 3, D), optional=True),
        B, T, Dm, D, H, io,
        _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _ptr(dev_status, "dev_status", torch.int32, optional=True), _stream_handle(stream))
    if st != 0:
        raise RGLRUError(st, "rglru_block_fwd")
    return out, h_T, conv_state_out

