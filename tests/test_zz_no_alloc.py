"""GPU test of rglru_fwd_noalloc, the forward entry point that allocates nothing.

Some callers cannot allocate device memory once they run: a serving loop that
reserves the whole device for its own pool at start-up, or a plugin inside a
framework that owns the allocator. For them the library keeps its scratch in
a fixed static device array. This test calls that entry point through the C
ABI twice in a row, on different problems (one of them the full B=8, T=2048,
D=1024, H=16 bf16 forward), and checks each result against the ordinary entry
point (which takes a caller workspace) within the parity tolerances of the
other tests. It also checks that a problem too large for the fixed scratch is
refused before anything runs, that invalid sizes get rglru_fwd's status, and
that the Python binding of the entry point gives the same result. This file
sorts last so that a run stopping at the first failure has run every other
test first.
"""
import ctypes

import pytest
import torch

from gated_linear_recurrence_rglru_b200 import _abi
from gated_linear_recurrence_rglru_b200.workloads import WORKLOADS, generate
from oracle.compare import channel_rms, max_rel_err

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
CASES = [
    WORKLOADS["hawk_block"],                                    # the full bf16 forward shape
    WORKLOADS["tiny_f32"].with_shape(B=3, T=133, D=128, H=2, h0_var=1.0, seed=62),
    WORKLOADS["hawk_block"].with_shape(B=2, T=300, D=256, H=4, h0_var=0.5, bias_std=0.3, seed=61),
]


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc_call(g, wl, y, hT, cs):
    lib = _abi.LIB
    io = 0 if wl.io == "f32" else 1
    stream = torch.cuda.current_stream().cuda_stream
    return lib.rglru_fwd_noalloc(
        _p(g["x"]), _p(g["conv_w"]), _p(g["W_a"]), _p(g["b_a"]), _p(g["W_x"]), _p(g["b_x"]),
        _p(g["Lambda"]), _p(g["h0"]), None, _p(y), _p(hT), _p(cs),
        wl.B, wl.T, wl.D, wl.H, io, stream)


def _compare(wl, y, hT, y_ref, h_ref):
    yr = y_ref.float().cpu().numpy()
    e_y = max_rel_err(y.float().cpu().numpy(), yr)
    e_h = max_rel_err(hT.cpu().numpy(), h_ref.cpu().numpy(), scale=channel_rms(yr, 1)[:, 0, :])
    assert e_y <= TOL[wl.io] and e_h <= TOL[wl.io], (wl, e_y, e_h)


def test_noalloc_matches_workspace_entry_point_twice(cuda_device):
    for wl in CASES[:2]:   # two calls in a row, different problems, one shared scratch
        t = generate(wl)
        g = {k: (v.to(cuda_device) if v is not None else None) for k, v in t.items()}
        w = [g[k] for k in ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")]
        y_ref, h_ref, cs_ref = _abi.rglru_fwd(g["x"], *w, h0=g["h0"], algo="generic")
        y = torch.full_like(g["x"], float("nan"))
        hT = torch.full((wl.B, wl.D), float("nan"), device=cuda_device)
        cs = torch.empty(wl.B, 3, wl.D, device=cuda_device, dtype=wl.dtype)
        assert _noalloc_call(g, wl, y, hT, cs) == 0
        torch.cuda.synchronize()
        _compare(wl, y, hT, y_ref, h_ref)
        assert torch.equal(cs, cs_ref)


def test_noalloc_python_binding(cuda_device):
    wl = CASES[2]
    t = generate(wl)
    g = {k: (v.to(cuda_device) if v is not None else None) for k, v in t.items()}
    w = [g[k] for k in ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")]
    y_ref, h_ref, _ = _abi.rglru_fwd(g["x"], *w, h0=g["h0"], algo="generic")
    y = torch.full_like(g["x"], float("nan"))
    hT = torch.full((wl.B, wl.D), float("nan"), device=cuda_device)
    _abi.rglru_fwd_noalloc(g["x"], *w, h0=g["h0"], y=y, h_T=hT)
    torch.cuda.synchronize()
    _compare(wl, y, hT, y_ref, h_ref)
    with pytest.raises(TypeError):
        _abi.rglru_fwd_noalloc(g["x"], *w, h0=g["h0"])       # y is the caller's: required


def test_noalloc_refuses_problems_beyond_its_scratch(cuda_device):
    # B*H = 1 splits T=5000 into 295 segments: 12 B x 295 x 1024 channels > 2 MiB.
    x = torch.zeros(1, 5000, 1024, device=cuda_device, dtype=torch.bfloat16)
    y = torch.full_like(x, 7.0)
    st = _abi.LIB.rglru_fwd_noalloc(_p(x), _p(x), _p(x), _p(x), _p(x), _p(x), _p(x), None,
                                    None, _p(y), None, None, 1, 5000, 1024, 1, 1,
                                    torch.cuda.current_stream().cuda_stream)
    assert st == 5                                  # RGLRU_ERR_WORKSPACE, nothing launched
    # invalid sizes: the status rglru_fwd gives (bw > 1024 is UNSUPPORTED)
    st = _abi.LIB.rglru_fwd_noalloc(_p(x), _p(x), _p(x), _p(x), _p(x), _p(x), _p(x), None,
                                    None, _p(y), None, None, 1, 8, 2048, 1, 1,
                                    torch.cuda.current_stream().cuda_stream)
    assert st == 2
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)
