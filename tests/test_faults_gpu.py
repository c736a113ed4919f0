"""Failure detection on the GPU without a GPU fault: a tile that never
publishes its carry (a flag that nothing sets) makes its successors' bounded
waits run out; the kernel must report RGLRU_ERR_TIMEOUT through the status
word, return in bounded time, and leave the context usable."""
import time

import numpy as np
import pytest
import torch

import gated_linear_recurrence_rglru_b200 as rg
from gated_linear_recurrence_rglru_b200._abi import FwdOptions
from gated_linear_recurrence_rglru_b200.workloads import WORKLOADS, generate
from oracle import rglru_oracle as orc
from oracle.compare import max_rel_err

pytestmark = pytest.mark.gpu

WL = WORKLOADS["hawk_block"].with_shape(B=1, T=64 * 12, D=128, H=2, seed=71)


def _inputs(dev):
    t = generate(WL)
    return t, {k: (v.to(dev) if v is not None else None) for k, v in t.items()}


def test_unpublished_tile_times_out_and_context_survives(cuda_device):
    t, g = _inputs(cuda_device)
    w = [g[k] for k in ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")]
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    opts = FwdOptions(wait_limit_ns=50_000_000, fault_unpublished_tile=4)   # tile 3
    t0 = time.time()
    rg.rglru_fwd(g["x"], *w, algo="tensor", dev_status=status, options=opts)
    torch.cuda.synchronize()
    word = int(status.item())
    assert word & 0xFF == 4                         # RGLRU_ERR_TIMEOUT
    assert (word >> 8) & 0xFF == 5                  # ... in the look-back for a carry word
    assert time.time() - t0 < 20.0
    # same context, normal call: correct again
    status.zero_()
    y, _, _ = rg.rglru_fwd(g["x"], *w, algo="tensor", dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    yo, _, _ = orc.rglru_fwd(t["x"], t["conv_w"], t["W_a"], t["b_a"], t["W_x"], t["b_x"],
                             t["Lambda"])
    assert max_rel_err(y.float().cpu().numpy(), yo) <= 2e-2


def test_unpublished_tile_times_out_with_wide_heads(cuda_device):
    """The same with 256-wide heads (32-token tiles, gate weights in TMEM, two
    units per head): the stalled tile's look-back names the failure and the
    next call is correct."""
    wl = WORKLOADS["hawk_block"].with_shape(B=1, T=32 * 12, D=512, H=2, seed=73)
    t = generate(wl)
    g = {k: (v.to(cuda_device) if v is not None else None) for k, v in t.items()}
    w = [g[k] for k in ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")]
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    opts = FwdOptions(wait_limit_ns=50_000_000, fault_unpublished_tile=4)
    t0 = time.time()
    rg.rglru_fwd(g["x"], *w, algo="tensor", dev_status=status, options=opts)
    torch.cuda.synchronize()
    word = int(status.item())
    assert word & 0xFF == 4
    assert (word >> 8) & 0xFF == 5
    assert time.time() - t0 < 20.0
    status.zero_()
    y, _, _ = rg.rglru_fwd(g["x"], *w, algo="tensor", dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    yo, _, _ = orc.rglru_fwd(t["x"], t["conv_w"], t["W_a"], t["b_a"], t["W_x"], t["b_x"],
                             t["Lambda"])
    assert max_rel_err(y.float().cpu().numpy(), yo) <= 2e-2


def test_too_short_wait_limit_is_refused(cuda_device):
    _, g = _inputs(cuda_device)
    w = [g[k] for k in ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")]
    with pytest.raises(rg.RGLRUError) as ei:
        rg.rglru_fwd(g["x"], *w, algo="tensor", options=FwdOptions(wait_limit_ns=1000))
    assert ei.value.status == 1
    with pytest.raises(rg.RGLRUError) as ei:
        rg.rglru_fwd(g["x"], *w, algo="tensor", options=FwdOptions(fault_unpublished_tile=-1))
    assert ei.value.status == 1


def test_zeroed_options_with_kernel_events(cuda_device):
    """Zero-initialised options are the defaults (no fault); the kernel events
    they carry are recorded around the compute kernel."""
    t, g = _inputs(cuda_device)
    w = [g[k] for k in ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")]
    eb, ee = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    eb.record()
    ee.record()
    torch.cuda.synchronize()
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    opts = FwdOptions(kernel_begin_event=eb.cuda_event, kernel_end_event=ee.cuda_event)
    y, _, _ = rg.rglru_fwd(g["x"], *w, algo="tensor", dev_status=status, options=opts)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert 0.0 < eb.elapsed_time(ee) < 1000.0
    yo, _, _ = orc.rglru_fwd(t["x"], t["conv_w"], t["W_a"], t["b_a"], t["W_x"], t["b_x"],
                             t["Lambda"])
    assert max_rel_err(y.float().cpu().numpy(), yo) <= 2e-2
