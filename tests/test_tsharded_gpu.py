"""Time-sharded forward through the CUDA library: two ranks (processes) on
cuda:0 exchange the Conv1D halo and the (A, H) segment aggregates through gloo
(host copies; no kernel of one rank waits on the other's), each runs the
library's forward on its segment, and the gathered result must match the
float64 oracle over the whole sequence within the parity bars."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_linear_recurrence_rglru_b200.workloads import WORKLOADS, generate
from oracle import rglru_oracle as orc
from oracle.compare import channel_rms, max_rel_err

pytestmark = pytest.mark.gpu

KEYS = ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")
TOL = {"f32": 1e-4, "bf16": 2e-2}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case(io):
    wl = WORKLOADS["long_context"].with_shape(B=2, T=700, D=256, H=2, io=io, h0_var=0.5,
                                              bias_std=0.3, seed=91)
    t = generate(wl)
    t["conv_state_in"] = torch.randn(wl.B, 3, wl.D,
                                     generator=torch.Generator().manual_seed(92)).to(wl.dtype)
    return wl, t


def _worker(rank, ws, port, io, lengths, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        from gated_linear_recurrence_rglru_b200 import tsharded
        dev = torch.device("cuda:0")
        wl, t = _case(io)
        g = {k: (v.to(dev) if v is not None else None) for k, v in t.items()}
        t0 = sum(lengths[:rank])
        x_local = g["x"][:, t0:t0 + lengths[rank]].contiguous()
        y, hT = tsharded.rglru_fwd_tsharded(x_local, *[g[k] for k in KEYS], h0=g["h0"],
                                            conv_state_in=g["conv_state_in"])
        torch.cuda.synchronize()
        out[rank] = (y.float().cpu().numpy(), hT.cpu().numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_tsharded_forward_two_ranks(cuda_device, io):
    lengths = (411, 289)
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, io, lengths, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=600)
        assert p.exitcode == 0
    wl, t = _case(io)
    yo, hTo, _ = orc.rglru_fwd(t["x"], *[t[k] for k in KEYS], h0=t["h0"],
                               conv_state=t["conv_state_in"])
    y = np.concatenate([out[r][0] for r in range(2)], axis=1)
    e_y = max_rel_err(y, yo)
    e_h = max(max_rel_err(out[r][1], hTo, scale=channel_rms(yo, 1)[:, 0, :]) for r in range(2))
    assert e_y <= TOL[io] and e_h <= TOL[io], (e_y, e_h)
