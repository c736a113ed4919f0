"""Time-sharded forward (gated_linear_recurrence_rglru_b200.tsharded) with gloo
ranks on the CPU: every rank holds one time segment of the sequence, runs the
rank-local forward (here the float64 oracle, standing in for the CUDA library),
and exchanges only the Conv1D halo and the (A, H) segment aggregates. The
gathered result must equal the oracle over the whole sequence, including
segments shorter than the three-token Conv1D history, a nonzero h0 and a
caller conv history before the first segment."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_linear_recurrence_rglru_b200 import tsharded
from gated_linear_recurrence_rglru_b200.workloads import WORKLOADS, generate
from oracle import rglru_oracle as orc

KEYS = ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_fwd(x, conv_w, W_a, b_a, W_x, b_x, Lambda, h0=None, conv_state_in=None):
    y, hT, cs = orc.rglru_fwd(x, conv_w, W_a, b_a, W_x, b_x, Lambda, h0=h0,
                              conv_state=conv_state_in)
    return torch.from_numpy(y), torch.from_numpy(hT), torch.from_numpy(cs)


def _case(seed):
    wl = WORKLOADS["hawk_block"].with_shape(B=2, T=sum((9, 1, 2, 7)), D=64, H=2, io="f32",
                                            h0_var=0.5, bias_std=0.5, seed=seed)
    t = generate(wl)
    g = torch.Generator().manual_seed(seed + 1)
    t["conv_state_in"] = torch.randn(wl.B, 3, wl.D, generator=g)
    return {k: (v.double() if isinstance(v, torch.Tensor) else v) for k, v in t.items()}


def _worker(rank, ws, port, lengths, seed, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        t = _case(seed)
        t0 = sum(lengths[:rank])
        x_local = t["x"][:, t0:t0 + lengths[rank]].contiguous()
        y, hT = tsharded.rglru_fwd_tsharded(x_local, *[t[k] for k in KEYS], h0=t["h0"],
                                            conv_state_in=t["conv_state_in"], fwd=_oracle_fwd)
        out[rank] = (y.numpy(), hT.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lengths", [(10, 9), (9, 1, 2, 7)])
def test_tsharded_matches_the_whole_sequence(lengths):
    ws = len(lengths)
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, ws, port, lengths, 71, out)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    t = _case(71)
    yo, hTo, _ = orc.rglru_fwd(t["x"], *[t[k] for k in KEYS], h0=t["h0"],
                               conv_state=t["conv_state_in"])
    y = np.concatenate([out[r][0] for r in range(ws)], axis=1)
    np.testing.assert_allclose(y, yo, rtol=1e-11, atol=1e-12)
    for r in range(ws):
        np.testing.assert_allclose(out[r][1], hTo, rtol=1e-11, atol=1e-12)


def test_aggregates_compose_like_the_scan():
    """The affine form h_T(h0) = A h0 + H that the exchange relies on, with A from
    the shut input gate: checked on the oracle for one segment."""
    t = _case(72)
    w = [t[k] for k in KEYS]
    x = t["x"][:, :6]
    B, D = x.shape[0], x.shape[2]
    _, H, _ = _oracle_fwd(x, *w, h0=torch.zeros(B, D))
    shut = torch.full_like(t["b_x"], tsharded.GATE_SHUT)
    _, A, _ = _oracle_fwd(x, *w[:4], shut, w[5], h0=torch.ones(B, D))
    it = orc.intermediates(x, *w)
    np.testing.assert_allclose(A.numpy(), np.prod(it["a"], axis=1), rtol=1e-13)
    h0 = t["h0"]
    _, hT, _ = _oracle_fwd(x, *w, h0=h0)
    np.testing.assert_allclose(hT.numpy(), A.numpy() * h0.numpy() + H.numpy(), rtol=1e-12,
                               atol=1e-14)
