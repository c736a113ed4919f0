"""GPU parity of the backward (rglru_bwd through the C ABI) against the float64
backward oracle (oracle/rglru_backward.py, itself pinned by finite differences).

Bars: fp32 I/O 1e-4, bf16 I/O 2e-2, as for the forward. For bf16 I/O and heads
32, 64 or 128 wide the two in-loop gate contractions run on the tensor cores
with bf16 operands (u and d z rounded like the forward's u), the rest in fp32. dx and the conv
history's gradient use the forward's metric: max |g - o| / max(|o|, per-channel
RMS of o); dh0 is floored at its RMS over the whole tensor. Parameter gradients,
which sum over every token, use the norm-wise max |g - o| / max |o| per tensor.
Cases span several 8-token groups, a ragged tail, one and many segments,
heads from 32 to 1024 channels (every block shape the launcher picks), h0, a
conv history and a state-gradient input dh_T.
"""
import numpy as np
import pytest
import torch

import gated_linear_recurrence_rglru_b200 as rg
from gated_linear_recurrence_rglru_b200.workloads import WORKLOADS, generate
from oracle.compare import BWD_FLOOR, channel_rms, max_rel_err
from oracle.rglru_backward import rglru_bwd as bwd_oracle

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}

CASES = [
    WORKLOADS["tiny_f32"].with_shape(B=2, T=37, D=64, H=2, h0_var=1.0, bias_std=0.5, seed=41),
    WORKLOADS["tiny_f32"].with_shape(B=1, T=600, D=256, H=1, h0_var=0.5, bias_std=0.3, seed=42),
    WORKLOADS["hawk_block"].with_shape(B=2, T=301, D=128, H=2, h0_var=0.5, bias_std=0.5, seed=43),
    WORKLOADS["hawk_block"].with_shape(B=1, T=1100, D=256, H=1, h0_var=0.1, seed=44),
    WORKLOADS["griffin2b"].with_shape(B=1, T=200, D=512, H=2, h0_var=0.1, seed=45),
    # 128-wide heads (4 segments of 128 threads per block), 1024-wide heads
    # (one 1024-thread segment per block) and the hawk_block head layout at full
    # length (64 segments of 32 tokens per sequence, 4 per block)
    WORKLOADS["hawk_block"].with_shape(B=1, T=700, D=256, H=2, h0_var=0.5, seed=46),
    WORKLOADS["tiny_f32"].with_shape(B=1, T=90, D=1024, H=1, h0_var=0.5, seed=47),
    WORKLOADS["hawk_block"].with_shape(B=2, T=2048, D=1024, H=16, h0_var=0.1, seed=48),
    # 32-wide heads (8 segments per block) and 96-wide heads (5 segments of 96
    # threads, weights in shared memory, CUDA-core contractions)
    WORKLOADS["hawk_block"].with_shape(B=2, T=77, D=128, H=4, h0_var=0.5, bias_std=0.5, seed=49),
    WORKLOADS["hawk_block"].with_shape(B=1, T=50, D=192, H=2, h0_var=0.5, seed=50),
    # the bench workload itself (B=8, T=2048, D=1024, H=16, bf16), every output
    WORKLOADS["hawk_block"],
    # shorter than one 8-token group: T = 5 (fp32), 7 (bf16, 32-wide heads), 1 (bf16)
    WORKLOADS["tiny_f32"].with_shape(B=3, T=5, D=64, H=2, h0_var=0.5, bias_std=0.3, seed=52),
    WORKLOADS["hawk_block"].with_shape(B=1, T=7, D=64, H=2, h0_var=0.5, seed=53),
    # B*T = 2 in bf16: below one 8-token group the library takes fp32 operands for the
    # gate contractions (bf16 operands would exceed the bar here by design: see
    # tests/test_backward_bf16_operands.py)
    WORKLOADS["hawk_block"].with_shape(B=2, T=1, D=128, H=2, h0_var=1.0, seed=51),
    # the tensor-core kernels with T shorter than one group (B*T = 12): one segment per
    # sequence whose staged rows are mostly past its end or in the conv history
    WORKLOADS["hawk_block"].with_shape(B=4, T=3, D=256, H=4, h0_var=0.5, bias_std=0.3, seed=54),
]


def _grads(wl, dev, with_csi, with_dhT):
    t = generate(wl)
    g = torch.Generator().manual_seed(wl.seed + 1000)
    dy = torch.randn(wl.B, wl.T, wl.D, generator=g).to(wl.dtype)
    dh_T = torch.randn(wl.B, wl.D, generator=g) if with_dhT else None
    csi = torch.randn(wl.B, 3, wl.D, generator=g).to(wl.dtype) if with_csi else None
    d = lambda v: v.to(dev) if v is not None else None  # noqa: E731
    out = rg.rglru_bwd(d(t["x"]), d(t["conv_w"]), d(t["W_a"]), d(t["b_a"]), d(t["W_x"]),
                       d(t["b_x"]), d(t["Lambda"]), d(dy), h0=d(t["h0"]),
                       conv_state_in=d(csi), dh_T=d(dh_T), want_dh0=True,
                       want_dconv_state=True)
    torch.cuda.synchronize()
    ref = bwd_oracle(t["x"], t["conv_w"], t["W_a"], t["b_a"], t["W_x"], t["b_x"], t["Lambda"],
                     dy, h0=t["h0"], conv_state=csi, dh_T=dh_T)
    return out, ref


def _normwise(g, o):
    den = np.max(np.abs(o))
    return float(np.max(np.abs(g - o)) / den) if den > 0 else float(np.max(np.abs(g)))


@pytest.mark.parametrize("with_csi,with_dhT", [(False, False), (True, True)])
@pytest.mark.parametrize("wl", CASES, ids=lambda w: f"{w.io}-B{w.B}-T{w.T}-D{w.D}-H{w.H}")
def test_backward_matches_oracle(cuda_device, wl, with_csi, with_dhT):
    out, ref = _grads(wl, cuda_device, with_csi, with_dhT)
    tol = TOL[wl.io]
    errs = {}
    dx = out["dx"].float().cpu().numpy()
    errs["dx"] = max_rel_err(dx, ref["dx"], floor=BWD_FLOOR)
    rms = channel_rms(ref["dx"], 1)[:, 0, :]
    # dh0 (B, D): floored at its RMS over the whole tensor (with one batch row a
    # per-channel floor would be |dh0| itself, undefined where it cancels to 0)
    g0, o0 = out["dh0"].cpu().numpy(), ref["dh0"]
    errs["dh0"] = float(np.max(np.abs(g0 - o0) / np.maximum(np.abs(o0), np.sqrt(np.mean(o0 ** 2)))))
    errs["dconv_state"] = max_rel_err(out["dconv_state"].cpu().numpy(), ref["dconv_state"],
                                      scale=rms[:, None, :], floor=BWD_FLOOR)
    for k in ("dconv_w", "dW_a", "db_a", "dW_x", "db_x", "dLambda"):
        errs[k] = _normwise(out[k].cpu().numpy(), ref[k])
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, (wl, bad, errs)


def test_backward_is_deterministic_in_its_sequence_outputs(cuda_device):
    """dx and dh0 come from plain stores (no atomics): two calls agree bit for bit."""
    wl = CASES[2]
    a, _ = _grads(wl, cuda_device, True, True)
    b, _ = _grads(wl, cuda_device, True, True)
    assert torch.equal(a["dx"], b["dx"]) and torch.equal(a["dh0"], b["dh0"])


def test_backward_rejects_aliasing(cuda_device):
    wl = CASES[0]
    t = generate(wl)
    d = {k: (v.to(cuda_device) if v is not None else None) for k, v in t.items()}
    dy = torch.randn_like(d["x"])
    with pytest.raises(rg.RGLRUError) as ei:
        rg.rglru_bwd(d["x"], d["conv_w"], d["W_a"], d["b_a"], d["W_x"], d["b_x"], d["Lambda"],
                     dy, out={"dx": d["x"]})
    assert ei.value.status == 1
