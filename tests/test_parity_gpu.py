"""GPU parity: the CUDA library (through the C ABI) against the float64 oracle.

Bars (max relative error, floored at 0.75 times the channel RMS, a floor derived
in oracle/compare.py and tests/test_bf16_operand_rounding.py): fp32 I/O 1e-4,
bf16 I/O (fp32 state) 2e-2. Output buffers start as NaN, so an element the
kernels never write fails the comparison. The conv state outputs are copies
of inputs and must match bit for bit. Small cases span several tiles and a
ragged tail; the full-size workloads run in the bench's launch configuration
and are checked on whole (batch row) or (head) blocks, which the layer keeps
independent of each other, so the sampled check is exact for those blocks.
"""
import numpy as np
import pytest
import torch

import gated_linear_recurrence_rglru_b200 as rg
from gated_linear_recurrence_rglru_b200.workloads import WORKLOADS, generate
from oracle import rglru_oracle as orc
from oracle.compare import channel_rms, max_rel_err

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
ALGOS = ["generic", "tensor"]
DEC_ALGOS = ["generic", "tensor"]


def need_algo(wl, algo):
    """Skip when the algorithm does not cover this shape / dtype (e.g. tensor needs bf16)."""
    if rg.fwd_launches(wl.B, wl.T, wl.D, wl.H, wl.dtype, algo) == 0:
        pytest.skip(f"{algo} does not cover {wl}")


def to_dev(t, dev):
    return {k: (v.to(dev) if v is not None else None) for k, v in t.items()}


def check_fwd(wl, algo, dev, with_csi=False, csi_seed=11):
    need_algo(wl, algo)
    t = generate(wl)
    csi = None
    if with_csi:
        g = torch.Generator().manual_seed(csi_seed)
        csi = torch.randn(wl.B, 3, wl.D, generator=g).to(wl.dtype)
    g = to_dev(t, dev)
    # outputs start as NaN: every element must be written
    y = torch.full_like(g["x"], float("nan"))
    hT = torch.full((wl.B, wl.D), float("nan"), device=dev)
    cs = torch.full((wl.B, 3, wl.D), float("nan"), device=dev, dtype=wl.dtype)
    rg.rglru_fwd(g["x"], g["conv_w"], g["W_a"], g["b_a"], g["W_x"], g["b_x"], g["Lambda"],
                 h0=g["h0"], conv_state_in=csi.to(dev) if csi is not None else None, algo=algo,
                 y=y, h_T=hT, conv_state_out=cs)
    torch.cuda.synchronize()
    yo, hTo, cso = orc.rglru_fwd(t["x"], t["conv_w"], t["W_a"], t["b_a"], t["W_x"], t["b_x"],
                                 t["Lambda"], h0=t["h0"], conv_state=csi)
    e_y = max_rel_err(y.float().cpu().numpy(), yo)
    e_h = max_rel_err(hT.cpu().numpy(), hTo, scale=channel_rms(yo, 1)[:, 0, :])
    assert np.array_equal(cs.float().cpu().numpy(), cso), "conv_state_out differs"
    tol = TOL[wl.io]
    assert e_y <= tol and e_h <= tol, (wl, algo, e_y, e_h)
    return e_y, e_h


SMALL = [
    WORKLOADS["tiny_f32"],
    WORKLOADS["tiny_f32"].with_shape(B=2, T=37, D=64, H=2, h0_var=1.0, bias_std=0.5, seed=21),
    WORKLOADS["tiny_f32"].with_shape(B=1, T=1, D=32, H=1, h0_var=1.0, seed=22),
    WORKLOADS["tiny_f32"].with_shape(B=3, T=2, D=48, H=3, seed=23),
    WORKLOADS["hawk_block"].with_shape(B=2, T=300, D=256, H=4, h0_var=0.5, bias_std=0.5, seed=31),
    WORKLOADS["hawk_block"].with_shape(B=3, T=129, D=256, H=2, seed=32),
    WORKLOADS["hawk_block"].with_shape(B=1, T=200, D=512, H=2, h0_var=0.1, seed=33),
    WORKLOADS["hawk_block"].with_shape(B=1, T=3, D=128, H=1, seed=34),
    WORKLOADS["long_context"].with_shape(B=1, T=5000, D=256, H=2, seed=35),
    WORKLOADS["long_context"].with_shape(B=1, T=1000, D=512, H=2, seed=36),
    WORKLOADS["griffin2b"].with_shape(B=3, T=100, D=768, H=3, bias_std=0.5, seed=37),
    WORKLOADS["hawk_block"].with_shape(B=2, T=1, D=128, H=2, h0_var=1.0, seed=38),
    WORKLOADS["hawk_block"].with_shape(B=2, T=64, D=256, H=4, seed=39),
    WORKLOADS["hawk_block"].with_shape(B=2, T=65, D=256, H=2, h0_var=1.0, seed=40),
    # 256-wide heads: a sequence shorter than the Conv1D history; one token past
    # a 32-token tile with several rows and heads
    WORKLOADS["hawk_block"].with_shape(B=2, T=2, D=512, H=2, h0_var=1.0, seed=43),
    WORKLOADS["hawk_block"].with_shape(B=3, T=33, D=1024, H=4, bias_std=0.5, seed=44),
    # 256-wide heads, 144 units of 7 tiles on 148 CTAs: CTAs steal from one another's
    # units and reload the staged TMEM weights many times
    WORKLOADS["griffin2b"].with_shape(B=24, T=200, D=768, H=3, bias_std=0.5, seed=46),
]


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("idx", range(len(SMALL)))
def test_fwd_small(cuda_device, algo, idx):
    check_fwd(SMALL[idx], algo, cuda_device)


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_fwd_with_conv_state_in(cuda_device, algo, io):
    wl = WORKLOADS["hawk_block"].with_shape(B=2, T=70, D=256, H=4, io=io, h0_var=0.3, seed=41)
    check_fwd(wl, algo, cuda_device, with_csi=True)


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("T", [2, 70])
def test_fwd_with_conv_state_in_wide_heads(cuda_device, algo, T):
    """conv_state_in / conv_state_out with 256-wide heads, where a unit's
    Conv1D covers the head's 256 channels and writes its own 128 to the state."""
    wl = WORKLOADS["hawk_block"].with_shape(B=2, T=T, D=512, H=2, h0_var=0.3, seed=45)
    check_fwd(wl, algo, cuda_device, with_csi=True, csi_seed=12)


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_fwd_split_composition(cuda_device, algo, io):
    """fwd over T equals fwd over T1 then fwd over T - T1 from (h_T1, conv_state_T1)."""
    wl = WORKLOADS["hawk_block"].with_shape(B=2, T=96, D=256, H=4, io=io, h0_var=0.3, seed=42)
    need_algo(wl, algo)
    tol = 1e-5 if io == "f32" else 1e-2
    t = to_dev(generate(wl), cuda_device)
    w = [t[k] for k in ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")]
    y, hT, cs = rg.rglru_fwd(t["x"], *w, h0=t["h0"], algo=algo)
    y1, h1, c1 = rg.rglru_fwd(t["x"][:, :40].contiguous(), *w, h0=t["h0"], algo=algo)
    y2, h2, c2 = rg.rglru_fwd(t["x"][:, 40:].contiguous(), *w, h0=h1, conv_state_in=c1, algo=algo)
    torch.cuda.synchronize()
    torch.testing.assert_close(torch.cat([y1, y2], 1).float(), y.float(), rtol=tol, atol=tol)
    torch.testing.assert_close(h2, hT, rtol=tol, atol=tol)
    assert torch.equal(c2, cs)


def decode_run(wl, rows, dev, algo, steps):
    if rg.decode_launches(wl.B, wl.D, wl.H, wl.dtype, algo) == 0:
        pytest.skip(f"{algo} does not cover {wl}")
    t = generate(wl)
    g = to_dev(t, dev)
    w_dev = [g[k] for k in ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")]
    h = g["h"].clone()
    ring = g["conv_state"].clone()
    ys = []
    for s in range(steps):
        y_t = torch.full_like(g["x_steps"][s], float("nan"))    # must be fully written
        rg.rglru_decode_step(g["x_steps"][s], ring, s, h, *w_dev, algo=algo, y_t=y_t)
        assert bool(torch.isfinite(y_t.float()).all())
        ys.append(y_t[rows])
    torch.cuda.synchronize()
    # oracle on the sampled rows only (rows never interact)
    w = {k: t[k] for k in ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")}
    ho, ringo = orc.as_f64(t["h"][rows]), orc.as_f64(t["conv_state"][rows])
    yo = []
    for s in range(steps):
        y_t, ho, ringo = orc.rglru_decode_step(t["x_steps"][s][rows], ringo, s, ho, **w)
        yo.append(y_t)
    yo = np.stack(yo)
    yg = torch.stack(ys).float().cpu().numpy()
    e_y = max_rel_err(yg, yo, time_axis=0)
    e_h = max_rel_err(h[rows].cpu().numpy(), ho, scale=channel_rms(yo, 0)[0])
    assert np.array_equal(ring[rows].float().cpu().numpy(), ringo)
    return e_y, e_h


@pytest.mark.parametrize("algo", DEC_ALGOS)
# (2560, 512, 2): 256-wide heads, 2 heads x 160 row tiles = 320 (head, tile) pairs over the
# CTAs, so that CTA ranges hold several pairs and some cross the head boundary
@pytest.mark.parametrize("shape", [(70, 256, 4), (33, 256, 2), (45, 512, 2), (1, 128, 1),
                                   (2560, 512, 2)])
def test_decode_shapes_bf16(cuda_device, algo, shape):
    B, D, H = shape
    wl = WORKLOADS["decode_batch"].with_shape(B=B, D=D, H=H, decode_steps=5, bias_std=0.3,
                                              seed=53 + B)
    e_y, e_h = decode_run(wl, torch.arange(B), cuda_device, algo, 5)
    assert e_y <= TOL["bf16"] and e_h <= TOL["bf16"], (e_y, e_h)


@pytest.mark.parametrize("algo", DEC_ALGOS)
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_decode_small(cuda_device, algo, io):
    wl = WORKLOADS["decode_batch"].with_shape(B=37, D=256, H=4, io=io, decode_steps=7,
                                              bias_std=0.3, seed=51)
    rows = torch.arange(37)
    e_y, e_h = decode_run(wl, rows, cuda_device, algo, 7)
    assert e_y <= TOL[io] and e_h <= TOL[io], (e_y, e_h)


@pytest.mark.parametrize("algo", DEC_ALGOS)
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_decode_composes_with_fwd(cuda_device, algo, io):
    """fwd over T1 tokens then decode steps from its (h_T, conv_state_out) equals fwd over T."""
    wl = WORKLOADS["hawk_block"].with_shape(B=3, T=20, D=256, H=2, io=io, h0_var=0.5, seed=52)
    if rg.decode_launches(wl.B, wl.D, wl.H, wl.dtype, algo) == 0:
        pytest.skip(f"{algo} does not cover {wl}")
    tol = 2e-5 if io == "f32" else 2e-2
    t = to_dev(generate(wl), cuda_device)
    w = [t[k] for k in ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")]
    y, hT, _ = rg.rglru_fwd(t["x"], *w, h0=t["h0"], algo=algo)
    T1 = 13
    _, h, ring = rg.rglru_fwd(t["x"][:, :T1].contiguous(), *w, h0=t["h0"], algo=algo)
    for k, s in enumerate(range(T1, 20)):
        y_t = rg.rglru_decode_step(t["x"][:, s].contiguous(), ring, k, h, *w, algo=algo)
        torch.testing.assert_close(y_t.float(), y[:, s].float(), rtol=tol, atol=tol)
    torch.testing.assert_close(h, hT, rtol=tol, atol=tol)


# ------------------------------------------------ full-size workloads ----

def full_fwd_sampled(name, dev, algo, sample):
    wl = WORKLOADS[name]
    need_algo(wl, algo)
    t = generate(wl)
    g = to_dev(t, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    y = torch.full_like(g["x"], float("nan"))       # every element must be written
    hT = torch.full((wl.B, wl.D), float("nan"), device=dev)
    y, hT, cs = rg.rglru_fwd(g["x"], g["conv_w"], g["W_a"], g["b_a"], g["W_x"], g["b_x"],
                             g["Lambda"], h0=g["h0"], algo=algo, dev_status=status, y=y, h_T=hT)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.isfinite(y.float()).all() and torch.isfinite(hT).all()
    errs = []
    for kind, idx in sample:
        if kind == "rows":
            sl = (idx, slice(None), slice(None))
            ts = {k: (v[idx] if k in ("x", "h0") and v is not None else v) for k, v in t.items()}
            yg, hg = y[idx].float().cpu().numpy(), hT[idx].cpu().numpy()
            csg = cs[idx].float().cpu().numpy()
        else:  # whole heads: channels [h*bw, (h+1)*bw)
            bw = wl.bw
            ch = torch.cat([torch.arange(h * bw, (h + 1) * bw) for h in idx])
            ts = dict(t)
            ts["x"] = t["x"][:, :, ch]
            ts["conv_w"] = t["conv_w"][:, ch]
            ts["W_a"], ts["W_x"] = t["W_a"][idx], t["W_x"][idx]
            for k in ("b_a", "b_x", "Lambda"):
                ts[k] = t[k][ch]
            ts["h0"] = t["h0"][:, ch] if t["h0"] is not None else None
            yg = y[:, :, ch.to(dev)].float().cpu().numpy()
            hg = hT[:, ch.to(dev)].cpu().numpy()
            csg = cs[:, :, ch.to(dev)].float().cpu().numpy()
        yo, hTo, cso = orc.rglru_fwd(ts["x"], ts["conv_w"], ts["W_a"], ts["b_a"], ts["W_x"],
                                     ts["b_x"], ts["Lambda"], h0=ts["h0"])
        errs.append((max_rel_err(yg, yo), max_rel_err(hg, hTo, scale=channel_rms(yo, 1)[:, 0, :])))
        assert np.array_equal(csg, cso)
    tol = TOL[wl.io]
    assert all(e <= tol for pair in errs for e in pair), errs
    return errs


@pytest.mark.parametrize("algo", ALGOS)
def test_full_hawk_block(cuda_device, algo):
    full_fwd_sampled("hawk_block", cuda_device, algo, [("rows", torch.arange(8))])


@pytest.mark.parametrize("algo", ALGOS)
def test_full_griffin2b_sampled_rows(cuda_device, algo):
    full_fwd_sampled("griffin2b", cuda_device, algo, [("rows", torch.tensor([0, 15]))])


@pytest.mark.parametrize("algo", ALGOS)
def test_full_long_context_sampled_heads(cuda_device, algo):
    full_fwd_sampled("long_context", cuda_device, algo, [("heads", [0, 15])])


@pytest.mark.parametrize("algo", DEC_ALGOS)
def test_full_decode_batch_sampled_rows(cuda_device, algo):
    rows = torch.tensor([0, 1, 511, 1023])
    e_y, e_h = decode_run(WORKLOADS["decode_batch"], rows, cuda_device, algo, 256)
    assert e_y <= TOL["bf16"] and e_h <= TOL["bf16"], (e_y, e_h)
