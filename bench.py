"""Benchmark of the RG-LRU layer on B200: channel-tokens/s and achieved HBM GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--algo auto]
    python bench.py --impl reference ...      # the float64 CPU oracle on a bounded sample

A step is one rglru_fwd over the whole workload (Conv1D, gates, decay, scan
and the time-split carry), inputs resident in HBM. The headline workload is
long_context (B=1, T=131072, D=4096, H=16, bf16: the largest configuration);
the other forward workloads (hawk_block, griffin2b) are timed the same way as
`legs`, and decode_batch, the backward and the recurrent block (both on
hawk_block) as their own keys. The timed region is K
back-to-back steps between CUDA events on the launching stream, after W
untimed warm-up steps; each step reads and writes its own buffer set, and the
sets rotate so that the bytes touched between two uses of one set exceed 3x
the 126 MB L2 (no step finds its inputs in L2). Under torchrun every rank
runs the same workload on its own GPU (weak scaling over independent
batches, no collective on the data path); the time is the max over ranks.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_linear_recurrence_rglru_b200.workloads import WORKLOADS, generate  # noqa: E402

L2_BYTES = 126 * 2**20
METRIC = "RG-LRU channel-tokens/s and achieved HBM GB/s vs B200 peak (1 GPU)"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# --------------------------------------------------------------- clocks ----

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu_index = gpu_index
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "power_w_max": max(power) if power else None, "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------- our arm ----

def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, ws: int, device="cuda") -> float:
    """The max of v over all ranks (the job's time is its slowest rank's)."""
    if ws == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: int, steps: int, ms_max: float, ws: int) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return ws * units_per_rank * steps / (ms_max / 1e3)


# DRAM traffic of the forward kernel per launch, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), stored with a hash of the
# kernel sources it was taken on: a number taken on other sources is not reported
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")
KERNEL_SOURCES = ["fwd_tc.cu", "tc_gates.cuh", "tc_primitives.cuh", "common.cuh"]


def _code_only(src: str) -> str:
    """C++ source without comments and blank space (comment edits keep the hash)."""
    import re
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def kernel_source_hash(texts=None) -> str:
    """Hash of the code (comments and spacing removed) of the forward kernel's sources."""
    import hashlib
    h = hashlib.sha256()
    for fn in KERNEL_SOURCES:
        if texts is not None:
            src = texts[fn]
        else:
            with open(os.path.join(ROOT, "gated_linear_recurrence_rglru_b200", "csrc", fn)) as f:
                src = f.read()
        h.update(_code_only(src).encode())
    return h.hexdigest()[:16]


def kernel_traffic(wl, algo):
    """(kernel name, DRAM bytes per launch or None) of the workload's forward kernel."""
    import gated_linear_recurrence_rglru_b200 as rg
    if not (algo in ("auto", "tensor") and rg.fwd_launches(wl.B, wl.T, wl.D, wl.H, wl.dtype, "tensor") > 0):
        return "generic kernels (segment pass, carry, final pass)", None
    name = "fwd_tc_kernel"
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return name, None
    ent = rec.get("workloads", {}).get(wl.name)
    if ent is None or rec.get("source_hash") != kernel_source_hash():
        return name, None
    return name, ent["dram_bytes_per_launch"]


def fwd_bytes_per_chtok(wl) -> int:
    """Algorithmic HBM bytes per channel-token of the fused forward: read x, write y."""
    return 2 * (4 if wl.io == "f32" else 2)


def config_of(wl, ws, algo):
    """The config dict of a forward workload (the same for both arms of the bench)."""
    esz = 4 if wl.io == "f32" else 2
    set_bytes = 2 * wl.B * wl.T * wl.D * esz
    nsets = n_buffer_sets(set_bytes)
    return {"workload": f"{wl.name} B={wl.B} T={wl.T} D={wl.D} H={wl.H} bw={wl.bw} io={wl.io}",
            "algo": algo, "global_batch": wl.B * ws, "seq_len": wl.T,
            "parallelism": f"dp{ws} (independent batches)",
            "l2": f"{nsets} rotating buffer sets of {set_bytes / 1e6:.1f} MB "
                  f"(>3x L2 between reuses)"}


def n_buffer_sets(set_bytes):
    """Buffer sets rotated so that >3x L2 is touched between two uses of one set."""
    return max(2, math.ceil(3 * L2_BYTES / set_bytes) + 1)


def time_forward(rg, wl, dev, steps, warmup, algo, pk, soak_s=0.0, ws=1):
    """Time rglru_fwd on a workload: `steps` back-to-back steps between CUDA events
    on the launching stream after `warmup` untimed ones, then the same steps again
    with the kernel events that the library records around its compute kernel.
    Returns the leg's figures (times are this rank's)."""
    t = generate(wl)
    g = {k: (v.to(dev) if v is not None else None) for k, v in t.items()}
    w = [g[k] for k in ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")]
    B, T, D, H = wl.B, wl.T, wl.D, wl.H
    esz = 4 if wl.io == "f32" else 2
    nsets = n_buffer_sets(2 * B * T * D * esz)
    xs = [g["x"]] + [g["x"].clone() for _ in range(nsets - 1)]
    ys = [torch.empty_like(g["x"]) for _ in range(nsets)]
    hT = [torch.empty(B, D, device=dev) for _ in range(nsets)]
    cs = [torch.empty(B, 3, D, device=dev, dtype=wl.dtype) for _ in range(nsets)]
    wsb = rg.fwd_workspace_bytes(B, T, D, H, wl.dtype)
    work = [torch.empty(max(wsb, 1), device=dev, dtype=torch.uint8) for _ in range(nsets)]
    status = torch.zeros(1, device=dev, dtype=torch.int32)
    stream = torch.cuda.current_stream()
    # per timed step, a pair of events that the library records right around its
    # compute kernel(s) on this stream: the kernel's own launch duration
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for eb, ee in kev:
        eb.record(stream)
        ee.record(stream)
    torch.cuda.synchronize()
    kopts = [rg.FwdOptions(kernel_begin_event=eb.cuda_event, kernel_end_event=ee.cuda_event)
             for eb, ee in kev]

    def step(i, opts=None):
        k = i % nsets
        rg.rglru_fwd(xs[k], *w, h0=g["h0"], y=ys[k], h_T=hT[k], conv_state_out=cs[k],
                     workspace=work[k], dev_status=status, algo=algo, options=opts)

    i = 0
    soak_t0 = time.time()
    while time.time() - soak_t0 < soak_s:         # untimed load around the timed region
        for _ in range(20):
            step(i)
            i += 1
        torch.cuda.synchronize()
    for _ in range(warmup):
        step(i)
        i += 1
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step(i)
        i += 1
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    ms_local = e0.elapsed_time(e1)
    for j in range(steps):
        step(i, kopts[j])
        i += 1
    torch.cuda.synchronize()
    kernel_ms = sum(eb.elapsed_time(ee) for eb, ee in kev) / steps
    post_t0 = time.time()
    while time.time() - post_t0 < soak_s:
        for _ in range(20):
            step(i)
            i += 1
        torch.cuda.synchronize()
    word = int(status.item())
    if word != 0:
        raise SystemExit(f"device status word {word:#x}: {rg.status_str(word & 0xFF)} "
                         f"(wait site {(word >> 8) & 0xFF}, block {word >> 16})")
    chtok = B * T * D
    bytes_step = fwd_bytes_per_chtok(wl) * chtok
    kname, traffic = kernel_traffic(wl, algo)
    ms_step = ms_local / steps
    achieved = bytes_step / (kernel_ms / 1e3) / 1e9
    achieved_step = bytes_step / (ms_step / 1e3) / 1e9
    leg = {"workload": config_of(wl, ws, algo)["workload"], "steps": steps,
           "ms_per_step": ms_step, "value": chtok / (ms_step / 1e3), "unit": "channel-tokens/s",
           "hbm_gbs": achieved_step,
           "gpu_launches_per_step": rg.fwd_launches(B, T, D, H, wl.dtype, algo),
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"],
                        "unit": "GB/s", "frac": achieved / pk["hbm_gbs"], "traffic": traffic,
                        "kernel": kname, "kernel_ms": kernel_ms,
                        "timing": "CUDA events recorded by the library around the kernel on "
                                  "the launching stream, every step of a second pass of the "
                                  "same K steps right after the timed one",
                        "step_achieved": achieved_step, "peak_source": pk["source"],
                        "algorithmic_bytes_per_launch": bytes_step}}
    leg["_ms_total"] = ms_local
    leg["_inputs"] = (t, g, w)
    return leg


FWD_LEGS = ("hawk_block", "griffin2b", "long_context")


def run_ours(a, ws, rank, local):
    import gated_linear_recurrence_rglru_b200 as rg

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = WORKLOADS[a.workload]
    if wl.decode_steps:
        raise SystemExit("--workload must be a forward workload; decode is reported as 'decode'")
    pk = peaks()
    sampler = ClockSampler(local)
    head = time_forward(rg, wl, dev, a.steps, a.warmup, a.algo, pk, soak_s=a.soak_s, ws=ws)
    clocks = sampler.stop()
    ms = max_over_ranks(head.pop("_ms_total"), ws)
    t, g, w = head.pop("_inputs")
    ms_step = ms / a.steps
    chtok = wl.B * wl.T * wl.D
    value = weak_scaling_value(chtok, a.steps, ms, ws)
    out = {
        "metric": METRIC, "value": value, "unit": "channel-tokens/s", "n_gpus": ws,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.io, "data": "synthetic (seeded; recipe of the workload)",
        "config": config_of(wl, ws, a.algo),
        "hbm_gbs": fwd_bytes_per_chtok(wl) * chtok / (ms_step / 1e3) / 1e9,
        "roofline": head["roofline"],
        "gpu_launches": head["gpu_launches_per_step"] * a.steps,
        "clocks": clocks,
    }
    if a.legs:
        # the other forward workloads, each timed and measured the same way (this rank)
        legs = {}
        for name in FWD_LEGS:
            if name == wl.name:
                continue
            leg = time_forward(rg, WORKLOADS[name], dev, min(a.steps, 100), a.warmup, a.algo,
                               pk, ws=ws)
            leg.pop("_ms_total")
            leg.pop("_inputs")
            legs[name] = leg
        out["legs"] = legs
    if a.e2e:
        out["e2e"] = run_e2e(rg, wl, g, w, dev, a)
    if a.cpu_baseline and ws == 1 and rank == 0:
        out["cpu_baseline"] = cpu_baseline(wl, a.cpu_seconds, t)
    del t, g, w
    torch.cuda.empty_cache()
    if a.decode:
        out["decode"] = run_decode(rg, dev, a, pk)
    if a.backward:
        out["backward"] = run_backward(rg, WORKLOADS["hawk_block"], dev, a, pk)
    if a.block:
        out["block"] = run_block(rg, WORKLOADS["hawk_block"], dev, a, pk)
    return out


def run_e2e(rg, wl, g, w, dev, a):
    """Same metric through the public API with host buffers: every step copies its
    input x from pinned host memory to the device, runs the forward and copies y
    back to pinned host memory, all inside the timed region. Steps are pipelined
    the way a serving loop runs them: three buffer sets and three streams, so that
    the copy-in of step i+1 and the copy-out of step i-1 overlap the forward of
    step i (every copy still belongs to exactly one step)."""
    B, T, D, H = wl.B, wl.T, wl.D, wl.H
    nbuf = 3 if g["x"].numel() * g["x"].element_size() < 2**29 else 2
    x_host = [g["x"].cpu().pin_memory() for _ in range(nbuf)]
    y_host = [torch.empty_like(x_host[0]).pin_memory() for _ in range(nbuf)]
    x_dev = [torch.empty_like(g["x"]) for _ in range(nbuf)]
    y_dev = [torch.empty_like(g["x"]) for _ in range(nbuf)]
    wsb = rg.fwd_workspace_bytes(B, T, D, H, wl.dtype)
    work = [torch.empty(max(wsb, 1), device=dev, dtype=torch.uint8) for _ in range(nbuf)]
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_done = [ev() for _ in range(nbuf)]
    comp_done = [ev() for _ in range(nbuf)]
    out_done = [ev() for _ in range(nbuf)]
    used = [False] * nbuf

    def step(i):
        k = i % nbuf
        with torch.cuda.stream(s_in):
            if used[k]:
                s_in.wait_event(comp_done[k])          # x_dev[k] read by step i - nbuf
            x_dev[k].copy_(x_host[k], non_blocking=True)
            in_done[k].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(in_done[k])
            if used[k]:
                s_comp.wait_event(out_done[k])         # y_dev[k] read back by step i - nbuf
            rg.rglru_fwd(x_dev[k], *w, h0=g["h0"], y=y_dev[k], workspace=work[k],
                         algo=a.algo, want_state=False, stream=s_comp)
            comp_done[k].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[k])
            y_host[k].copy_(y_dev[k], non_blocking=True)
            out_done[k].record(s_out)
        used[k] = True

    for i in range(nbuf):
        step(i)
    torch.cuda.synchronize()
    n = max(6, min(a.steps, 30 if nbuf == 3 else 10))
    main = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    for s_ in (s_in, s_comp, s_out):
        s_.wait_event(e0)
    for i in range(n):
        step(i)
    main.wait_stream(s_out)
    e1.record(main)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    esz = x_host[0].element_size()
    return {"value": B * T * D / (ms / 1e3), "unit": "channel-tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": B * T * D * esz, "d2h_bytes_per_step": B * T * D * esz,
            "steps": n, "pipelining": f"{nbuf} buffer sets, copy-in / forward / copy-out streams"}


def run_backward(rg, wl, dev, a, pk):
    """Backward of a workload: gradients of <dy, y> + <dh_T, h_T> for every
    input, one rglru_bwd per step, inputs resident, rotating dy / dx sets."""
    B, T, D, H = wl.B, wl.T, wl.D, wl.H
    t = generate(wl)
    g = {k: (v.to(dev) if v is not None else None) for k, v in t.items()}
    w = [g[k] for k in ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")]
    esz = 4 if wl.io == "f32" else 2
    gen = torch.Generator(device=dev)
    gen.manual_seed(wl.seed + 1000)
    nsets = 3
    dys = [torch.randn(B, T, D, generator=gen, device=dev).to(wl.dtype) for _ in range(nsets)]
    dh_T = torch.randn(B, D, generator=gen, device=dev)
    ws = torch.empty(rg.bwd_workspace_bytes(B, T, D, H, wl.dtype), device=dev, dtype=torch.uint8)
    outs = [None] * nsets

    def step(i):
        k = i % nsets
        outs[k] = rg.rglru_bwd(g["x"], *w, dys[k], h0=g["h0"], dh_T=dh_T, workspace=ws,
                               out=outs[k])

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    steps = max(5, min(a.steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        step(i)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    bytes_step = 3 * esz * B * T * D    # read x and dy, write dx
    gbs = bytes_step / (ms / 1e3) / 1e9
    return {"workload": f"{wl.name} backward B={B} T={T} D={D} H={H} io={wl.io}",
            "value": B * T * D / (ms / 1e3), "unit": "channel-tokens/s", "ms_per_step": ms,
            "steps": steps, "gpu_launches_per_step": rg.bwd_launches(B, T, D, H, wl.dtype),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": None,
                         "algorithmic_bytes_per_launch": bytes_step,
                         "note": "step time of all five launches; the three gate "
                                 "contractions (2 bw MACs per channel-token each) on the "
                                 "tensor cores (bf16 operands, fp32 accumulate) for bf16 I/O "
                                 "with 64/128-wide heads, the rest fp32 on CUDA cores; "
                                 "the intermediates in a workspace (the gates r, i and d u in "
                                 "fp32, u, d z_a, d z_x in bf16: 18 B per channel-token "
                                 "written and re-read) are not algorithmic"}}


def run_block(rg, wl, dev, a, pk):
    """The recurrent block around the layer on the same workload (Dm = D): input and
    gate projections, the layer, GeLU gating and the output projection, one
    rglru_block_fwd per step, inputs resident, three rotating x / out sets."""
    from gated_linear_recurrence_rglru_b200.workloads import generate_block
    B, T, D, H = wl.B, wl.T, wl.D, wl.H
    Dm = D
    t = generate_block(wl, Dm)
    gd = {k: (v.to(dev) if v is not None else None) for k, v in t.items()}
    wts = [gd[k] for k in ("W_in", "W_gate", "W_out", "conv_w", "W_a", "b_a", "W_x", "b_x",
                           "Lambda")]
    nsets = 3
    xs = [gd["x"]] + [torch.randn_like(gd["x"], dtype=torch.float32).to(wl.dtype)
                      for _ in range(nsets - 1)]
    outs = [torch.empty_like(gd["x"]) for _ in range(nsets)]
    ws = torch.empty(rg.block_fwd_workspace_bytes(B, T, Dm, D, H, wl.dtype), device=dev,
                     dtype=torch.uint8)

    def step(i):
        k = i % nsets
        rg.rglru_block_fwd(xs[k], *wts, h0=gd["h0"], out=outs[k], workspace=ws,
                           want_state=False)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    steps = max(5, min(a.steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        step(i)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    flops = 3 * 2 * B * T * Dm * D
    tfs = flops / (ms / 1e3) / 1e12
    return {"workload": f"{wl.name} recurrent block B={B} T={T} Dm={Dm} D={D} H={H} io={wl.io}",
            "value": B * T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
            "roofline": {"bound": "tensor", "achieved": tfs, "peak": pk["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": tfs / pk["bf16_tflops"], "traffic": None,
                         "algorithmic_flops_per_step": flops,
                         "note": "three dense projections (the library's tcgen05 GEMM, bf16 "
                                 "operands, fp32 accumulation in TMEM; the GeLU gating fused "
                                 "into the gate projection's epilogue) over the step time, "
                                 "which also holds the layer (about 42 us)"}}


def run_decode(rg, dev, a, pk):
    """Decode workload: B=1024 sequences, one step per launch, state in place. The
    inputs are the workload's own seeded draws (the ones the parity tests check)."""
    wl = WORKLOADS["decode_batch"]
    steps = a.decode_steps
    t = generate(wl.with_shape(decode_steps=max(steps, 1)))
    B, D, H, bw = wl.B, wl.D, wl.H, wl.bw
    x = t["x_steps"].to(dev)
    conv_w, W_a, b_a, W_x, b_x, Lam = (t[k].to(dev) for k in ("conv_w", "W_a", "b_a", "W_x",
                                                               "b_x", "Lambda"))
    h = t["h"].to(dev)
    ring = t["conv_state"].to(dev)
    del t
    ys = torch.empty(steps, B, D, device=dev, dtype=wl.dtype)
    stream = torch.cuda.current_stream()

    def one(s_):
        rg.rglru_decode_step(x[s_], ring, s_, h, conv_w, W_a, b_a, W_x, b_x, Lam, y_t=ys[s_],
                             algo=a.algo)

    for s_ in range(3):
        one(s_)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s_ in range(steps):
        one(s_)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_eager = e0.elapsed_time(e1) / steps
    # the same steps captured once in a CUDA graph (the launches of all steps are
    # recorded with their own x_t, pos and y_t) and replayed: per step without
    # host launch gaps
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        with torch.cuda.graph(graph, stream=cap):
            for s_ in range(steps):
                one(s_)
    stream.wait_stream(cap)
    graph.replay()
    torch.cuda.synchronize()
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    del graph
    bytes_step = 20 * B * D   # x 2 + ring read 6 + ring write 2 + h read/write 8 + y 2
    gbs = bytes_step / (ms / 1e3) / 1e9
    return {"workload": f"decode_batch B={B} D={D} H={H} bw={bw} io=bf16, {steps} steps",
            "value": B * D / (ms / 1e3), "unit": "channel-tokens/s", "us_per_step": ms * 1e3,
            "timing": f"{steps} steps captured in one CUDA graph, replayed; CUDA events",
            "us_per_step_eager": ms_eager * 1e3,
            "gpu_launches_per_step": rg.decode_launches(B, D, H, wl.dtype, a.algo),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": None,
                         "algorithmic_bytes_per_launch": bytes_step},
            "inputs": "the decode_batch workload's seeded draws (workloads.generate)",
            "l2": "state, ring and weights total 113 MB; the state is re-read each step "
                  "(L2 may hold part of it, as in real decoding)"}


# ------------------------------------------------------------ CPU oracle --

def cpu_baseline(wl, seconds, t=None):
    """The float64 oracle, as it stands, on every host core over a bounded sample of
    the workload (independent (batch row, head) blocks; see oracle/timing.py)."""
    from oracle import timing
    return timing.measure(t if t is not None else generate(wl), wl, seconds)


# -------------------------------------------------------- reference arm --

def run_reference(a, ws, rank):
    """The reference arm: the float64 oracle on the host's cores, the same metric
    and config as our arm; nothing here loads the CUDA library."""
    if rank != 0:
        return None
    wl = WORKLOADS[a.workload]
    t = generate(wl)
    from oracle import timing
    for _ in range(a.warmup):
        timing.measure(t, wl, 0.3)
    per = [timing.measure(t, wl, a.ref_seconds) for _ in range(a.steps)]
    v = statistics.median(p["value"] for p in per)
    base = dict(per[-1])
    base["value"] = v
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "channel-tokens/s",
            "n_gpus": ws, "steps": a.steps, "warmup": a.warmup, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded; recipe of the workload)",
            "config": config_of(wl, ws, a.algo),
            "cpu_baseline": base,
            "e2e": {"value": v, "unit": "channel-tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long_context", choices=sorted(WORKLOADS))
    ap.add_argument("--algo", default="auto", choices=["auto", "generic", "tensor"])
    ap.add_argument("--soak-s", type=float, default=1.5,
                    help="untimed seconds of the same steps before and after the timed "
                         "region, so the clock sampler sees the load")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--no-legs", dest="legs", action="store_false",
                    help="skip the other forward workloads (hawk_block, griffin2b, ...)")
    ap.add_argument("--no-decode", dest="decode", action="store_false")
    ap.add_argument("--no-backward", dest="backward", action="store_false")
    ap.add_argument("--no-block", dest="block", action="store_false")
    ap.add_argument("--decode-steps", type=int, default=256)
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-seconds", type=float, default=4.0)
    a = ap.parse_args(argv)
    if a.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if a.impl == "reference":
        out = run_reference(a, ws, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return 0
    ws, rank, local = dist_setup()
    out = run_ours(a, ws, rank, local)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
