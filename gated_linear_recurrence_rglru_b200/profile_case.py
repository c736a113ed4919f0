"""Run a few calls of one workload through the library, for profiler captures.

    python -m gated_linear_recurrence_rglru_b200.profile_case long_context:16384 3
    python -m gated_linear_recurrence_rglru_b200.profile_case decode_batch 4

A forward workload (optionally cut to T tokens with `name:T`) runs `calls`
forwards on rotating copies of x, so that consecutive launches do not find
their input in L2; `decode_batch` runs `calls` decode steps. The inputs are the
workload's seeded synthetic recipe. Exits non-zero if a call reports an error.
A profiler then selects launches by kernel name and index, e.g.
`ncu -k regex:fwd_tc -s 1 -c 1 ...`.
"""
from __future__ import annotations

import argparse
import sys

import torch

from . import _abi
from .workloads import WORKLOADS, generate

WEIGHTS = ("conv_w", "W_a", "b_a", "W_x", "b_x", "Lambda")


def _device_inputs(wl, dev):
    t = generate(wl)
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in t.items()}


def run_forward(wl, calls: int, dev) -> None:
    g = _device_inputs(wl, dev)
    w = [g[k] for k in WEIGHTS]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    xs = [g["x"]] + [g["x"].clone() for _ in range(2)]
    y = torch.empty_like(g["x"])
    for i in range(calls):
        _abi.rglru_fwd(xs[i % len(xs)], *w, h0=g["h0"], dev_status=status, y=y)
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise SystemExit(f"forward reported status word {int(status.item()):#x}")


def run_decode(wl, calls: int, dev) -> None:
    g = _device_inputs(wl.with_shape(decode_steps=calls), dev)
    w = [g[k] for k in WEIGHTS]
    h, ring = g["h"].clone(), g["conv_state"].clone()
    for s in range(calls):
        _abi.rglru_decode_step(g["x_steps"][s], ring, s, h, *w)
    torch.cuda.synchronize(dev)


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("case", help="workload name, optionally name:T for a forward cut to T tokens")
    ap.add_argument("calls", type=int, nargs="?", default=3)
    args = ap.parse_args(argv)
    name, _, T = args.case.partition(":")
    if name not in WORKLOADS:
        ap.error(f"unknown workload {name!r} (one of {', '.join(WORKLOADS)})")
    wl = WORKLOADS[name]
    if not torch.cuda.is_available():
        raise SystemExit("profile_case needs a CUDA device")
    dev = torch.device("cuda:0")
    if wl.decode_steps > 0:
        run_decode(wl, args.calls, dev)
    else:
        run_forward(wl.with_shape(T=int(T)) if T else wl, args.calls, dev)
    print("ok", args.case, args.calls)
    return 0


if __name__ == "__main__":
    sys.exit(main())
