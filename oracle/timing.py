"""Times the float64 oracle on the host's cores (bench infrastructure only).

TEST INFRASTRUCTURE ONLY: bench.py's CPU-baseline leg and its reference arm
call this; nothing on the product path does. It adds no arithmetic of its
own: it runs oracle.rglru_oracle.rglru_fwd, unchanged, on independent pieces
of a workload in worker processes.

Batch rows never interact in the layer, and neither do heads (the gates are
block-diagonal per head, the Conv1D and the scan are per channel), so one
(batch row, head) block over the first Tp tokens is a complete problem of its
own. Blocks go to a pool of worker processes ("spawn": the parent may already
hold a CUDA context), one per host core, each with single-threaded numpy.
"""
from __future__ import annotations

import math
import os
import time

import numpy as np

_THREAD_VARS = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")


def _run_block(args):
    from oracle import rglru_oracle as orc
    t0 = time.perf_counter()
    orc.rglru_fwd(*args[:7], h0=args[7])
    return time.perf_counter() - t0


def _f64(t):
    return None if t is None else t.detach().to("cpu").double().numpy()


def head_blocks(t: dict, wl, rows: int, Tp: int, reps: int = 1) -> list:
    """Argument tuples of rglru_fwd for the (row, head) blocks of the first `rows`
    batch rows and `Tp` tokens, repeated `reps` times."""
    bw = wl.bw
    x = _f64(t["x"][:rows, :Tp])
    cw, Wa, Wx = _f64(t["conv_w"]), _f64(t["W_a"]), _f64(t["W_x"])
    ba, bx, lam = _f64(t["b_a"]), _f64(t["b_x"]), _f64(t["Lambda"])
    h0 = _f64(t["h0"][:rows]) if t.get("h0") is not None else None
    out = []
    for _ in range(reps):
        for r in range(rows):
            for h in range(wl.H):
                c = slice(h * bw, (h + 1) * bw)
                out.append((x[r:r + 1, :, c].copy(), cw[:, c].copy(), Wa[h:h + 1].copy(),
                            ba[c].copy(), Wx[h:h + 1].copy(), bx[c].copy(), lam[c].copy(),
                            None if h0 is None else h0[r:r + 1, c].copy()))
    return out


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def measure(t: dict, wl, seconds: float, procs: int | None = None) -> dict:
    """Channel-tokens/s of the oracle on `procs` worker processes (default: every
    host core), over a sample grown until one round takes about `seconds`."""
    import multiprocessing as mp
    procs = procs or host_cores()
    saved = {k: os.environ.get(k) for k in _THREAD_VARS}
    for k in _THREAD_VARS:
        os.environ[k] = "1"
    try:
        pool = mp.get_context("spawn").Pool(procs)
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    try:
        pool.map(_run_block, head_blocks(t, wl, 1, min(wl.T, 16), 1)[:procs])   # warm the workers
        rows, Tp, reps = 1, min(wl.T, 256), 1
        while True:
            blocks = head_blocks(t, wl, rows, Tp, reps)
            t0 = time.perf_counter()
            per = pool.map(_run_block, blocks, chunksize=1)
            wall = time.perf_counter() - t0
            if wall >= 0.7 * seconds or (rows == wl.B and Tp == wl.T and reps >= 64):
                break
            grow = max(2, int(math.ceil(seconds / max(wall, 1e-3))))
            if Tp < wl.T:
                Tp = min(wl.T, Tp * grow)
            elif rows < wl.B:
                rows = min(wl.B, rows * grow)
            else:
                reps *= grow
    finally:
        pool.close()
        pool.join()
    work = len(blocks) * Tp * wl.bw
    one_core = Tp * wl.bw / float(np.mean(per))
    return {"value": work / wall, "unit": "channel-tokens/s", "cores": procs, "kind": "oracle",
            "single_core_value": one_core,
            "sample": (f"{reps} x {rows} of {wl.B} batch rows x the first {Tp} of {wl.T} tokens "
                       f"x {wl.H} heads = {len(blocks)} independent (row, head) blocks of "
                       f"{wl.bw} channels, float64 numpy oracle, {procs} worker processes "
                       f"(one per host core), {wall:.1f} s wall")}
