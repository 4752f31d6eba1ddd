"""Pipeline timeline of one attention CTA, from a tuning build.

A build with ``INFINI_NVCC_FLAGS=-DINFINI_ATTN_TRACE=<cta>`` makes ``attn_tc_kernel``
record ``%clock64`` at its pipeline events for CTA ``<cta>`` into a device array
(``infini_attn_debug_trace`` copies it out).  This script runs a few forwards of a
workload and prints, for each work item that CTA processed, when its roles reached
each event, plus the per-key-tile steady state of the CTA's first item.  Times are SM
cycles relative to the CTA's start.

    INFINI_NVCC_FLAGS=-DINFINI_ATTN_TRACE=5 python -m compressive_memory_transformer_sm_b200.build --force
    python -m compressive_memory_transformer_sm_b200.trace --workload 1b_layer --mode linear

Slot layout (see ``ATTN_TRACE`` in ``csrc/sm100_attn.cuh``): softmax warpgroup k, item it
at ``1024 k + 16 it + e``; its first item's key tile j at ``1024 k + 512 + 8 j + e``; the
MMA warp at ``2048 + 16 it + e``; the TMA thread at ``3072 + 16 it + e``; start at 4000.
"""
from __future__ import annotations

import argparse
import ctypes

import numpy as np
import torch

from . import api, workloads as W
from . import LINEAR, DELTA


def read_trace() -> np.ndarray:
    fn = getattr(api.lib, "infini_attn_debug_trace", None)
    if fn is None:
        raise SystemExit("the library was built without a trace: rebuild it with INFINI_NVCC_FLAGS=-DINFINI_ATTN_TRACE=<cta>")
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int]
    buf = (ctypes.c_ulonglong * 4096)()
    if fn(buf, 4096) != 0:
        raise SystemExit("infini_attn_debug_trace failed")
    return np.array(buf, dtype=np.int64)


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", default="1b_layer", choices=sorted(W.WORKLOADS))
    ap.add_argument("--mode", default="linear", choices=("linear", "delta"))
    ap.add_argument("--runs", type=int, default=3)
    args = ap.parse_args()
    w = W.WORKLOADS[args.workload]
    if w.streaming:
        raise SystemExit("streaming workloads: trace one segment_step through the Python API instead")
    mode = LINEAR if args.mode == "linear" else DELTA
    q, k, v, beta = W.make_inputs(w, device="cuda")
    M, z = W.empty_state(w, device="cuda")
    out = torch.empty_like(v)
    for _ in range(args.runs):
        M.zero_()
        z.zero_()
        api.infini_attn_forward(q, k, v, beta, M, z, out, w.N, mode)
    torch.cuda.synchronize()
    t = read_trace()
    t0 = t[4000]

    def rel(x):
        return int(x - t0) if x > t0 else None  # None: not reached in the last forward

    print(f"{w.name} {args.mode}: setup done at {rel(t[4001])}")
    names = dict(take=0, S0=1, lastP=2, sq_start=9, sq_math=10, SQ=3, MEM=4, OF=5)
    for it in range(64):
        p = 3072 + 16 * it
        if rel(t[p]) is None:
            break
        m = 2048 + 16 * it
        print(f"item {it} (index {t[p + 8]}): TMA claim {rel(t[p])}, Q issued {rel(t[p + 2])}, "
              f"M_(s-1) issued {rel(t[p + 3])} | MMA Q seen {rel(t[m + 1])}, S_0(0) {rel(t[m + 2])}, "
              f"last P V {rel(t[m + 4])}, memory read {rel(t[m + 5])} / {rel(t[m + 6])}")
        for k_ in (0, 1):
            c = 1024 * k_ + 16 * it
            ev = {n: rel(t[c + e]) for n, e in names.items()}
            print(f"    warpgroup {k_}: {int(t[c + 8])} key tiles, " + ", ".join(f"{n} {v}" for n, v in ev.items()))
    for k_ in (0, 1):
        nk = int(t[1024 * k_ + 8])
        if nk < 4 or rel(t[1024 * k_]) is None:
            continue
        ev = lambda e: np.array([t[1024 * k_ + 512 + 8 * j + e] for j in range(nk)], dtype=np.int64)  # noqa: E731
        s_seen, p_done = ev(0), ev(1)
        mid = slice(1, nk - 1)
        print(f"first item, warpgroup {k_}: median tile period {np.median(np.diff(s_seen)[mid]):.0f}, "
              f"softmax (S seen -> P stored) {np.median((p_done - s_seen)[mid]):.0f}, "
              f"P stored -> next S seen {np.median((s_seen[1:] - p_done[:-1])[mid]):.0f}")


if __name__ == "__main__":
    main()
