"""Benchmark of the Infini-attention forward on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--mode linear|delta]
                [--impl ours|reference]

A step is one pass of the whole forward (segment chunking, memory update,
local attention, memory read, gate) over one batch of the workload with the
inputs resident in HBM: one ``infini_attn_forward`` call, or for the
streaming workload one ``infini_attn_segment_step`` call per segment.  The
default workload is the 8B-shaped long input (B=2, H=32, d=128, N=8192,
L=524288, bf16); both update rules are timed on the same inputs, the linear
rule gives the headline figures and the delta rule's are under ``modes``.
``--workload`` / ``--mode`` select another workload or a single rule.  Under torchrun each rank runs its own copy of
the workload on its own GPU (independent (batch, head) problems, no
collective on the data path): weak scaling, value = tokens of all ranks /
max over ranks of the step time.

Timing: W warm-up steps, then K steps, each bracketed by CUDA events on the
launching stream.  Between steps, outside the events, the initial state is
reset to M_0 = 0, z_0 = 0 and a 1 GiB buffer is written so that no step
starts with its inputs in the 126 MB L2 (the write also lets the host
enqueue the step before the GPU reaches it).  A barrier and a device
synchronisation on both sides of the timed region.

``--impl reference`` times the fp64 CPU oracle on the host cores instead
(each step a bounded sample of the same workload); under torchrun only
rank 0 runs it.
"""

from __future__ import annotations

import argparse
import hashlib
import gc
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from compressive_memory_transformer_sm_b200 import DELTA, LINEAR  # noqa: E402
from compressive_memory_transformer_sm_b200 import workloads as W  # noqa: E402

METRIC = "Infini-attn fwd tokens/s per layer; TFLOP/s and % of B200 bf16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLUSH_BYTES = 1 << 30
PHASE_NAMES = ("update", "state", "attention", "rope", "projections", "backward_cuda_cores", "backward_tensor",
               "backward_memory_tensor")


# ------------------------------------------------------------------ work model
def algorithmic_flops(w: W.Workload, mode: int):
    """(attention kernel FLOPs, memory-update FLOPs) per step.

    Attention: n(n+1)(dk+dv) per segment for the unmasked causal half of
    Q K^T and P V, plus 2 n dk dv for sigma(Q) M_{s-1}.  Update: 2 n dk dv for
    sigma(K)^T U, plus 2 n dk dv for sigma(K) M_{s-1} under the delta rule.
    """
    attn = upd = 0
    for s0 in range(0, w.L, w.N):
        n = min(w.N, w.L - s0)
        attn += n * (n + 1) * (w.dk + w.dv) + 2 * n * w.dk * w.dv
        upd += (2 if mode == LINEAR else 4) * n * w.dk * w.dv
    return w.B * w.H * attn, w.B * w.H * upd


def algorithmic_bytes(w: W.Workload):
    """q, k, v read once and out written once in the input dtype, M and z read and written once (fp32)."""
    es = torch.finfo(w.dtype).bits // 8
    return w.B * w.H * (w.L * (2 * w.dk + 2 * w.dv) * es + 2 * (w.dk * w.dv + w.dk) * 4)


# ------------------------------------------------------------------ ranks
def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def init_dist(backend: str, timeout_s: float = 120.0):
    import datetime

    import torch.distributed as dist

    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
    return rank, world


def max_over_ranks(x: float, device) -> float:
    """The slowest rank's value (every rank takes the same collective step)."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def rank_seed(w: W.Workload, rank: int) -> int:
    """Each rank solves its own independent problem of the same shape."""
    return w.seed + 7 * rank


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock, power and throttle reasons while the GPU works."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(gpu_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), float(f[3]) if f[3] not in ("[N/A]", "N/A") else None,
                             float(f[4]), f[6], f[7], f[8], f[9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        busy = [r for r in rows if r[3] > 0] or rows
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in busy for i, v in enumerate(r[4:8]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in busy), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "samples_under_load": len([r for r in rows if r[3] > 0]),
                "power_w_max": max((r[2] for r in rows if r[2] is not None), default=None)}


# ------------------------------------------------------------------ peaks / traffic
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    with open(os.path.join(ROOT, "compressive_memory_transformer_sm_b200", "csrc", "sm100_attn.cuh"), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def measured_traffic(workload: str, mode: str):
    """DRAM bytes per attention launch from the committed ncu summary, if it matches the current kernel."""
    path = os.path.join(ROOT, "profiles", "attn_tc_kernel_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    if d.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    e = d.get("per_launch_bytes", {}).get(f"{workload}/{mode}")
    return None if e is None else float(e)


# ------------------------------------------------------------------ oracle timing (CPU)
def oracle_sample(w: W.Workload, mode: int, q, k, v, beta, budget_s: float, max_segments=None):
    """Runs the fp64 oracle over consecutive segments of head (0, 0) until the time budget is spent.

    Returns (tokens processed, seconds, segments).  Inputs are one head's [L, d] host tensors.
    """
    from oracle import infini_ref as R

    Q, K, V = (t.double().numpy() for t in (q, k, v))
    M = np.zeros((w.dk, w.dv))
    z = np.zeros(w.dk)
    tokens = segs = 0
    t0 = time.perf_counter()
    for s0, s1 in R.segment_bounds(w.L, w.N):
        _, M, z, _ = R.infini_attention_segment(Q[s0:s1], K[s0:s1], V[s0:s1], M, z, float(beta), mode)
        tokens += s1 - s0
        segs += 1
        if time.perf_counter() - t0 >= budget_s or (max_segments and segs >= max_segments):
            break
    return tokens, time.perf_counter() - t0, segs


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def one_head_host(w: W.Workload, seed: int):
    """Head (0, 0) of the workload's inputs, generated on the CPU with the same recipe."""
    one = w.with_(B=1, H=1)
    q, k, v, beta = W.make_inputs(one, device="cpu", seed=seed)
    return q[0, 0], k[0, 0], v[0, 0], beta[0]


def cpu_baseline(w: W.Workload, mode: int, budget_s: float):
    q, k, v, beta = one_head_host(w, w.seed)
    tokens, secs, segs = oracle_sample(w, mode, q, k, v, beta, budget_s)
    # tokens/s of the whole workload = one head's tokens/s divided by the B*H heads it must serve
    per_head = tokens / secs
    return {"value": per_head / (w.B * w.H), "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"fp64 NumPy oracle, head (0,0), first {segs} segment(s) ({tokens} tokens) in {secs:.2f} s; "
                      f"tokens/s scaled by 1/(B*H) = 1/{w.B * w.H} to the whole workload"}


# ------------------------------------------------------------------ our arm
def run_ours(args, w: W.Workload, modes):
    """Times every rule in ``modes`` on the same inputs; the first one is the headline line."""
    from compressive_memory_transformer_sm_b200 import api

    rank, world = init_dist("nccl")
    _, _, local = dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    q, k, v, beta = W.make_inputs(w, device=dev, seed=rank_seed(w, rank))
    M, z = W.empty_state(w, device=dev)
    out = torch.empty_like(v)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flags = api.FLAG_FORCE_SIMT if args.force_simt else 0
    if w.streaming:
        S = w.segments
        seg = lambda t: t.view(w.B, w.H, S, w.N, t.shape[3]).permute(2, 0, 1, 3, 4).contiguous()  # noqa: E731
        q, k, v = seg(q), seg(k), seg(v)
        out = torch.empty_like(v)

    def reset_state():  # M_0 = 0, z_0 = 0 are inputs: set before a step's events
        M.zero_()
        z.zero_()

    def step(mode):
        if w.streaming:
            for s in range(w.segments):
                api.infini_attn_segment_step(q[s], k[s], v[s], beta, M, z, out[s], mode, stream=stream)
        elif flags or args.rope:
            api.infini_attn_forward_ex(q, k, v, beta, M, z, out, w.N, mode, flags=flags, stream=stream,
                                       rope_base=args.rope)
        else:
            api.infini_attn_forward(q, k, v, beta, M, z, out, w.N, mode, stream=stream)

    peaks, peak_src = load_peaks()
    sampler = ClockSampler(local)
    per_mode = {}
    for mode in modes:
        for _ in range(args.warmup):
            reset_state()
            flush.fill_(1)
            step(mode)
        torch.cuda.synchronize(dev)
        api.infini_attn_profile_read(reset=True)

        # ------------------------------------------------------------ timed region
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        # The attention launch is timed with events inside the timed steps,
        # except for streaming workloads: an event pair around each of their
        # ~40 us launches adds ~8 us of device time per call (measured), so
        # their launch time comes from the breakdown pass below instead.
        api.infini_attn_profile_enable(0 if w.streaming else 1 << api.PHASE_ATTN)
        barrier(dev)
        torch.cuda.synchronize(dev)
        launches0 = api.infini_attn_launch_count()
        # Hold the stream for a few ms so that the host queues the timed steps
        # ahead of the device: the events then time device work back to back, not
        # host launch jitter (the e2e measurement below includes the host).
        if hasattr(torch.cuda, "_sleep"):
            torch.cuda._sleep(int(2e6 + 1e6 * args.steps))  # ~0.5 ms per step: room for host hiccups
        gc_was_enabled = gc.isenabled()
        gc.disable()
        wall0 = time.perf_counter()
        for i in range(args.steps):
            reset_state()
            flush.fill_(i & 0xff)
            evs[i][0].record(stream)
            step(mode)
            evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
        barrier(dev)
        wall = time.perf_counter() - wall0
        if gc_was_enabled:
            gc.enable()
        launches = api.infini_attn_launch_count() - launches0
        api.infini_attn_profile_enable(0)
        if api.infini_attn_device_status() != api.INFINI_OK:
            raise RuntimeError("a device-side wait timed out during the benchmark")
        step_ms = [a.elapsed_time(b) for a, b in evs]
        ms_local = sum(step_ms) / len(step_ms)
        attn_ms, attn_n = api.infini_attn_profile_read(reset=True)
        attn_ms_per_launch_local = attn_ms[api.PHASE_ATTN] / max(1, attn_n[api.PHASE_ATTN])

        # per-phase breakdown: a second pass of K steps with every launch bracketed
        api.infini_attn_profile_enable((1 << api.PHASES) - 1)
        for i in range(args.steps):
            reset_state()
            flush.fill_(i & 0xff)
            step(mode)
        torch.cuda.synchronize(dev)
        api.infini_attn_profile_enable(0)
        phase_ms, phase_n = api.infini_attn_profile_read(reset=True)

        if w.streaming:
            attn_ms_per_launch_local = phase_ms[api.PHASE_ATTN] / max(1, phase_n[api.PHASE_ATTN])
        ms = max_over_ranks(ms_local, dev)
        attn_ms_per_launch = max_over_ranks(attn_ms_per_launch_local, dev)
        f_attn, f_upd = algorithmic_flops(w, mode)
        per_launch_attn_flops = f_attn / (w.segments if w.streaming else 1)
        achieved = per_launch_attn_flops / (attn_ms_per_launch * 1e-3) / 1e12
        sustained = attn_ms_per_launch > 10.0
        peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
        per_mode[mode] = {
            "ms_per_step": ms, "value": w.B * w.L * world / (ms * 1e-3),
            "step_ms_min_max": [min(step_ms), max(step_ms)],
            "tflops": (f_attn + f_upd) * world / (ms * 1e-3) / 1e12,
            "pct_of_bf16_peak": 100.0 * (f_attn + f_upd) / (ms * 1e-3) / 1e12 / peak,
            "hbm_gbs": algorithmic_bytes(w) * world / (ms * 1e-3) / 1e9,
            "roofline": {"kernel": "attn_tc_kernel" if not args.force_simt else "simt_attn_kernel",
                         "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak,
                         "traffic": measured_traffic(w.name, W.MODE_NAMES[mode]),
                         "peak_source": f"{peak_src} {'bf16_tflops_sustained' if sustained else 'bf16_tflops'}",
                         "launch_ms": attn_ms_per_launch, "flops_per_launch": per_launch_attn_flops,
                         "launch_timed": ("breakdown pass (per-launch events perturb streaming launches)"
                                          if w.streaming else "timed steps")},
            "phases_ms_per_step": {name: phase_ms[i] / args.steps for i, name in enumerate(PHASE_NAMES)},
            "phase_launches_per_step": {name: phase_n[i] / args.steps for i, name in enumerate(PHASE_NAMES)},
            "gpu_launches": int(launches), "wall_s_timed_region": wall,
        }
    clocks = sampler.stop() if sampler else None
    head = per_mode[modes[0]]
    del q, k, v, out, flush
    torch.cuda.empty_cache()

    # ---------------------------------------------------------------- end to end, host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, modes[0], dev, stream, rank)

    result = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "step_ms_min_max": head["step_ms_min_max"],
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "N": w.N, "dk": w.dk, "dv": w.dv,
                   "mode": W.MODE_NAMES[modes[0]], "modes_timed": [W.MODE_NAMES[m] for m in modes],
                   "path": "simt" if args.force_simt else "tensor",
                   "rope_base": args.rope or None,
                   "streaming_steps": w.segments if w.streaming else 0,
                   "l2": "1 GiB buffer written between timed steps (outside the step events)",
                   "parallelism": f"independent problem per rank x{world}"},
        "tflops": head["tflops"], "pct_of_bf16_peak": head["pct_of_bf16_peak"], "hbm_gbs": head["hbm_gbs"],
        "roofline": head["roofline"], "phases_ms_per_step": head["phases_ms_per_step"],
        "phase_launches_per_step": head["phase_launches_per_step"],
        "gpu_launches": head["gpu_launches"], "clocks": clocks, "wall_s_timed_region": head["wall_s_timed_region"],
        "modes": {W.MODE_NAMES[m]: r for m, r in per_mode.items()},
    }
    if e2e is not None:
        result["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, modes[0], args.cpu_budget)
    if rank == 0:
        print(json.dumps(result), flush=True)
    import torch.distributed as dist

    if dist.is_initialized():
        dist.destroy_process_group()


def run_e2e(args, w: W.Workload, mode: int, dev, stream, rank):
    """Same metric through the public call with pinned HOST buffers: H2D of the step's inputs,
    the forward, D2H of the output and the state, all inside each step's events."""
    from compressive_memory_transformer_sm_b200 import api

    dq, dk_, dv_, db = W.make_inputs(w, device=dev, seed=rank_seed(w, rank))
    try:
        hq, hk, hv = (torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (dq, dk_, dv_))
        ho = torch.empty(w.B, w.H, w.L, w.dv, dtype=w.dtype, pin_memory=True)
    except RuntimeError as e:  # not enough pinnable host memory for this workload
        return {"value": None, "unit": "tokens/s", "unavailable": f"pinned host buffers: {str(e).splitlines()[0]}"}
    for h, d in ((hq, dq), (hk, dk_), (hv, dv_)):
        h.copy_(d)
    hb = db.cpu().pin_memory()
    hM = torch.zeros(w.B, w.H, w.dk, w.dv).pin_memory()
    hz = torch.zeros(w.B, w.H, w.dk).pin_memory()
    dM = torch.empty(hM.shape, device=dev)
    dz = torch.empty(hz.shape, device=dev)
    do = torch.empty(ho.shape, dtype=w.dtype, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hb, hM, hz))
    d2h = sum(t.numel() * t.element_size() for t in (ho, hM, hz))

    # The heads are independent problems: a whole-sequence step is pipelined over groups of
    # heads -- group i + 1's inputs copy in on one stream while group i computes on the
    # launching stream and group i - 1's output copies out on a third (both copy engines and
    # the SMs busy at once).  Every byte still crosses PCIe inside the step.
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    hg = max(1, w.H // 8)  # heads per group
    groups = [(b, h0, min(w.H, h0 + hg)) for b in range(w.B) for h0 in range(0, w.H, hg)]

    def step():
        if w.streaming:
            for d, h in ((dq, hq), (dk_, hk), (dv_, hv), (db, hb), (dM, hM), (dz, hz)):
                d.copy_(h, non_blocking=True)
            S = w.segments
            for s in range(S):
                sl = slice(s * w.N, (s + 1) * w.N)
                api.infini_attn_forward_ex(dq[:, :, sl], dk_[:, :, sl], dv_[:, :, sl], db, dM, dz, do[:, :, sl],
                                           w.N, mode, stream=stream)
            for h, d in ((ho, do), (hM, dM), (hz, dz)):
                h.copy_(d, non_blocking=True)
            return
        start = torch.cuda.Event()
        start.record(stream)
        s_in.wait_event(start)
        s_out.wait_event(start)
        with torch.cuda.stream(s_in):
            db.copy_(hb, non_blocking=True)
        for b, h0, h1 in groups:
            sel = (slice(b, b + 1), slice(h0, h1))
            with torch.cuda.stream(s_in):
                for d, h in ((dq, hq), (dk_, hk), (dv_, hv), (dM, hM), (dz, hz)):
                    d[sel].copy_(h[sel], non_blocking=True)
                e_in = torch.cuda.Event()
                e_in.record(s_in)
            stream.wait_event(e_in)
            api.infini_attn_forward(dq[sel], dk_[sel], dv_[sel], db[h0:h1], dM[sel], dz[sel], do[sel], w.N, mode,
                                    stream=stream)
            e_c = torch.cuda.Event()
            e_c.record(stream)
            s_out.wait_event(e_c)
            with torch.cuda.stream(s_out):
                for h, d in ((ho, do), (hM, dM), (hz, dz)):
                    h[sel].copy_(d[sel], non_blocking=True)
        e_out = torch.cuda.Event()
        e_out.record(s_out)
        stream.wait_event(e_out)

    for _ in range(max(1, min(args.warmup, args.e2e_steps))):
        flush.fill_(1)
        step()
    torch.cuda.synchronize(dev)
    n = max(1, min(args.steps, args.e2e_steps))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    barrier(dev)
    for i in range(n):
        flush.fill_(i & 0xff)
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier(dev)
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / n, dev)
    world = int(os.environ.get("WORLD_SIZE", 1))
    return {"value": w.B * w.L * world / (ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": n, "mode": W.MODE_NAMES[mode],
            "path": "pinned host -> device, forward, device -> pinned host, per step, pipelined over groups of "
                    "heads (copy in, compute and copy out on three streams)" if not w.streaming else
                    "pinned host -> device, forward, device -> pinned host, per step"}


# ------------------------------------------------------------------ reference arm
LAYER_METRIC = "Infini-attn layer fwd tokens/s (QKV projection + Infini-attention + output projection)"


def run_layer(args, w: W.Workload, mode: int):
    """``--layer``: the full multi-head layer through ``infini_attn_layer_forward`` on the
    workload's shape with d_model = H * 128, timed like the default line (device events
    per step, L2 flushed and the state reset between steps, outside the events)."""
    from compressive_memory_transformer_sm_b200 import api

    rank, world = init_dist("nccl")
    _, _, local = dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    D = w.H * w.dk
    x, w_qkv, w_o, beta = W.make_layer_inputs(w.B, w.H, w.L, D, seed=rank_seed(w, rank), device=dev)
    M, z = W.empty_state(w, device=dev)
    y = torch.empty(w.B, w.L, D, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(api.infini_attn_layer_workspace_size(w.B, w.H, w.L, w.N, D, mode), dtype=torch.uint8,
                     device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        M.zero_()
        z.zero_()
        flush.fill_(1)

    for _ in range(args.warmup):
        step()
        api.infini_attn_layer_forward(x, w_qkv, w_o, beta, M, z, y, w.H, w.N, mode, workspace=ws, stream=stream)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(local)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(dev)
    torch.cuda.synchronize(dev)
    launches0 = api.infini_attn_launch_count()
    if hasattr(torch.cuda, "_sleep"):
        torch.cuda._sleep(int(2e6 + 1e6 * args.steps))
    for i in range(args.steps):
        step()
        evs[i][0].record(stream)
        api.infini_attn_layer_forward(x, w_qkv, w_o, beta, M, z, y, w.H, w.N, mode, workspace=ws, stream=stream)
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier(dev)
    launches = api.infini_attn_launch_count() - launches0
    clocks = sampler.stop() if sampler else None
    if api.infini_attn_device_status() != api.INFINI_OK:
        raise RuntimeError("a device-side wait timed out during the benchmark")
    step_ms = [a.elapsed_time(b) for a, b in evs]
    ms = max_over_ranks(sum(step_ms) / len(step_ms), dev)
    # per-phase breakdown: a second pass with every launch bracketed
    api.infini_attn_profile_read(reset=True)
    api.infini_attn_profile_enable((1 << api.PHASES) - 1)
    for _ in range(args.steps):
        step()
        api.infini_attn_layer_forward(x, w_qkv, w_o, beta, M, z, y, w.H, w.N, mode, workspace=ws, stream=stream)
    torch.cuda.synchronize(dev)
    api.infini_attn_profile_enable(0)
    phase_ms, phase_n = api.infini_attn_profile_read(reset=True)
    f_attn, f_upd = algorithmic_flops(w, mode)
    f_proj = 2 * w.B * w.L * D * (3 * w.H * w.dk) + 2 * w.B * w.L * (w.H * w.dv) * D
    proj_ms = phase_ms[api.PHASE_PROJ] / args.steps
    peaks, peak_src = load_peaks()
    peak = peaks["bf16_tflops_sustained"] if ms > 10.0 else peaks["bf16_tflops"]
    tflops = (f_attn + f_upd + f_proj) * world / (ms * 1e-3) / 1e12
    result = {
        "metric": LAYER_METRIC, "value": w.B * w.L * world / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "step_ms_min_max": [min(step_ms), max(step_ms)], "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "N": w.N, "d_model": D,
                   "mode": W.MODE_NAMES[mode], "layer": "x W_qkv -> Infini-attention -> A W_o",
                   "l2": "1 GiB buffer written between timed steps (outside the step events)"},
        "tflops": tflops, "pct_of_bf16_peak": 100.0 * tflops / world / peak,
        "peak_source": f"{peak_src} {'bf16_tflops_sustained' if ms > 10.0 else 'bf16_tflops'}",
        "flops_per_step": {"projections": f_proj, "attention": f_attn, "update": f_upd},
        "phases_ms_per_step": {name: phase_ms[i] / args.steps for i, name in enumerate(PHASE_NAMES)},
        "projection_gemm": {"kernel": "gemm_tc_kernel", "ms_per_step": proj_ms, "launches_per_step":
                            phase_n[api.PHASE_PROJ] / args.steps,
                            "tflops": f_proj / (proj_ms * 1e-3) / 1e12 if proj_ms > 0 else None},
        "gpu_launches": int(launches), "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(result), flush=True)


DECODE_METRIC = "Infini-attn token-level streaming decode tokens/s (one token per (b, h) per call, fold per segment)"


def run_decode(args, w: W.Workload, mode: int):
    """``--decode``: one step = one segment of N tokens fed through ``infini_attn_decode_step``
    one token at a time (cache append, attention over the segment so far, memory read, gate;
    the fold into M, z on the segment's last token).  Device events around each segment."""
    from compressive_memory_transformer_sm_b200 import api

    rank, world = init_dist("nccl")
    _, _, local = dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    seg = w.with_(name=w.name, L=w.N)
    q, k, v, beta = W.make_inputs(seg, device=dev, seed=rank_seed(w, rank))
    qs = [q[:, :, t].contiguous() for t in range(w.N)]
    ks = [k[:, :, t].contiguous() for t in range(w.N)]
    vs = [v[:, :, t].contiguous() for t in range(w.N)]
    M, z = W.empty_state(w, device=dev)
    kc = torch.zeros(w.B, w.H, w.N, w.dk, dtype=w.dtype, device=dev)
    vc = torch.zeros(w.B, w.H, w.N, w.dv, dtype=w.dtype, device=dev)
    o = torch.empty(w.B, w.H, w.dv, dtype=w.dtype, device=dev)

    def segment():
        for t in range(w.N):
            api.infini_attn_decode_step(qs[t], ks[t], vs[t], kc, vc, beta, M, z, o, t, mode, stream=stream)

    for _ in range(args.warmup):
        segment()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(local)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(dev)
    torch.cuda.synchronize(dev)
    launches0 = api.infini_attn_launch_count()
    for i in range(args.steps):
        evs[i][0].record(stream)
        segment()
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier(dev)
    launches = api.infini_attn_launch_count() - launches0
    clocks = sampler.stop() if sampler else None
    if api.infini_attn_device_status() != api.INFINI_OK:
        raise RuntimeError("a device-side wait timed out during the benchmark")
    step_ms = [a.elapsed_time(b) for a, b in evs]
    ms = max_over_ranks(sum(step_ms) / len(step_ms), dev)
    result = {
        "metric": DECODE_METRIC, "value": w.B * w.N * world / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "us_per_token": 1e3 * ms / w.N,
        "higher_is_better": True, "step_ms_min_max": [min(step_ms), max(step_ms)], "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "dk": w.dk, "dv": w.dv,
                   "mode": W.MODE_NAMES[mode], "step": "one segment of N decode calls, fold on the last"},
        "gpu_launches": int(launches), "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(result), flush=True)


BACKWARD_METRIC = "Infini-attn bwd tokens/s per layer (gradients of q, k, v, beta, M_0, z_0 through the forward)"
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965  # SMs x fp32 lanes x FMA x max SM clock (GHz): 74.4 TFLOP/s


def run_backward(args, w: W.Workload, mode: int):
    """``--backward``: one step = one ``infini_attn_backward`` call (forward recomputation
    included) on the workload's shape, timed like the default line."""
    from compressive_memory_transformer_sm_b200 import api

    rank, world = init_dist("nccl")
    _, _, local = dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    q, k, v, beta = W.make_inputs(w, device=dev, seed=rank_seed(w, rank))
    g = torch.Generator(device=dev)
    g.manual_seed(rank_seed(w, rank) + 1)
    d_out = torch.randn(v.shape, generator=g, device=dev).to(w.dtype)
    ws = torch.empty(api.infini_attn_backward_workspace_size(w.B, w.H, w.L, w.N, w.dk, w.dv, mode), dtype=torch.uint8,
                     device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        return api.infini_attn_backward(q, k, v, beta, d_out, w.N, mode, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(local)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(dev)
    torch.cuda.synchronize(dev)
    launches0 = api.infini_attn_launch_count()
    for i in range(args.steps):
        flush.fill_(i & 0xff)
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier(dev)
    launches = api.infini_attn_launch_count() - launches0
    clocks = sampler.stop() if sampler else None
    if api.infini_attn_device_status() != api.INFINI_OK:
        raise RuntimeError("a device-side wait timed out during the benchmark")
    step_ms = [a.elapsed_time(b) for a, b in evs]
    ms = max_over_ranks(sum(step_ms) / len(step_ms), dev)
    api.infini_attn_profile_read(reset=True)
    api.infini_attn_profile_enable((1 << api.PHASES) - 1)
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize(dev)
    api.infini_attn_profile_enable(0)
    phase_ms, phase_n = api.infini_attn_profile_read(reset=True)
    # algorithmic work: the forward recomputation plus the backward's products (local
    # attention: S, dP, dV, dK, dQ = 5 causal products of n(n+1)/2 pairs x d x 2 FLOP per
    # segment; memory read and update: about 12 n dk dv for the linear rule, 18 for delta)
    f_fwd_attn, f_fwd_upd = algorithmic_flops(w, mode)
    f_local = f_mem = 0
    for s0 in range(0, w.L, w.N):
        n = min(w.N, w.L - s0)
        f_local += 5 * n * (n + 1) * w.dk
        f_mem += (12 if mode == LINEAR else 18) * n * w.dk * w.dv
    f_local *= w.B * w.H
    f_mem *= w.B * w.H
    total = f_fwd_attn + f_fwd_upd + f_local + f_mem
    tflops = total * world / (ms * 1e-3) / 1e12
    tc_ms = phase_ms[api.PHASE_BWD_TC] / args.steps
    peaks, peak_src = load_peaks()
    if tc_ms > 0:  # the local attention's gradients on the tensor cores (bf16, head size 128)
        sustained = tc_ms > 10.0
        peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
        achieved = f_local / (tc_ms * 1e-3) / 1e12
        roofline = {"kernel": "bwd_dq_tc_kernel + bwd_dkdv_tc_kernel", "bound": "tensor", "achieved": achieved,
                    "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None,
                    "peak_source": f"{peak_src} {'bf16_tflops_sustained' if sustained else 'bf16_tflops'}",
                    "launch_ms": tc_ms, "flops_per_step": f_local}
    else:
        roofline = {"kernel": "backward (CUDA cores, fp32)", "bound": "alu", "achieved": tflops / world,
                    "peak": FP32_ALU_TFLOPS, "unit": "TFLOP/s", "frac": tflops / world / FP32_ALU_TFLOPS,
                    "peak_source": "148 SMs x 128 fp32 lanes x 2 (FMA) x 1.965 GHz"}
    result = {
        "metric": BACKWARD_METRIC, "value": w.B * w.L * world / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "step_ms_min_max": [min(step_ms), max(step_ms)], "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "N": w.N, "dk": w.dk, "dv": w.dv,
                   "mode": W.MODE_NAMES[mode], "step": "infini_attn_backward (forward recomputed inside)",
                   "l2": "1 GiB buffer written between timed steps (outside the step events)"},
        "tflops": tflops, "flops_per_step": total, "roofline": roofline,
        "phases_ms_per_step": {name: phase_ms[i] / args.steps for i, name in enumerate(PHASE_NAMES)},
        "gpu_launches": int(launches), "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(result), flush=True)


def run_reference(args, w: W.Workload, mode: int):
    rank, world, _ = dist_env()
    if rank != 0:
        return  # only rank 0 times the CPU oracle
    q, k, v, beta = one_head_host(w, w.seed)
    budget = args.ref_step_budget
    for _ in range(args.warmup):
        oracle_sample(w, mode, q, k, v, beta, budget, max_segments=1)
    tokens = 0
    secs = 0.0
    segs = 0
    for _ in range(args.steps):
        t, s, n = oracle_sample(w, mode, q, k, v, beta, budget, max_segments=1)
        tokens += t
        secs += s
        segs += n
    per_head = tokens / secs
    value = per_head / (w.B * w.H)
    cores = blas_threads()
    sample = (f"each step: fp64 NumPy oracle on the first segment ({w.N if w.N < w.L else w.L} tokens) of head "
              f"(0,0); tokens/s scaled by 1/(B*H) = 1/{w.B * w.H} to the whole workload")
    f_attn, f_upd = algorithmic_flops(w, mode)
    result = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "N": w.N, "dk": w.dk, "dv": w.dv,
                   "mode": W.MODE_NAMES[mode]},
        "tflops": value / (w.B * w.L) * (f_attn + f_upd) / 1e12,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(result), flush=True)


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=sorted(W.WORKLOADS), default=W.LONG_8B.name)
    ap.add_argument("--mode", choices=("linear", "delta"), default=None)
    ap.add_argument("--force-simt", action="store_true", help="time the CUDA-core kernels instead")
    ap.add_argument("--shape", default=None, help="B,H,L,N override of the workload's sizes (for profiling)")
    ap.add_argument("--rope", type=float, default=0.0,
                    help="rotary position embeddings with this base on the local attention (0: none)")
    ap.add_argument("--layer", action="store_true",
                    help="time the full layer (QKV projection + attention + output projection) instead")
    ap.add_argument("--decode", action="store_true",
                    help="time token-level streaming decode (one segment of single-token calls per step)")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (infini_attn_backward, forward recomputed inside)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3, help="timed steps of the host-buffer measurement")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-step-budget", type=float, default=5.0)
    return ap.parse_args(argv)


def main(argv=None):
    args = parse(argv)
    w = W.WORKLOADS[args.workload]
    if args.shape:
        B, H, L, N = (int(x) for x in args.shape.split(","))
        w = w.with_(name=f"{w.name}@{B}x{H}x{L}x{N}", B=B, H=H, L=L, N=N)
    modes = ({"linear": LINEAR, "delta": DELTA}[args.mode],) if args.mode else tuple(w.modes)
    mode = modes[0]
    if args.rope and (w.streaming or args.layer or args.decode or args.backward):
        raise SystemExit("--rope applies to the whole-sequence forward (infini_attn_forward_ex) only")
    if args.warmup < 3 and args.impl == "ours":
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args, w, mode)
    elif args.layer:
        run_layer(args, w, mode)
    elif args.decode:
        run_decode(args, w, mode)
    elif args.backward:
        run_backward(args, w, mode)
    else:
        run_ours(args, w, modes)


if __name__ == "__main__":
    main()
