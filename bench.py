#!/usr/bin/env python
"""Throughput of the biased-attention forward on B200: TFLOP/s and % of roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload tri_1024] [--impl ours|reference]

A step is one evo_attn_fwd call over one batch of the workload (default: the
large triangle-attention case, B=1, N=S=1024, H=4, D=32, bf16, synthetic
seeded inputs).  FLOPs per step are 4*B*N*H*S^2*D.  The kernel-only number
(``value``) times K back-to-back calls on inputs resident in HBM (1.1 GB of
inputs, larger than the 126 MB L2, so no flush is needed between steps) with
CUDA events on the launching stream, bracketed by a barrier and a device
synchronize, max over ranks.  ``e2e`` times the host-memory entry point
(``evo_attn_fwd_host``) on the same workload: every step copies the inputs
from pinned host memory and O / LSE back, in chunks of n slices whose copies
overlap the kernels of the neighbouring chunks.

Multi-GPU: the forward pass has no exchange step; each rank runs its own
replica of the workload on its own GPU (weak scaling, no data-path
collective).  ``--impl reference`` times the float64 CPU oracle instead (rank
0 only), on a bounded sample of (b, n, h) slices per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from triangle_biased_attention_b200 import workloads as W  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
KERNEL_SOURCES = ["common.cuh", "ptx_sm100.cuh", "tile_sm100.cuh", "fwd_tri_sm100.cuh", "evo_attn.cu"]
KERNEL_SOURCES_BWD = ["common.cuh", "ptx_sm100.cuh", "tile_sm100.cuh", "bwd_simt.cuh", "bwd_tri_sm100.cuh",
                      "evo_attn.cu"]
KERNEL_SOURCES_TRIMUL = ["common.cuh", "ptx_sm100.cuh", "tile_sm100.cuh", "trimul_sm100.cuh", "evo_attn.cu"]
KERNEL_NAME = "evo_fwd_tri_kernel"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="tri_1024", choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--op", default="attn", choices=["attn", "trimul"],
                    help="attn: biased attention (--pass fwd|bwd); trimul: the triangle-multiplication "
                         "contraction on --trimul-workload")
    ap.add_argument("--trimul-workload", default="trimul_768", choices=sorted(W.TRIMUL_WORKLOADS))
    ap.add_argument("--incoming", action="store_true", help="trimul: the incoming direction")
    ap.add_argument("--pass", dest="which", default="fwd", choices=["fwd", "bwd"],
                    help="fwd: the forward pass (the headline metric); bwd: the backward pass "
                         "(evo_attn_bwd: dQ, dK, dV and the requested bias gradients)")
    ap.add_argument("--e2e-steps", type=int, default=5,
                    help="steps of the host-memory leg (0 skips it; e2e is then null)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--flush-l2", action="store_true",
                    help="write a 256 MB buffer before every timed step and time the kernels alone (cold L2)")
    return ap.parse_args()


# ------------------------------------------------------------------ plumbing
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if (args.impl == "ours" and torch.cuda.is_available()) else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"]))}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(sources=None) -> str:
    h = hashlib.sha256()
    for name in (KERNEL_SOURCES if sources is None else sources):
        with open(os.path.join(ROOT, "triangle_biased_attention_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, sources=None):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary (key: the workload, "bwd:<workload>" for the backward), if it was
    taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[workload]
        if e.get("kernel_source_hash") == kernel_source_hash(sources):
            return float(e["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        pass
    return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, index: int, period_s: float = 0.005):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML unavailable: no clock record
            self._nv = None
        self.period = period_s

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def record(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ------------------------------------------------------------------ oracle leg
def time_oracle(case, slices_per_step: int, steps: int, warmup: int, seed: int):
    """Times the float64 CPU oracle on `steps` samples of `slices_per_step`
    (b, n, h) slices each.  Returns (seconds per step, flops per step, cores)."""
    import oracle
    B, N, S, H, D = case.shape
    total = B * N * H
    rng = torch.Generator().manual_seed(seed)
    cores = oracle.max_threads()
    flops_slice = 4 * S * S * D
    per_step = []

    def sample():
        idx = torch.randint(0, total, (slices_per_step,), generator=rng).tolist()
        return [(i // (N * H), (i // H) % N, i % H) for i in idx]

    for _ in range(warmup):
        oracle.attention_slices(case.q, case.k, case.v, case.mask, case.pair, sample())
    for _ in range(steps):
        sl = sample()
        t0 = time.perf_counter()
        oracle.attention_slices(case.q, case.k, case.v, case.mask, case.pair, sl)
        per_step.append(time.perf_counter() - t0)
    return sum(per_step) / len(per_step), flops_slice * slices_per_step, cores


def cpu_model() -> str:
    """The host CPU's model name and logical CPU count, from /proc/cpuinfo."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return f"{line.split(':', 1)[1].strip()} ({os.cpu_count()} logical CPUs)"
    except OSError:
        pass
    return f"unknown ({os.cpu_count()} logical CPUs)"


def cpu_baseline(case, args, target_s: float = 10.0):
    """The oracle on random (b, n, h) slices of the workload, in chunks of
    4 slices per host core, until about `target_s` seconds have been spent."""
    import oracle
    cores = oracle.max_threads()
    chunk = 4 * cores
    done_sec = done_flops = 0.0
    n_slices = 0
    seed = args.seed
    while done_sec < target_s and n_slices < case.q.shape[0] * case.q.shape[1] * case.q.shape[3]:
        sec, fl, cores = time_oracle(case, chunk, 1, 0, seed)
        done_sec += sec
        done_flops += fl
        n_slices += chunk
        seed += 1
    return {"value": done_flops / done_sec / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "cpu": cpu_model(), "nproc": os.cpu_count(),
            "sample": f"{n_slices} random (b,n,h) slices of {args.workload} ({done_flops / 1e9:.0f} GFLOP "
                      f"in {done_sec:.1f} s, float64 C, OpenMP)"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    wl = W.WORKLOADS[args.workload]
    case = W.make_case(args.workload, args.seed)
    import oracle
    cores = oracle.max_threads()
    # each step: one slice per host core, so a step is ~0.1-0.5 s of work
    slices = max(1, cores)
    sec, flops, cores = time_oracle(case, slices, args.steps, args.warmup, args.seed)
    tflops = flops / sec / 1e12
    line = {
        "metric": "Evoformer attn fwd TFLOP/s and % of roofline (triangle attn, N_res=1024)",
        "value": tflops, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded numpy PCG64)",
        "config": workload_config(wl), "impl": "reference",
        "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "cpu": cpu_model(), "nproc": os.cpu_count(),
                         "sample": f"{slices} random (b,n,h) slices of {args.workload} per step"},
        "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(wl, flush=False):
    return {"workload": wl.name, "B": wl.B, "N": wl.N, "S": wl.S, "H": wl.H, "D": wl.D,
            "dtype": "bf16" if wl.dtype == torch.bfloat16 else "fp32",
            "l2": ("256 MB written before every step; kernels timed alone (cold L2)" if flush else
                   "inputs (%.2f GB) %s the 126 MB L2; no flush" % (
                       alg_bytes(wl) / 1e9, "larger than" if alg_bytes(wl) > 126e6 else "NOT larger than")),
            "parallelism": "replicas (one full workload per GPU)"}


def pair_bias_stream(wl) -> int:
    """Bytes of pair-bias tiles loaded per launch (0 without a pair bias, or
    when S % 8 != 0 and the softmax reads the bias from global memory)."""
    if wl.name.startswith("msa_col") or wl.dtype == torch.float32 or wl.S % 8:
        return 0
    ns = 3 if wl.D <= 32 else (2 if wl.D == 64 else 1)
    qb = (wl.S + 127) // 128
    tiles = qb * wl.H * ((wl.N + ns - 1) // ns) * wl.B
    return tiles * qb * 128 * 128 * 2


def alg_bytes(wl) -> int:
    es = 2 if wl.dtype == torch.bfloat16 else 4
    qkvo = 4 * wl.B * wl.N * wl.S * wl.H * wl.D * es
    pair = wl.B * wl.H * wl.S * wl.S * es if not wl.name.startswith("msa_col") else 0
    mask = wl.B * wl.N * wl.S * es
    lse = wl.B * wl.N * wl.H * wl.S * 4
    return qkvo + pair + mask + lse


# ------------------------------------------------------------------ our arm
def run_ours(args, rank, world, local):
    import triangle_biased_attention_b200 as evo
    wl = W.WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    case = W.make_case(args.workload, args.seed + rank)
    q, k, v = (t.to(dev) for t in (case.q, case.k, case.v))
    mask = case.mask.to(dev) if case.mask is not None else None
    pair = case.pair.to(dev) if case.pair is not None else None
    out = torch.empty_like(q)
    lse = torch.empty((wl.B, wl.N, wl.H, wl.S), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)
    flops = wl.flops

    def step():
        evo.evo_attn(q, k, v, mask, pair, out=out, lse=lse, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
    status = evo.evo_attn_sync_status(stream.cuda_stream)
    if status != evo.EVO_OK:
        raise RuntimeError(f"kernel status {status}: {evo.evo_attn_strerror(status)}")

    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index)
    barrier(world)
    torch.cuda.synchronize(dev)
    if args.flush_l2:
        # cold L2: a 256 MB write (twice the 126 MB L2) before every step; only
        # the kernels are timed, each between its own pair of events
        scratch = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        with sampler:
            for e0, e1 in evs:
                with torch.cuda.stream(stream):
                    scratch.fill_(1)
                e0.record(stream)
                step()
                e1.record(stream)
            torch.cuda.synchronize(dev)
        barrier(world)
        ms = sum(e0.elapsed_time(e1) for e0, e1 in evs)
    else:
        with sampler:
            start.record(stream)
            for _ in range(args.steps):
                step()
            stop.record(stream)
            torch.cuda.synchronize(dev)
        barrier(world)
        ms = start.elapsed_time(stop)
    status = evo.evo_attn_sync_status(stream.cuda_stream)
    if status != evo.EVO_OK:
        raise RuntimeError(f"kernel status {status}: {evo.evo_attn_strerror(status)}")
    ms_max = max_over_ranks(ms, world, dev)
    ms_per_step = ms_max / args.steps
    value = world * flops * args.steps / (ms_max * 1e-3) / 1e12

    # end to end: pinned host inputs -> device -> kernel -> O, LSE back to
    # pinned host, through the host-memory entry point (chunked, overlapped)
    pin = lambda t: None if t is None else t.pin_memory()
    host_in = [pin(t) for t in (case.q, case.k, case.v, case.mask, case.pair)]
    host_o = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    host_lse = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host_in if t is not None)
    d2h = host_o.numel() * host_o.element_size() + host_lse.numel() * host_lse.element_size()
    dev_bufs = (q, k, v, mask, pair, out, lse)

    def e2e_step():
        evo.evo_attn_from_host(*host_in, out=host_o, lse=host_lse, device_buffers=dev_bufs, stream=stream)

    e2e = None
    if args.e2e_steps > 0:
        with torch.cuda.stream(stream):
            for _ in range(2):
                e2e_step()
            torch.cuda.synchronize(dev)
            barrier(world)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.e2e_steps):
                e2e_step()
            e1.record(stream)
            torch.cuda.synchronize(dev)
        barrier(world)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / args.e2e_steps
        e2e = {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": args.e2e_steps}

    peaks, peak_src = load_peaks()
    achieved = flops / (ms / args.steps * 1e-3) / 1e12  # this rank's kernel, per launch
    t_flop = flops / (peaks["bf16_tflops"] * 1e12)
    t_mem = alg_bytes(wl) / (peaks["hbm_gbs"] * 1e9)
    bound = "tensor" if t_flop >= t_mem else "hbm"
    if bound == "tensor":
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"]}
    else:
        gbs = alg_bytes(wl) / (ms / args.steps * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"]}
    roof["traffic"] = recorded_traffic(args.workload)
    roof["peak_source"] = f"{peak_src} (MEASURED_PEAKS.json burst figure)" if peak_src == "measured" \
        else "fallback (6.65 TB/s, 1.59 PFLOP/s)"
    roof["alg_flops_per_launch"] = flops
    roof["alg_bytes_per_launch"] = alg_bytes(wl)
    bias = pair_bias_stream(wl)
    if bias:
        # the pair-bias tiles the kernel moves from L2 into shared memory: one
        # 128 x 128 tile per (tile, key block), shared by the slices of a tile
        roof["pair_bias_stream"] = {"l2_to_sm_bytes_per_launch": bias,
                                    "gbs": bias / (ms / args.steps * 1e-3) / 1e9,
                                    "unique_bytes": wl.B * wl.H * wl.S * wl.S * 2}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(case, args)

    if rank == 0:
        line = {
            "metric": "Evoformer attn fwd TFLOP/s and % of roofline (triangle attn, N_res=1024)",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded numpy PCG64, bf16)",
            "config": workload_config(wl, args.flush_l2),
            "roofline_pct": 100.0 * roof["frac"] if bound == "tensor" else 100.0 * roof["frac"],
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": args.steps,
            "kernel": KERNEL_NAME,
            "clocks": sampler.record(),
        }
        print(json.dumps(line), flush=True)


def bwd_flops(wl) -> int:
    # five products of 2*S*S*D each per (b, n, h): S = Q K^T (recomputed),
    # dP = dO V^T, dV = P^T dO, dK = dT^T Q, dQ = dT K
    return 10 * wl.B * wl.N * wl.H * wl.S * wl.S * wl.D


def upstream_grad(case, seed: int):
    import numpy as np
    rng = np.random.Generator(np.random.PCG64(50_000 + seed))
    return torch.from_numpy(rng.standard_normal(case.q.shape, dtype=np.float32)).to(case.q.dtype)


def cpu_baseline_bwd(case, do, args, target_s: float = 10.0):
    """The oracle's backward on random (b, n, h) slices until about
    `target_s` seconds have been spent."""
    import oracle
    B, N, S, H, D = case.shape
    cores = oracle.max_threads()
    rng = torch.Generator().manual_seed(args.seed)
    done_sec = 0.0
    n_slices = 0
    while done_sec < target_s and n_slices < B * N * H:
        idx = torch.randint(0, B * N * H, (cores,), generator=rng).tolist()
        sl = [(i // (N * H), (i // H) % N, i % H) for i in idx]
        t0 = time.perf_counter()
        oracle.default().attention_bwd_slices(case.q, case.k, case.v, case.mask, case.pair, do, sl)
        done_sec += time.perf_counter() - t0
        n_slices += len(sl)
    flops = 10.0 * S * S * D * n_slices
    return {"value": flops / done_sec / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "cpu": cpu_model(), "nproc": os.cpu_count(),
            "sample": f"backward of {n_slices} random (b,n,h) slices of {args.workload} "
                      f"({flops / 1e9:.0f} GFLOP in {done_sec:.1f} s, float64 C, OpenMP)"}


def run_ours_bwd(args, rank, world, local):
    """The backward pass: each step is one evo_attn_bwd call (zeroing of the
    fp32 accumulators, row statistics, the gradient kernel, the rounding
    kernel) on the forward's outputs, every gradient requested."""
    import triangle_biased_attention_b200 as evo
    wl = W.WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    case = W.make_case(args.workload, args.seed + rank)
    do_h = upstream_grad(case, args.seed + rank)
    q, k, v, do = (t.to(dev) for t in (case.q, case.k, case.v, do_h))
    mask = case.mask.to(dev) if case.mask is not None else None
    pair = case.pair.to(dev) if case.pair is not None else None
    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        o, lse = evo.evo_attn(q, k, v, mask, pair, stream=stream)
    B, N, S, H, D = q.shape
    ws = torch.empty(evo.evo_attn_bwd_workspace_size(B, N, S, H, D), dtype=torch.uint8, device=dev)

    def step():
        return evo.evo_attn_backward(q, k, v, mask, pair, o, lse, do, workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
    status = evo.evo_attn_sync_status(stream.cuda_stream)
    if status != evo.EVO_OK:
        raise RuntimeError(f"kernel status {status}: {evo.evo_attn_strerror(status)}")
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index)
    barrier(world)
    torch.cuda.synchronize(dev)
    with sampler:
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(args.steps):
                step()
            stop.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    ms = start.elapsed_time(stop)
    status = evo.evo_attn_sync_status(stream.cuda_stream)
    if status != evo.EVO_OK:
        raise RuntimeError(f"kernel status {status}: {evo.evo_attn_strerror(status)}")
    ms_max = max_over_ranks(ms, world, dev)
    flops = bwd_flops(wl)
    value = world * flops * args.steps / (ms_max * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    achieved = flops / (ms / args.steps * 1e-3) / 1e12
    roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": achieved / peaks["bf16_tflops"],
            "traffic": recorded_traffic("bwd:" + args.workload, KERNEL_SOURCES_BWD),
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json burst figure)" if peak_src == "measured"
            else "fallback (6.65 TB/s, 1.59 PFLOP/s)",
            "alg_flops_per_launch": flops,
            "timed": "whole evo_attn_bwd call (3 kernels and the zeroing copies of the fp32 sums)"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_bwd(case, do_h, args)
    if rank == 0:
        line = {
            "metric": "Evoformer attn bwd TFLOP/s (dQ, dK, dV, dmask, dpair; 10*B*N*H*S^2*D flops)",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded numpy PCG64, bf16)",
            "config": workload_config(wl), "roofline": roof, "cpu_baseline": cpu, "e2e": None,
            "gpu_launches": 3 * args.steps, "kernel": "evo_bwd_tri_kernel", "clocks": sampler.record(),
        }
        print(json.dumps(line), flush=True)


def run_ours_trimul(args, rank, world, local):
    """Triangle multiplication: each step is one evo_trimul call (two transposes
    to channel-first copies, the tcgen05 batched GEMM, the transpose back)."""
    import triangle_biased_attention_b200 as evo
    Bt, N, C = W.TRIMUL_WORKLOADS[args.trimul_workload]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    a_h, b_h = W.trimul_case(Bt, N, C, torch.bfloat16, args.seed + rank)
    a, b = a_h.to(dev), b_h.to(dev)
    z = torch.empty_like(a)
    ws = torch.empty(evo.evo_trimul_workspace_size(Bt, N, C), dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(dev)
    outgoing = not args.incoming

    def step():
        evo.trimul(a, b, outgoing, out=z, workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
    if evo.evo_attn_sync_status(stream.cuda_stream) != evo.EVO_OK:
        raise RuntimeError("kernel status")
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index)
    barrier(world)
    torch.cuda.synchronize(dev)
    with sampler:
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(args.steps):
                step()
            stop.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    ms = start.elapsed_time(stop)
    if evo.evo_attn_sync_status(stream.cuda_stream) != evo.EVO_OK:
        raise RuntimeError("kernel status")
    ms_max = max_over_ranks(ms, world, dev)
    flops = 2 * Bt * C * N ** 3
    alg = 3 * Bt * N * N * C * 2
    value = world * flops * args.steps / (ms_max * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    achieved = flops / (ms / args.steps * 1e-3) / 1e12
    t_flop = flops / (peaks["bf16_tflops"] * 1e12)
    t_mem = alg / (peaks["hbm_gbs"] * 1e9)
    roof = {"bound": "tensor" if t_flop >= t_mem else "hbm", "achieved": achieved, "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"], "traffic": None,
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json burst figure)" if peak_src == "measured"
            else "fallback (6.65 TB/s, 1.59 PFLOP/s)",
            "alg_flops_per_launch": flops, "alg_bytes_per_launch": alg,
            "timed": "whole evo_trimul call (two transposes in, the GEMM, one transpose out)"}
    roof["traffic"] = recorded_traffic("trimul:" + args.trimul_workload, KERNEL_SOURCES_TRIMUL)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle.trimul as OT
        # the oracle on a bounded sample of the same problem: channels in
        # groups of 8 until about 10 s have been spent
        sec, done = 0.0, 0
        while sec < 10.0 and done < C:
            cs = min(8, C - done)
            t0 = time.perf_counter()
            OT.trimul(a_h[..., done:done + cs], b_h[..., done:done + cs], outgoing)
            sec += time.perf_counter() - t0
            done += cs
        import numpy as _np
        cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
        cpu = {"value": 2 * Bt * done * N ** 3 / sec / 1e12, "unit": "TFLOP/s", "cores": cores,
               "kind": "oracle", "cpu": cpu_model(), "nproc": os.cpu_count(),
               "sample": f"{done} of {C} channels of {args.trimul_workload} ({sec:.1f} s, float64 numpy matmul, "
                         f"numpy {_np.__version__})"}
    if rank == 0:
        line = {
            "metric": "triangle multiplication TFLOP/s (2*Bt*C*N^3 flops)",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded numpy PCG64, bf16)",
            "config": {"workload": args.trimul_workload, "Bt": Bt, "N": N, "C": C,
                       "direction": "outgoing" if outgoing else "incoming",
                       "l2": "inputs (%.2f GB) larger than the 126 MB L2; no flush" % (alg / 1e9),
                       "parallelism": "replicas (one full workload per GPU)"},
            "roofline": roof, "cpu_baseline": cpu, "e2e": None, "gpu_launches": 4 * args.steps,
            "kernel": "evo_trimul_gemm_kernel", "clocks": sampler.record(),
        }
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        elif args.op == "trimul":
            run_ours_trimul(args, rank, world, local)
        elif args.which == "bwd":
            run_ours_bwd(args, rank, world, local)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
