"""Benchmark of the structured-mask attention hot path on B200.

One step = one ``sattn_fwd`` call (rotary prep pass, block/band planning and
the tcgen05 attention kernel) over the Llama-2-7B-shaped LM-Infinite layer:
B=1, 32 heads, T=16384, d=128, bf16, n_start=4, L_pretrain=w=4096, capped
RoPE theta=1e4, sink keys scaled x8.  Metric: effective TFLOP/s counted over
unmasked (q, k) pairs at 4*d FLOPs each (whole job, all ranks), with tokens/s
alongside.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: one process per GPU (torchrun); every rank runs its own
independent problem (heads/batches are independent), so per-GPU work is
fixed as N grows ("scaling": "weak") and no data-path collective exists;
the only collectives are the barrier and the max-over-ranks of the timings.

``--impl reference`` times the fp64 CPU oracle on the host cores (rank 0
only) on bounded row samples of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_structured_b200 import synth  # noqa: E402

WORKLOAD = "c2_lminf_16k"
METRIC = "effective TFLOP/s over unmasked pairs (fraction of bf16 TC peak), tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (read + write) per launch of the attention kernel on this
# workload, from the ncu capture summarised in profiles/; None when the
# kernel changed since the counters were taken.
ATTN_TRAFFIC_BYTES = None  # the kernel changed since the last DRAM capture


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def unmasked_pairs_per_head(wl) -> int:
    """Closed-form count of kept (q, k) pairs of one head for a workload with
    no separators and no top-k: row i keeps min(i+1, n_start+w+1) keys."""
    i = np.arange(wl.T, dtype=np.int64)
    return int(np.minimum(i + 1, wl.n_start + wl.window + 1).sum())


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def config_dict(wl, pairs_per_rank):
    return {
        "workload": "%s: LM-Infinite Lambda-mask layer, B=%d H=%d T=%d d=%d bf16, n_start=%d, L_pretrain=w=%d, "
                    "capped RoPE theta=%g, keys 0-3 x8" % (wl.name, wl.B, wl.Hq, wl.T, wl.d, wl.n_start, wl.window,
                                                          wl.rope_theta),
        "B": wl.B, "H": wl.Hq, "T": wl.T, "d": wl.d, "n_start": wl.n_start, "window": wl.window,
        "L_pretrain": wl.L_pretrain, "rope_theta": wl.rope_theta,
        "unmasked_pairs_per_rank": pairs_per_rank,
        "l2": "no flush: each step reads Q,K,V (384 MB) and its 256 MB rotated copies, > 126 MB L2",
    }


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, fallback_index: int = 0):
        self.gpu_id = gpu_id
        self.fallback_index = fallback_index
        try:
            self.n_gpus = len(subprocess.run(["nvidia-smi", "-L"], capture_output=True, text=True,
                                             timeout=30).stdout.strip().splitlines())
        except (OSError, subprocess.SubprocessError):
            self.n_gpus = 0
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, ValueError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        mine = [ln for ln in self.lines if ln.split(",")[0].strip().lower() == self.gpu_id.lower()]
        if not mine:  # uuid format mismatch: fall back to the visible device's line
            idx = self.fallback_index
            mine = [ln for x, ln in enumerate(self.lines) if self.n_gpus and x % self.n_gpus == idx]
        for ln in mine:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def profile_collect(lib):
    import ctypes
    names = ctypes.create_string_buffer(32 * 64)
    launches = (ctypes.c_int32 * 64)()
    total = (ctypes.c_double * 64)()
    n = ctypes.c_int32(0)
    lib.sattn_profile_collect(names, launches, total, 64, ctypes.byref(n))
    out = {}
    for x in range(n.value):
        nm = names.raw[32 * x: 32 * x + 32].split(b"\0")[0].decode()
        out[nm] = (int(launches[x]), float(total[x]))
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    import long_context_structured_b200 as sa
    from long_context_structured_b200 import _lib

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        log("note: --gpus %d but WORLD_SIZE %d; using WORLD_SIZE" % (args.gpus, world))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    wl = synth.WORKLOADS[WORKLOAD]
    if args.heads:
        wl = wl.scaled(Hq=args.heads, Hkv=args.heads)
    pairs_head = unmasked_pairs_per_head(wl)
    pairs = pairs_head * wl.B * wl.Hq
    flops_step = 4.0 * wl.d * pairs  # per rank
    inp = synth.make_inputs(wl, seed=rank)
    to_t = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    qh, kh, vh = (to_t(inp[x]).pin_memory() for x in ("q", "k", "v"))
    q, k, v = qh.to(dev), kh.to(dev), vh.to(dev)
    kw = dict(n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain, rope_theta=wl.rope_theta)
    O = torch.empty_like(q)
    lse = torch.empty((wl.B, wl.Hq, wl.T), dtype=torch.float32, device=dev)
    lib = _lib.load()

    for _ in range(args.warmup):
        sa.fwd(q, k, v, out=O, lse=lse, **kw)
    torch.cuda.synchronize()
    if sa.stream_status() != 0:
        raise RuntimeError("device status word reports a failure after warm-up")

    gpu_uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    phys = int(vis.split(",")[local]) if vis and vis.split(",")[local].strip().isdigit() else local
    clocks = ClockSampler(gpu_uuid, phys)
    clocks.start()
    time.sleep(0.3)
    profile_collect(lib)  # drop anything recorded before
    lib.sattn_profile_enable(1)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        sa.fwd(q, k, v, out=O, lse=lse, **kw)
    e1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    lib.sattn_profile_enable(0)
    clk = clocks.stop()
    elapsed_ms = e0.elapsed_time(e1)
    prof = profile_collect(lib)
    status = sa.stream_status()

    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_step = float(t.item()) / args.steps
    value = flops_step * world / (ms_step * 1e-3) / 1e12
    tokens_s = wl.B * wl.T * world / (ms_step * 1e-3)

    attn_launches, attn_ms = prof.get("attn_tc", (0, 0.0))
    attn_avg_ms = attn_ms / max(attn_launches, 1)
    at = torch.tensor([attn_avg_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(at, op=dist.ReduceOp.MAX)
    attn_avg_ms = float(at.item())
    peaks, peak_src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    achieved = flops_step / (attn_avg_ms * 1e-3) / 1e12 if attn_avg_ms > 0 else None
    gpu_launches = sum(n for n, _ in prof.values())

    # end to end through the public call with host buffers (H2D + D2H inside)
    e2e = None
    if rank == 0 or world > 1:
        n_e2e = max(3, min(10, args.steps))
        sa.fwd(qh, kh, vh, **kw)  # warm the host path
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record()
        for _ in range(n_e2e):
            Oh, lh = sa.fwd(qh, kh, vh, **kw)
        s1.record()
        torch.cuda.synchronize()
        te = torch.tensor([s0.elapsed_time(s1) / n_e2e], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(te, op=dist.ReduceOp.MAX)
        ms_e2e = float(te.item())
        e2e = {"value": round(flops_step * world / (ms_e2e * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
               "ms_per_step": round(ms_e2e, 3), "steps": n_e2e,
               "h2d_bytes_per_step": int(qh.nbytes + kh.nbytes + vh.nbytes),
               "d2h_bytes_per_step": int(Oh.nbytes + lh.nbytes),
               "path": "long_context_structured_b200.fwd on pinned host tensors"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, inp, args.cpu_rows)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1); keys 0-3 x8)",
        "config": config_dict(wl, pairs),
        "tokens_per_s": round(tokens_s, 1),
        "frac_of_bf16_peak": round(value / world / peak, 4),
        "roofline": {
            "kernel": "attn_tc2_kernel<128>", "bound": "tensor",
            "achieved": None if achieved is None else round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": None if achieved is None else round(achieved / peak, 4),
            "traffic": ATTN_TRAFFIC_BYTES,
            "peak_source": "%s bf16_tflops (burst)" % peak_src,
            "frac_of_sustained": None if achieved is None else round(achieved / float(peaks.get(
                "bf16_tflops_sustained", peak)), 4),
            "avg_launch_ms": round(attn_avg_ms, 4), "algorithmic_flops_per_launch": flops_step,
        },
        "kernels": {k: {"launches": n, "avg_ms": round(ms / max(n, 1), 5)} for k, (n, ms) in prof.items()},
        "gpu_launches": gpu_launches,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "clocks": clk,
        "device_status": status,
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# ---------------------------------------------------------------------------

def _oracle_sample(wl, n_rows, seed):
    """Rows spread over all heads and positions, seeded."""
    rng = np.random.default_rng(seed)
    heads = rng.integers(0, wl.Hq, n_rows)
    pos = rng.integers(0, wl.T, n_rows)
    return np.stack([np.zeros(n_rows, np.int64), heads, pos], axis=1)


def _pairs_of_rows(wl, rows):
    i = rows[:, 2]
    return int(np.minimum(i + 1, wl.n_start + wl.window + 1).sum())


def cpu_baseline(wl, inp, n_rows):
    from oracle import oracle as O
    O.build()
    p = O.params_of(wl)
    rows = _oracle_sample(wl, n_rows, 1234)
    nthreads = O.nthreads_default()
    t0 = time.perf_counter()
    O.fwd_rows(p, inp["q"], inp["k"], inp["v"], None, rows, nthreads=nthreads)
    dt = time.perf_counter() - t0
    flops = 4.0 * wl.d * _pairs_of_rows(wl, rows)
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": nthreads, "kind": "oracle",
            "sample": "%d seeded rows (b, h, i) of the same workload, all heads, fp64, %.1f s" % (n_rows, dt),
            "seconds": round(dt, 2)}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import oracle as O
    O.build()
    wl = synth.WORKLOADS[WORKLOAD]
    inp = synth.make_inputs(wl, seed=0)
    p = O.params_of(wl)
    nthreads = O.nthreads_default()
    rows_per_step = args.ref_rows

    def step(s):
        # one head per step, rows spread over positions
        rows = _oracle_sample(wl, rows_per_step, 100 + s)
        rows[:, 1] = s % wl.Hq
        O.fwd_rows(p, inp["q"], inp["k"], inp["v"], None, rows, nthreads=nthreads)
        return _pairs_of_rows(wl, rows)

    for s in range(args.warmup):
        step(s)
    t0 = time.perf_counter()
    pairs = 0
    for s in range(args.steps):
        pairs += step(args.warmup + s)
    dt = time.perf_counter() - t0
    value = 4.0 * wl.d * pairs / dt / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1); keys 0-3 x8)",
        "config": config_dict(wl, unmasked_pairs_per_head(wl) * wl.B * wl.Hq),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": nthreads, "kind": "oracle",
                         "sample": "each step: %d seeded rows of one head (heads cycle), fp64 C oracle"
                                   % rows_per_step},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-rows", type=int, default=8192, help="rows in the CPU-oracle baseline sample")
    ap.add_argument("--ref-rows", type=int, default=32, help="rows per step of the reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--heads", type=int, default=0, help="override the head count (profiling captures only)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
