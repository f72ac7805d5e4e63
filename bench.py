"""Benchmark of the structured-mask attention hot path on B200.

One step = one call of the whole hot path over one batch of synthetic input
(rotary prep, block map / separator gather / top-k selection where the
workload has them, and the tcgen05 attention kernel).  The default workload is
the largest single-GPU configuration: the LM-Infinite layer with per-head
top-k middle tokens, B=1, 32 heads, T=32768, d=128, bf16, n_start=4,
L_pretrain=w=4096, capped RoPE theta=1e4, k=5 with 64 planted key/query
clusters per head.  ``--workload`` selects one of the other workloads (the
16K LM-Infinite layer, the SepLLM GQA layer, segmented execution, decoding,
backward, ...) to measure their kernels the same way.
Metric: effective TFLOP/s counted over unmasked (q, k) pairs at 4*d FLOPs
each (whole job, all ranks), with tokens/s alongside.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload c2|c3|c4|c5]

Multi-GPU: one process per GPU (torchrun).  By default every rank runs its
own independent problem (heads/batches are independent), so per-GPU work is
fixed as N grows ("scaling": "weak") and no data-path collective exists;
the only collectives are the barrier and the max-over-ranks of the timings.
``--split heads`` instead splits ONE layer over the ranks by kv-head groups
("scaling": "strong"): each rank computes its heads' block, and the blocks
are all-gathered once after the timed steps (NCCL; its time reported apart
as ``head_gather``).

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

# decoding steps (one new token per sequence) over the caches of these workloads
DECODE_ALIASES = {"c2d": "c2_lminf_16k", "c3d": "c3_sepllm_gqa_8k", "c4d": "c4_lminf_topk_32k"}
BWD_ALIASES = {"c2b": "c2_lminf_16k", "c3b": "c3_sepllm_gqa_8k"}
# stress sizes for the HBM-bound helpers: the block map on B*T = 2^26 flags
# (a2s) and the separator gather on the SepLLM layer at 16x its batch (c3x16)
STRESS_ALIASES = {"a2s": "blockmap_stress_2e26"}
EXTRA_WORKLOADS = {"c3x16": ("c3_sepllm_gqa_8k", dict(name="c3_sepllm_gqa_8k_x16", B=64))}
STREAM_ALIASES = {"c3s": "stream_sepllm_gqa"}
# SepLLM streaming generation: 16 sequences of the Llama-3-8B-shaped layer
# (32 query / 8 kv heads, d = 128) with a 4096-slot cache (a = 4 initial,
# s = 1024 separator, w = 2048 local slots), separators at rate 0.1
STREAM_WORKLOADS = {"stream_sepllm_gqa": dict(B=16, Hq=32, Hkv=8, d=128, a=4, s=1024, w=2048, c=4096, rate=0.1,
                                              rope_theta=5e5, warm_tokens=6144)}
TREE_ALIASES = {"c6t": "tree_cross_128k"}
# SharedLLM tree cross-attention: a 128K-token context in 64 chunks of 2048,
# depth 3, leaf rate 2 (global compression 4), 4096 decoder queries
TREE_WORKLOADS = {"tree_cross_128k": dict(B=1, Hq=32, Hkv=32, Tq=4096, d=128, n_chunks=64, chunk_len=2048,
                                          depth=3, alpha_leaf=2, rope_theta=1e4)}
BWD_FLOPS_PER_PAIR_D = 10  # backward: S recomputed, dP, dV, dK, dQ -- five products of 2d FLOPs per pair
WORKLOAD_ALIASES = {"c2": "c2_lminf_16k", "c3": "c3_sepllm_gqa_8k", "c4": "c4_lminf_topk_32k",
                    "c5": "c5_segmented_32k"}
DEFAULT_WORKLOAD = "c4"
METRIC = "effective TFLOP/s over unmasked pairs (fraction of bf16 TC peak), tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (read + write) per launch of the dominant kernel of the default
# workload (topk_score_kernel): dram__bytes_read.sum + dram__bytes_write.sum of
# an ncu capture of the 4-head cut, times 8 for 32 heads (the launch is a grid
# over heads and every head reads and writes the same amount); None when the
# kernel changed since the counters were taken.
TOPK_SCORE_TRAFFIC_BYTES = (61482752 + 13227264) * 8
# CPU-oracle rows per sample (about 10-30 s of host work on the GPU machine); the
# top-k workload's oracle also scans every middle key per row
CPU_ROWS = {"c4": 6144}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ---------------------------------------------------------------------------
# algorithmic work per workload (closed-form counts of kept (q, k) pairs)
# ---------------------------------------------------------------------------

def lambda_pairs_per_row(wl) -> np.ndarray:
    """Kept keys of each row from the starting span and the window: row i
    keeps min(i+1, n_start+w+1) keys."""
    i = np.arange(wl.T, dtype=np.int64)
    return np.minimum(i + 1, wl.n_start + wl.window + 1)


def middle_candidates_per_row(wl) -> np.ndarray:
    """Middle keys n_start <= j < i - w of each row (no separators)."""
    i = np.arange(wl.T, dtype=np.int64)
    return np.maximum(0, i - wl.window - wl.n_start)


def unmasked_pairs(wl, is_sep=None) -> int:
    """Kept (q, k) pairs summed over batch and heads for one workload."""
    if wl.segmented:
        S, N = wl.seg_S, wl.T // wl.seg_S
        t = np.arange(S, dtype=np.int64) + 1
        per_local = N * int(t.sum()) + (N - 1) * S * wl.seg_M
        per_long = N * int(t.sum()) + (N - 1) * S * wl.seg_R
        n_long = len(wl.long_heads)
        return wl.B * ((wl.Hq - n_long) * per_local + n_long * per_long)
    base = lambda_pairs_per_row(wl)
    per_head = np.full(wl.B, int(base.sum()), dtype=np.int64)
    if is_sep is not None:
        i = np.arange(wl.T, dtype=np.int64)
        for b in range(wl.B):
            f = is_sep[b].astype(np.int64).copy()
            f[: wl.n_start] = 0
            pre = np.concatenate([[0], np.cumsum(f)])  # pre[x] = separators n_start <= j < x
            per_head[b] += int(pre[np.clip(i - wl.window, 0, wl.T)].sum())
    if wl.topk > 0:
        per_head += int(np.minimum(wl.topk, middle_candidates_per_row(wl)).sum())
    return int(per_head.sum()) * wl.Hq


def scored_candidates(wl) -> int:
    """Middle (q, k) pairs the top-k selector scores (2*d FLOPs each)."""
    if wl.topk <= 0:
        return 0
    return int(middle_candidates_per_row(wl).sum()) * wl.B * wl.Hq


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def describe(wl) -> str:
    if wl.segmented:
        return ("%s: segmented execution, one layer, B=%d H=%d (%d long) T=%d d=%d bf16, S=%d, tail M=%d, "
                "prefix R=%d (top-%d blocks of %d), RoPE theta=%g" % (
                    wl.name, wl.B, wl.Hq, len(wl.long_heads), wl.T, wl.d, wl.seg_S, wl.seg_M, wl.seg_R,
                    wl.seg_R // wl.retr_block, wl.retr_block, wl.rope_theta))
    if wl.sep_rate > 0:
        return ("%s: SepLLM layer, B=%d Hq=%d Hkv=%d T=%d d=%d bf16, separator ids %d of %d at rate %.2f, "
                "n_start=%d, w=%d, RoPE theta=%g" % (wl.name, wl.B, wl.Hq, wl.Hkv, wl.T, wl.d, wl.sep_ids,
                                                     wl.sep_vocab, wl.sep_rate, wl.n_start, wl.window,
                                                     wl.rope_theta))
    s = ("%s: LM-Infinite Lambda-mask layer, B=%d H=%d T=%d d=%d bf16, n_start=%d, L_pretrain=w=%d, "
         "capped RoPE theta=%g" % (wl.name, wl.B, wl.Hq, wl.T, wl.d, wl.n_start, wl.window, wl.rope_theta))
    if wl.sink_scale != 1.0:
        s += ", keys 0-3 x%g" % wl.sink_scale
    if wl.topk > 0:
        s += ", top-%d middle keys per head (%d planted clusters)" % (wl.topk, wl.plant)
    return s


def config_dict(wl, pairs_per_rank, decode=False, n_copies=0, backward=False, parallelism="dp1"):
    prefix = ("decoding step (one new token per sequence at position T-1) over the cache of " if decode else
              "backward pass (dQ, dK, dV of sum(dO*O); %d FLOPs per kept pair per d) of " % BWD_FLOPS_PER_PAIR_D
              if backward else "")
    c = {"workload": prefix + describe(wl), "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "T": wl.T, "d": wl.d}
    if wl.segmented:
        c.update({"S": wl.seg_S, "M": wl.seg_M, "R": wl.seg_R, "retr_block": wl.retr_block,
                  "long_heads": len(wl.long_heads), "rope_theta": wl.rope_theta})
    else:
        c.update({"n_start": wl.n_start, "window": wl.window, "L_pretrain": wl.L_pretrain,
                  "rope_theta": wl.rope_theta, "topk": wl.topk})
    c["unmasked_pairs_per_rank"] = pairs_per_rank
    c["parallelism"] = parallelism
    in_bytes = (wl.B * wl.Hq + 2 * wl.B * wl.Hkv) * wl.T * wl.d * 2
    if decode:
        c["l2"] = ("no flush: steps cycle through %d copies of the K/V cache, so successive steps read "
                   "more than the 126 MB L2 holds" % n_copies)
    else:
        c["l2"] = ("no flush: each step reads Q,K,V (%d MB) and writes their rotated copies, > 126 MB L2"
                   % (in_bytes >> 20))
    return c


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
# one workload: inputs, the step, the end-to-end call, algorithmic work
# ---------------------------------------------------------------------------

class Job:
    """Inputs of one workload on one rank (pinned host copies and device
    copies) and the hot-path call over them."""

    def __init__(self, wl, seed, dev, heads=None):
        import torch

        import long_context_structured_b200 as sa
        inp = synth.make_inputs(wl, seed=seed)
        self.full_wl, self.full_inp = wl, inp
        if heads is not None:
            # this rank's block of one layer: query heads [q0, q1) and the kv
            # heads [kv0, kv1) they read, cut from the full layer's inputs
            q0, q1, kv0, kv1 = heads
            cut = lambda a, lo, hi: np.ascontiguousarray(a[:, lo:hi])
            inp = dict(inp, q=cut(inp["q"], q0, q1), k=cut(inp["k"], kv0, kv1), v=cut(inp["v"], kv0, kv1))
            wl = wl.scaled(Hq=q1 - q0, Hkv=kv1 - kv0)
        self.sa, self.torch, self.wl, self.dev = sa, torch, wl, dev
        self.inp = inp
        to_t = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
        self.host = {x: to_t(inp[x]).pin_memory() for x in ("q", "k", "v")}
        if inp["is_sep"] is not None:
            self.host["is_sep"] = torch.from_numpy(inp["is_sep"]).pin_memory()
        self.devt = {x: t.to(dev) for x, t in self.host.items()}
        q = self.devt["q"]
        self.O = torch.empty_like(q)
        self.lse = torch.empty((wl.B, wl.Hq, wl.T), dtype=torch.float32, device=dev)
        if wl.segmented:
            self.kw = dict(S=wl.seg_S, M=wl.seg_M, R=wl.seg_R, retr_block=wl.retr_block,
                           is_long=[int(x) for x in inp["is_long"]], rope_theta=wl.rope_theta)
        else:
            self.kw = dict(n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain,
                           rope_theta=wl.rope_theta, topk=wl.topk)
        self.pairs = unmasked_pairs(wl, inp["is_sep"])
        self.flops = 4.0 * wl.d * self.pairs
        self.full_flops = 4.0 * wl.d * unmasked_pairs(self.full_wl, inp["is_sep"]) if heads is not None else None
        self.n_sep = 0 if inp["is_sep"] is None else int(inp["is_sep"][:, wl.n_start:].sum())

    def step(self):
        d = self.devt
        if self.wl.segmented:
            self.sa.segment_fwd(d["q"], d["k"], d["v"], out=self.O, lse=self.lse, **self.kw)
        else:
            self.sa.fwd(d["q"], d["k"], d["v"], is_sep=d.get("is_sep"), out=self.O, lse=self.lse, **self.kw)

    def host_step(self):
        """The public call on pinned host tensors: H2D, the hot path, D2H."""
        h = self.host
        if self.wl.segmented:
            return self.sa.segment_fwd(h["q"], h["k"], h["v"], **self.kw)
        return self.sa.fwd(h["q"], h["k"], h["v"], is_sep=h.get("is_sep"), **self.kw)

    def h2d_bytes(self):
        return int(sum(t.nbytes for t in self.host.values()))

    # algorithmic work of each launch group the library times ---------------
    def group_work(self):
        """{group: (bound, work per launch, unit)} for the groups whose
        algorithmic work has a closed form: FLOPs for the tensor-core kernels,
        bytes read + written of the named arrays for the HBM-bound ones."""
        wl = self.wl
        e = 2  # bf16 bytes
        rows_q = wl.B * wl.Hq * wl.T * wl.d * e
        rows_k = wl.B * wl.Hkv * wl.T * wl.d * e
        out = {}
        attn = "attn_tc_segment" if wl.segmented else "attn_tc"
        out[attn] = ("tensor", self.flops, "FLOP")
        prep = 2 * rows_q + 2 * rows_k  # Q, K read; Qr, Kr written
        if not wl.segmented:
            if wl.L_pretrain > 0 and (wl.topk > 0 or wl.sep_rate > 0):
                prep += rows_q  # Qc written
            prep += wl.B * wl.Hq * wl.T * min(wl.n_start, wl.T) * 4  # sink logits written
        out["prep_rope"] = ("hbm", prep, "B")
        if self.n_sep:
            out["sep_gather"] = ("hbm", self.n_sep * wl.Hkv * 4 * wl.d * e, "B")
        if wl.topk > 0:
            out["topk_score"] = ("tensor", 2.0 * wl.d * scored_candidates(wl), "FLOP")
        return out


def decode_keys(wl, is_sep) -> np.ndarray:
    """Kept keys of the last position i = T-1 per sequence (sinks, window,
    earlier separators)."""
    i = wl.T - 1
    n = min(wl.n_start, wl.T) + max(0, i - max(min(wl.n_start, wl.T), i - wl.window) + 1)
    out = np.full(wl.B, n, dtype=np.int64)
    if is_sep is not None:
        for b in range(wl.B):
            f = is_sep[b].astype(np.int64).copy()
            f[: wl.n_start] = 0
            out[b] += int(f[: max(0, i - wl.window)].sum())
    return out


class DecodeJob:
    """One decoding step per sequence over a workload's cache: the query of
    position T-1 against the structured key set of that position.  Several
    copies of the cache are cycled through so that successive steps read
    more than the L2 cache holds."""

    L2_BYTES = 126 * 2 ** 20

    def __init__(self, wl, seed, dev):
        import torch

        import long_context_structured_b200 as sa
        self.sa, self.torch, self.wl, self.dev = sa, torch, wl, dev
        inp = synth.make_inputs(wl, seed=seed)
        self.inp = inp
        to_t = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
        q = to_t(inp["q"])[:, :, wl.T - 1:wl.T, :].contiguous()
        self.host = {"q": q.pin_memory()}
        keys = decode_keys(wl, inp["is_sep"])
        self.kv_bytes = int(keys.sum()) * wl.Hkv * 2 * wl.d * 2  # kept K and V rows read per step
        self.n_copies = int(min(8, max(1, -(-2 * self.L2_BYTES // max(self.kv_bytes, 1)))))
        k, v = to_t(inp["k"]).to(dev), to_t(inp["v"]).to(dev)
        self.caches = [(k, v)] + [(k.clone(), v.clone()) for _ in range(self.n_copies - 1)]
        self.sep = None if inp["is_sep"] is None else torch.from_numpy(inp["is_sep"]).to(dev)
        self.qd = self.host["q"].to(dev)
        self.O = torch.empty_like(self.qd)
        self.lse = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device=dev)
        self.kw = dict(n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain, rope_theta=wl.rope_theta,
                       topk=wl.topk)
        self.pairs = int(keys.sum()) * wl.Hq
        if wl.topk > 0:
            # top-k: every middle candidate's K row is scored (read once per
            # kv group), and k more kept keys per head
            ncand = max(0, wl.T - 1 - wl.window - wl.n_start)
            self.kv_bytes += wl.B * wl.Hkv * ncand * wl.d * 2
            self.pairs += wl.B * wl.Hq * min(wl.topk, ncand)
        self.flops = 4.0 * wl.d * self.pairs
        self.n_step = 0

    def step(self):
        k, v = self.caches[self.n_step % self.n_copies]
        self.n_step += 1
        self.sa.decode_fwd(self.qd, k, v, is_sep=self.sep, out=self.O, lse=self.lse, **self.kw)

    def capture(self):
        """One CUDA graph per cache copy holding a whole step (block map,
        top-k and split-K kernels), as a generation loop replays it: a step
        of tens of microseconds is otherwise timed at the speed of the
        host's Python call path."""
        torch = self.torch
        side = torch.cuda.Stream(self.dev)
        side.wait_stream(torch.cuda.current_stream(self.dev))
        with torch.cuda.stream(side):
            for _ in range(self.n_copies):
                self.step()
        torch.cuda.current_stream(self.dev).wait_stream(side)
        torch.cuda.synchronize(self.dev)
        self.graphs = []
        for c in range(self.n_copies):
            g = torch.cuda.CUDAGraph()
            self.n_step = c
            with torch.cuda.graph(g):
                self.step()
            self.graphs.append(g)
        self.n_step = 0

    def graph_step(self):
        self.graphs[self.n_step % self.n_copies].replay()
        self.n_step += 1

    def host_step(self):
        """The query from pinned host memory, the step on the device-resident
        cache, O and LSE back to pinned host memory."""
        torch = self.torch
        qd = self.host["q"].to(self.dev, non_blocking=True)
        k, v = self.caches[0]
        O, lse = self.sa.decode_fwd(qd, k, v, is_sep=self.sep, **self.kw)
        oh = torch.empty(O.shape, dtype=O.dtype, pin_memory=True)
        lh = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        oh.copy_(O, non_blocking=True)
        lh.copy_(lse, non_blocking=True)
        torch.cuda.current_stream(self.dev).synchronize()
        return oh, lh

    def h2d_bytes(self):
        return int(self.host["q"].nbytes)

    def group_work(self):
        wl = self.wl
        q_o = 2 * wl.B * wl.Hq * wl.d * 2
        return {"decode": ("hbm", self.kv_bytes + q_o, "B")}


def sink_pairs(wl) -> int:
    """(q, k) pairs with k in the starting span j < n_start (fp32 side keys)."""
    i = np.arange(wl.T, dtype=np.int64)
    return int(np.minimum(min(wl.n_start, wl.T), i + 1).sum()) * wl.B * wl.Hq


class BwdJob:
    """One backward step of a workload: the forward's O and LSE and a seeded
    dO are resident; each step computes dQ, dK, dV through sattn_bwd."""

    def __init__(self, wl, seed, dev):
        import torch

        import long_context_structured_b200 as sa
        self.sa, self.torch, self.wl, self.dev = sa, torch, wl, dev
        inp = synth.make_inputs(wl, seed=seed)
        self.inp = inp
        f32 = wl.dtype == "f32"
        to_t = (lambda a: torch.from_numpy(a)) if f32 else \
            (lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16))
        self.host = {x: to_t(inp[x]).pin_memory() for x in ("q", "k", "v")}
        g = np.random.default_rng(seed + 7)
        do = g.standard_normal(inp["q"].shape).astype(np.float32)
        self.host["do"] = (torch.from_numpy(do) if f32 else torch.from_numpy(do).to(torch.bfloat16)).pin_memory()
        if inp["is_sep"] is not None:
            self.host["is_sep"] = torch.from_numpy(inp["is_sep"]).pin_memory()
        self.devt = {x: t.to(dev) for x, t in self.host.items()}
        d = self.devt
        self.kw = dict(n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain, rope_theta=wl.rope_theta)
        self.O, self.lse = sa.fwd(d["q"], d["k"], d["v"], is_sep=d.get("is_sep"), **self.kw)
        torch.cuda.synchronize()
        self.host["o"] = self.O.cpu().pin_memory()
        self.host["lse"] = self.lse.cpu().pin_memory()
        self.grads = (torch.empty_like(d["q"]), torch.empty_like(d["k"]), torch.empty_like(d["v"]))
        self.pairs = unmasked_pairs(wl, inp["is_sep"])
        self.tc_pairs = self.pairs - sink_pairs(wl)
        self.flops = float(BWD_FLOPS_PER_PAIR_D) * wl.d * self.pairs
        self.n_sep = 0 if inp["is_sep"] is None else int(inp["is_sep"][:, wl.n_start:].sum())

    def step(self):
        d = self.devt
        self.sa.bwd(d["q"], d["k"], d["v"], self.O, self.lse, d["do"], is_sep=d.get("is_sep"), grads=self.grads,
                    **self.kw)

    def host_step(self):
        """Inputs from pinned host memory, the backward call, the gradients
        back into pinned host memory."""
        torch = self.torch
        h = self.host
        dv = {x: t.to(self.dev, non_blocking=True) for x, t in h.items()}
        grads = self.sa.bwd(dv["q"], dv["k"], dv["v"], dv["o"], dv["lse"], dv["do"], is_sep=dv.get("is_sep"),
                            **self.kw)
        outs = []
        for t in grads:
            o = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
            o.copy_(t, non_blocking=True)
            outs.append(o)
        torch.cuda.current_stream(self.dev).synchronize()
        return outs

    def h2d_bytes(self):
        return int(sum(t.nbytes for t in self.host.values()))

    def group_work(self):
        wl = self.wl
        if wl.dtype == "f32":
            return {"bwd_f32": ("tensor", self.flops, "FLOP")}
        e = 2
        rows_q = wl.B * wl.Hq * wl.T * wl.d * e
        rows_k = wl.B * wl.Hkv * wl.T * wl.d * e
        out = {"bwd_dq": ("tensor", 6.0 * wl.d * self.tc_pairs, "FLOP"),      # S, dP, dQ
               "bwd_dkv": ("tensor", 8.0 * wl.d * self.tc_pairs, "FLOP"),     # S^T, dP^T, dV, dK
               # O, dO read; D and -LSE written; with sinks also dq_side (fp32) and per-pair P, dS
               "bwd_rows": ("hbm", 2 * rows_q + 8 * wl.B * wl.Hq * wl.T + (
                   2 * rows_q + 8 * min(wl.n_start, wl.T) * wl.B * wl.Hq * wl.T if wl.n_start else 0), "B"),
               # fp32 band dk/dv read, bf16 dk/dv written (separator and sink parts are small)
               "bwd_combine": ("hbm", 2 * rows_k * 2 + 2 * rows_k, "B")}
        if wl.n_start:  # Q and dO read, P and dS of the sink pairs read
            out["bwd_sink_keys"] = ("hbm", 2 * rows_q + 8 * min(wl.n_start, wl.T) * wl.B * wl.Hq * wl.T, "B")
        prep = 2 * rows_q + 2 * rows_k + wl.B * wl.Hq * wl.T * min(wl.n_start, wl.T) * 4
        if wl.L_pretrain > 0 and wl.sep_rate > 0:
            prep += rows_q
        out["prep_rope"] = ("hbm", prep, "B")
        return out


class TreeJob:
    """SharedLLM tree cross-attention over a compressed long context: the
    decoder queries against the kept rows of every context chunk."""

    def __init__(self, cfg, seed, dev):
        import torch

        import long_context_structured_b200 as sa
        self.sa, self.torch, self.cfg, self.dev = sa, torch, cfg, dev
        c = cfg
        g = torch.Generator().manual_seed(seed)
        Tc = c["n_chunks"] * c["chunk_len"]
        self.host = {"q": torch.randn(c["B"], c["Hq"], c["Tq"], c["d"], generator=g).bfloat16().pin_memory(),
                     "k": torch.randn(c["B"], c["Hkv"], Tc, c["d"], generator=g).bfloat16().pin_memory(),
                     "v": torch.randn(c["B"], c["Hkv"], Tc, c["d"], generator=g).bfloat16().pin_memory()}
        self.devt = {x: t.to(dev) for x, t in self.host.items()}
        self.kw = dict(n_chunks=c["n_chunks"], chunk_len=c["chunk_len"], depth=c["depth"],
                       alpha_leaf=c["alpha_leaf"], rope_theta=c["rope_theta"])
        self.O = torch.empty_like(self.devt["q"])
        self.lse = torch.empty(c["B"], c["Hq"], c["Tq"], dtype=torch.float32, device=dev)
        # the kept rows per chunk, as the library reports them
        _, _, idx = sa.tree_cross_fwd(self.devt["q"], self.devt["k"], self.devt["v"], with_index=True, **self.kw)
        self.n_kept = int((idx >= 0).sum().item())
        self.S = c["n_chunks"] * self.n_kept
        self.pairs = c["B"] * c["Hq"] * c["Tq"] * self.S
        self.flops = 4.0 * c["d"] * self.pairs

    def step(self):
        d = self.devt
        self.sa.tree_cross_fwd(d["q"], d["k"], d["v"], out=self.O, lse=self.lse, **self.kw)

    def host_step(self):
        h = self.host
        dv = {x: t.to(self.dev, non_blocking=True) for x, t in h.items()}
        O, lse = self.sa.tree_cross_fwd(dv["q"], dv["k"], dv["v"], **self.kw)
        oh = self.torch.empty(O.shape, dtype=O.dtype, pin_memory=True)
        lh = self.torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        oh.copy_(O, non_blocking=True)
        lh.copy_(lse, non_blocking=True)
        self.torch.cuda.current_stream(self.dev).synchronize()
        return oh, lh

    def h2d_bytes(self):
        return int(sum(t.nbytes for t in self.host.values()))

    def group_work(self):
        c = self.cfg
        rows_q = c["B"] * c["Hq"] * c["Tq"] * c["d"] * 2
        kept = c["B"] * c["Hkv"] * self.S * c["d"] * 2
        return {"attn_tc_cross": ("tensor", self.flops, "FLOP"),
                "tree_prep": ("hbm", 2 * rows_q + 4 * kept, "B")}


class StreamJob:
    """Streaming generation over SepLLM's four-part cache: each step appends
    one token per sequence (compacting on the device when full) and decodes
    its query over the cache.  The cache is warmed past several compactions
    first; steps cycle through precomputed token rows."""

    def __init__(self, cfg, seed, dev):
        import torch

        import long_context_structured_b200 as sa
        self.sa, self.torch, self.cfg, self.dev = sa, torch, cfg, dev
        c = cfg
        g = torch.Generator().manual_seed(seed)
        self.n_rows = 64
        self.k = torch.randn(self.n_rows, c["B"], c["Hkv"], c["d"], generator=g).bfloat16().to(dev)
        self.v = torch.randn(self.n_rows, c["B"], c["Hkv"], c["d"], generator=g).bfloat16().to(dev)
        self.q = torch.randn(self.n_rows, c["B"], c["Hq"], 1, c["d"], generator=g).bfloat16().to(dev)
        self.sep = (torch.rand(self.n_rows, c["B"], generator=g) < c["rate"]).to(torch.uint8).to(dev)
        self.cache = sa.StreamKV(c["B"], c["Hkv"], c["d"], c["a"], c["s"], c["w"], c["c"], device=dev)
        self.O = torch.empty(c["B"], c["Hq"], 1, c["d"], dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(c["B"], c["Hq"], dtype=torch.float32, device=dev)
        self.t = 0
        for _ in range(c["warm_tokens"]):
            self.append_only()
        torch.cuda.synchronize()
        sizes, _ = self.cache.read()
        self.len = sizes.sum(axis=1)

    def append_only(self):
        r = self.t % self.n_rows
        self.cache.append(self.k[r], self.v[r], self.sep[r])
        self.t += 1

    def step(self):
        r = self.t % self.n_rows
        self.append_only()
        self.cache.decode(self.q[r], rope_theta=self.cfg["rope_theta"], out=self.O, lse=self.lse)

    def mean_len(self):
        sizes, _ = self.cache.read()
        return float(sizes.sum(axis=1).mean())


def cpu_baseline_tree(cfg, n_rows=256):
    from oracle import oracle as O
    O.build()
    import torch
    c = cfg
    g = torch.Generator().manual_seed(0)
    bits = lambda t: t.bfloat16().view(torch.int16).numpy().view(np.uint16)
    Tc = c["n_chunks"] * c["chunk_len"]
    q = bits(torch.randn(1, 1, n_rows, c["d"], generator=g))
    k = bits(torch.randn(1, 1, Tc, c["d"], generator=g))
    v = bits(torch.randn(1, 1, Tc, c["d"], generator=g))
    p = O.params(1, 1, 1, n_rows, c["d"], "bf16", rope_theta=c["rope_theta"])
    nthreads = O.nthreads_default()
    t0 = time.perf_counter()
    O.tree_cross(p, c["n_chunks"], c["chunk_len"], c["depth"], c["alpha_leaf"], q, k, v, nthreads=nthreads)
    dt = time.perf_counter() - t0
    S = c["n_chunks"] * len(O.tree_index(c["chunk_len"], c["depth"], c["alpha_leaf"]))
    return {"value": round(4.0 * c["d"] * n_rows * S / dt / 1e12, 6), "unit": "TFLOP/s", "cores": nthreads,
            "kind": "oracle", "sample": "%d query rows of one head against all %d kept context rows, fp64, %.1f s"
            % (n_rows, S, dt), "seconds": round(dt, 2)}


def roofline_of(group, work, avg_ms, peaks, peak_src):
    bound, amount, unit = work
    if bound == "tensor":
        peak = float(peaks["bf16_tflops"])
        ach = amount / (avg_ms * 1e-3) / 1e12
        r = {"kernel": group, "bound": "tensor", "achieved": round(ach, 2), "peak": peak, "unit": "TFLOP/s",
             "frac": round(ach / peak, 4), "peak_source": "%s bf16_tflops (burst)" % peak_src,
             "frac_of_sustained": round(ach / float(peaks.get("bf16_tflops_sustained", peak)), 4),
             "algorithmic_flops_per_launch": amount}
    else:
        peak = float(peaks["hbm_gbs"])
        ach = amount / (avg_ms * 1e-3) / 1e9
        r = {"kernel": group, "bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
             "frac": round(ach / peak, 4), "peak_source": "%s hbm_gbs" % peak_src,
             "algorithmic_bytes_per_launch": amount}
    r["avg_launch_ms"] = round(avg_ms, 4)
    return r


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


def kernel_name(wl, group):
    """The kernel behind a launch group on this workload (for the JSON line)."""
    if group == "attn_tc":
        capped_sep = wl.L_pretrain > 0 and wl.sep_rate > 0
        return "attn_tc3_kernel<%d>" % wl.d if capped_sep else "attn_tc2_kernel<%d>" % wl.d
    if group == "attn_tc_segment":
        return "attn_tc2_kernel<%d>" % wl.d if wl.seg_S % 256 == 0 else "attn_tc3_kernel<%d>" % wl.d
    if group == "attn_tc_cross":
        return "attn_tc2_kernel<%d>" % TREE_WORKLOADS["tree_cross_128k"]["d"]
    d = wl.d if wl is not None else 128
    if group == "decode" and wl is not None and wl.topk > 0:
        return "decode_topk_logits_kernel + decode_topk_select_kernel + decode_partial_kernel + decode_combine_kernel"
    return {"prep_rope": "prep_kernel", "topk_score": "topk_score_kernel<%d>" % d, "topk_rerank": "topk_rerank_kernel<%d>" % d, "tree_prep": "tree_prep_kernel",
            "decode": "decode_partial_kernel + decode_combine_kernel",
            "sep_gather": "sep_gather_kernel", "bwd_dq": "bwd_dq_kernel<%d>" % d,
            "bwd_dkv": "bwd_dkv_kernel<%d>" % d, "bwd_f32": "bwd_f32_dq_kernel + bwd_f32_dkv_kernel",
            "bwd_rows": "bwd_rows_kernel", "bwd_combine": "bwd_combine_kernel",
            "bwd_sink_keys": "bwd_sink_keys_kernel"}.get(group, group)


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

    decode = args.workload in DECODE_ALIASES
    backward = args.workload in BWD_ALIASES
    tree = args.workload in TREE_ALIASES
    if tree:
        return run_tree(args, world, rank, dev)
    if args.workload in STREAM_ALIASES:
        return run_stream(args, world, rank, dev)
    if args.workload in STRESS_ALIASES:
        return run_blockmap_stress(args, world, rank, dev)
    aliases = DECODE_ALIASES if decode else (BWD_ALIASES if backward else WORKLOAD_ALIASES)
    if args.workload in EXTRA_WORKLOADS:
        base, kw = EXTRA_WORKLOADS[args.workload]
        wl = synth.WORKLOADS[base].scaled(**kw)
    else:
        wl = synth.WORKLOADS[aliases.get(args.workload, args.workload)]
    if args.heads:
        wl = wl.scaled(Hq=args.heads, Hkv=max(1, args.heads * wl.Hkv // wl.Hq),
                       long_heads=tuple(h for h in wl.long_heads if h < args.heads))
    split = args.split == "heads"
    if split:
        # one layer split over the ranks by kv-head groups (strong scaling)
        if decode or backward or wl.segmented:
            raise SystemExit("--split heads runs the prefill workloads c2, c3 and c4")
        if world > wl.Hkv:
            raise SystemExit("--split heads needs at most Hkv = %d ranks" % wl.Hkv)
        from long_context_structured_b200.shard import head_shard
        job = Job(wl, seed=0, dev=dev, heads=head_shard(wl.Hq, wl.Hkv, world, rank))
    else:
        job = (DecodeJob if decode else (BwdJob if backward else Job))(wl, seed=rank, dev=dev)
    lib = _lib.load()

    for _ in range(args.warmup):
        job.step()
    torch.cuda.synchronize()
    if sa.stream_status() != 0:
        raise RuntimeError("device status word reports a failure after warm-up")

    gpu_uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    phys = int(vis.split(",")[local]) if vis and vis.split(",")[local].strip().isdigit() else local
    clocks = ClockSampler(gpu_uuid, phys)
    clocks.start()
    time.sleep(0.3)
    plain = None
    if decode:
        job.capture()
        plain = job.graph_step
    elapsed_ms, prof = timed_passes(job.step, args.steps, lib, world, plain_step=plain)
    clk = clocks.stop()
    status = sa.stream_status()

    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_step = float(t.item()) / args.steps
    # whole-job work: every rank's own problem (weak), or the one split layer (strong)
    job_flops = job.full_flops if split else job.flops * world
    value = job_flops / (ms_step * 1e-3) / 1e12
    tokens_s = wl.B * (1 if decode else wl.T) * (1 if split else world) / (ms_step * 1e-3)

    # per-group device time per step (every group runs once per step; a group
    # may hold more than one kernel), max over ranks (same group order on
    # every rank)
    groups = sorted(prof)
    avg = torch.tensor([prof[g][1] / args.steps for g in groups] or [0.0], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(avg, op=dist.ReduceOp.MAX)
    avg_ms = {g: float(avg[x].item()) for x, g in enumerate(groups)}
    peaks, peak_src = load_peaks()
    work = job.group_work()
    kernels = {}
    for g in groups:
        n, ms = prof[g]
        kernels[g] = {"kernel": kernel_name(wl, g), "launches": n, "ms_per_step": round(avg_ms[g], 5),
                      "share": round(ms / max(sum(v[1] for v in prof.values()), 1e-12), 4)}
        if g in work and avg_ms[g] > 0:
            r = roofline_of(g, work[g], avg_ms[g], peaks, peak_src)
            kernels[g].update({"bound": r["bound"], "achieved": r["achieved"], "unit": r["unit"], "frac": r["frac"]})
    # the roofline line is the dominant kernel's (largest share of device time)
    dom = max((g for g in groups if g in work), key=lambda g: prof[g][1], default=None)
    roof = None
    if dom is not None:
        roof = roofline_of(dom, work[dom], avg_ms[dom], peaks, peak_src)
        roof["kernel"] = kernel_name(wl, dom)
        roof["traffic"] = TOPK_SCORE_TRAFFIC_BYTES if (dom == "topk_score" and args.workload == DEFAULT_WORKLOAD
                                                       and not args.heads) else None
    gpu_launches = sum(n for n, _ in prof.values())

    # end to end through the public call with host buffers (H2D + D2H inside)
    n_e2e = max(3, min(10, args.steps))
    # warm the host path: pinned output buffers come from the caching host
    # allocator once two calls' results have been alive at the same time
    for _ in range(3):
        outs = job.host_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record()
    for _ in range(n_e2e):
        outs = job.host_step()
    s1.record()
    torch.cuda.synchronize()
    te = torch.tensor([s0.elapsed_time(s1) / n_e2e], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(te, op=dist.ReduceOp.MAX)
    ms_e2e = float(te.item())
    e2e = {"value": round(job_flops / (ms_e2e * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
           "ms_per_step": round(ms_e2e, 3), "steps": n_e2e, "h2d_bytes_per_step": job.h2d_bytes(),
           "d2h_bytes_per_step": int(sum(o.nbytes for o in outs)),
           "path": ("long_context_structured_b200.decode_fwd: query from pinned host memory, device-resident cache, "
                    "outputs into pinned host memory") if decode else
                   ("long_context_structured_b200.bwd: Q, K, V, O, LSE, dO from pinned host memory, dQ, dK, dV "
                    "into pinned host memory") if backward else
                   ("long_context_structured_b200.%s on pinned host tensors (outputs into pinned host memory)"
                    % ("segment_fwd" if wl.segmented else "fwd"))}

    gather = None
    if split and world > 1:
        # the head blocks back into one layer on every rank (NCCL all-gather),
        # once, outside the timed steps
        from long_context_structured_b200.shard import gather_heads
        full = job.full_wl
        gather_heads(job.O, job.lse, full.Hq, full.Hkv, world)  # warm the communicator
        torch.cuda.synchronize()
        dist.barrier()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record()
        O_full, _ = gather_heads(job.O, job.lse, full.Hq, full.Hkv, world)
        g1.record()
        torch.cuda.synchronize()
        tg = torch.tensor([g0.elapsed_time(g1)], dtype=torch.float64, device=dev)
        dist.all_reduce(tg, op=dist.ReduceOp.MAX)
        gather = {"ms": round(float(tg.item()), 4), "bytes_per_rank_out": int(job.O.nbytes + job.lse.nbytes),
                  "full_shape": list(O_full.shape), "note": "all_gather of O and LSE, not in the step time"}
        del O_full

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_bwd(wl) if backward else cpu_baseline(wl, job.inp, cpu_rows_of(args), decode=decode)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    peak = float(peaks["bf16_tflops"])
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "strong" if split else "weak",
        "vs_baseline": None, "dtype": "f32" if wl.dtype == "f32" else "bf16",
        "data": "synthetic (seeded N(0,1)%s)" % ("; keys 0-3 x8" if wl.sink_scale != 1.0 else ""),
        "config": config_dict(job.full_wl if split else wl, job.pairs, decode=decode,
                              n_copies=getattr(job, "n_copies", 0), backward=backward,
                              parallelism=("heads%d (kv-head groups of one layer per rank)" % world) if split else
                              ("dp%d (an independent layer per rank)" % world)),
        "tokens_per_s": round(tokens_s, 1),
        "frac_of_bf16_peak": round(value / world / peak, 4),
        "roofline": roof,
        "kernels": kernels, "kernel_times": KERNEL_TIMES_NOTE,
        "step_timing": ("CUDA-graph replays of the whole step (one graph per cache copy), as a generation loop "
                        "runs it" if decode else "eager calls of the public API"),
        "gpu_launches": gpu_launches,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "clocks": clk,
        "device_status": status,
    }
    if gather is not None:
        line["head_gather"] = gather
    print(json.dumps(line), flush=True)


def run_tree(args, world, rank, dev):
    """The tree cross-attention workload: same timing, clocks and JSON line
    as the other workloads."""
    import torch
    import torch.distributed as dist

    import long_context_structured_b200 as sa
    from long_context_structured_b200 import _lib
    cfg = dict(TREE_WORKLOADS[TREE_ALIASES[args.workload]])
    if args.heads:
        cfg["Hq"] = cfg["Hkv"] = args.heads
    job = TreeJob(cfg, seed=rank, dev=dev)
    lib = _lib.load()
    for _ in range(args.warmup):
        job.step()
    torch.cuda.synchronize()
    if sa.stream_status() != 0:
        raise RuntimeError("device status word reports a failure after warm-up")
    gpu_uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    clocks = ClockSampler(gpu_uuid, int(os.environ.get("LOCAL_RANK", "0")))
    clocks.start()
    time.sleep(0.3)
    el_ms, prof = timed_passes(job.step, args.steps, lib, world)
    clk = clocks.stop()
    t = torch.tensor([el_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_step = float(t.item()) / args.steps
    value = job.flops * world / (ms_step * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    work = job.group_work()
    kernels, roof = {}, None
    for g in sorted(prof):
        n, ms = prof[g]
        avg = ms / args.steps
        kernels[g] = {"kernel": kernel_name(None, g), "launches": n, "ms_per_step": round(avg, 5),
                      "share": round(ms / max(sum(v[1] for v in prof.values()), 1e-12), 4)}
        if g in work and avg > 0:
            r = roofline_of(g, work[g], avg, peaks, peak_src)
            kernels[g].update({"bound": r["bound"], "achieved": r["achieved"], "unit": r["unit"], "frac": r["frac"]})
    dom = max((g for g in prof if g in work), key=lambda g: prof[g][1], default=None)
    if dom is not None:
        roof = roofline_of(dom, work[dom], prof[dom][1] / args.steps, peaks, peak_src)
        roof["kernel"] = kernel_name(None, dom)
        roof["traffic"] = None
    n_e2e = max(3, min(10, args.steps))
    for _ in range(3):  # warm the host path (pinned buffers cached)
        outs = job.host_step()
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record()
    for _ in range(n_e2e):
        outs = job.host_step()
    s1.record()
    torch.cuda.synchronize()
    ms_e2e = s0.elapsed_time(s1) / n_e2e
    cpu = cpu_baseline_tree(cfg) if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    c = cfg
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1))",
        "config": {"workload": "SharedLLM tree cross-attention (language-modelling policy): %d decoder queries over "
                               "a %d-token context in %d chunks of %d, depth %d, leaf rate %d (%d kept rows)"
                               % (c["Tq"], c["n_chunks"] * c["chunk_len"], c["n_chunks"], c["chunk_len"], c["depth"],
                                  c["alpha_leaf"], job.S),
                   "B": c["B"], "Hq": c["Hq"], "Hkv": c["Hkv"], "d": c["d"], "rope_theta": c["rope_theta"],
                   "pairs_per_rank": job.pairs,
                   "l2": "no flush: each step reads the %d MB context K/V and writes the kept rows, > 126 MB L2"
                         % (job.h2d_bytes() >> 20)},
        "tokens_per_s": round(c["B"] * c["Tq"] * world / (ms_step * 1e-3), 1),
        "frac_of_bf16_peak": round(value / world / float(peaks["bf16_tflops"]), 4),
        "roofline": roof, "kernels": kernels, "kernel_times": KERNEL_TIMES_NOTE,
        "gpu_launches": sum(n for n, _ in prof.values()),
        "e2e": {"value": round(job.flops * world / (ms_e2e * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_step": round(ms_e2e, 3), "steps": n_e2e, "h2d_bytes_per_step": job.h2d_bytes(),
                "d2h_bytes_per_step": int(sum(o.nbytes for o in outs)),
                "path": "long_context_structured_b200.tree_cross_fwd on inputs from pinned host memory"},
        "cpu_baseline": cpu, "clocks": clk, "device_status": sa.stream_status(),
    }
    print(json.dumps(line), flush=True)


def run_stream(args, world, rank, dev):
    """Streaming generation steps over the device-resident cache."""
    import torch
    import torch.distributed as dist

    import long_context_structured_b200 as sa
    from long_context_structured_b200 import _lib
    cfg = dict(STREAM_WORKLOADS[STREAM_ALIASES[args.workload]])
    job = StreamJob(cfg, seed=rank, dev=dev)
    lib = _lib.load()
    for _ in range(args.warmup):
        job.step()
    torch.cuda.synchronize()
    len0 = job.mean_len()
    gpu_uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    clocks = ClockSampler(gpu_uuid, int(os.environ.get("LOCAL_RANK", "0")))
    clocks.start()
    time.sleep(0.3)
    el_ms, _ = timed_pass(job.step, args.steps, lib, world, False)
    len1 = job.mean_len()  # the work of the step-time pass
    _, prof = timed_pass(job.step, args.steps, lib, world, True)
    clk = clocks.stop()
    t = torch.tensor([el_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_step = float(t.item()) / args.steps
    c = cfg
    mean_len = 0.5 * (len0 + len1)  # cached keys per sequence, averaged over the timed steps
    flops = 4.0 * c["d"] * c["Hq"] * c["B"] * mean_len
    value = flops * world / (ms_step * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    kv_bytes = mean_len * c["B"] * c["Hkv"] * 2 * c["d"] * 2
    work = {"stream_decode": ("hbm", kv_bytes + 4 * c["B"] * c["Hq"] * c["d"], "B"),
            "stream_append": ("hbm", 2 * c["B"] * c["Hkv"] * c["d"] * 2 * 2, "B")}
    kernels = {}
    for g in sorted(prof):
        n, ms = prof[g]
        avg = ms / args.steps
        kernels[g] = {"kernel": {"stream_decode": "decode_partial_kernel + decode_combine_kernel",
                                 "stream_append": "stream_append/plan/move kernels"}.get(g, g),
                      "launches": n, "ms_per_step": round(avg, 5),
                      "share": round(ms / max(sum(v[1] for v in prof.values()), 1e-12), 4)}
        if g in work and avg > 0:
            r = roofline_of(g, work[g], avg, peaks, peak_src)
            kernels[g].update({"bound": r["bound"], "achieved": r["achieved"], "unit": r["unit"], "frac": r["frac"]})
    roof = roofline_of("stream_decode", work["stream_decode"], prof["stream_decode"][1] / args.steps, peaks, peak_src)
    roof["kernel"] = "decode_partial_kernel + decode_combine_kernel"
    roof["traffic"] = None
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) K/V/Q rows, Bernoulli separators)",
        "config": {"workload": "SepLLM streaming generation: %d sequences, cache a=%d s=%d w=%d c=%d, one token "
                               "appended (with on-device compaction) and decoded per sequence per step"
                               % (c["B"], c["a"], c["s"], c["w"], c["c"]),
                   "B": c["B"], "Hq": c["Hq"], "Hkv": c["Hkv"], "d": c["d"], "rope_theta": c["rope_theta"],
                   "mean_cached_keys": round(mean_len, 1), "tokens_appended_before_timing": job.t - args.steps,
                   "l2": "no flush: the caches hold %d MB of K/V, > 126 MB L2"
                         % (c["B"] * c["Hkv"] * c["c"] * c["d"] * 4 >> 20)},
        "tokens_per_s": round(c["B"] * world / (ms_step * 1e-3), 1),
        "roofline": roof, "kernels": kernels, "kernel_times": KERNEL_TIMES_NOTE,
        "gpu_launches": sum(n for n, _ in prof.values()),
        "e2e": None, "cpu_baseline": None, "clocks": clk, "device_status": sa.stream_status(),
    }
    print(json.dumps(line), flush=True)


def timed_pass(step, steps, lib, world, profiled):
    """`steps` calls of `step` bracketed by a barrier and a synchronize on
    both sides, with or without the library's per-launch-group CUDA events.
    Returns (elapsed ms, {group: (launches, ms)})."""
    import torch
    import torch.distributed as dist

    profile_collect(lib)  # drop anything recorded before
    lib.sattn_profile_enable(1 if profiled else 0)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    lib.sattn_profile_enable(0)
    return e0.elapsed_time(e1), profile_collect(lib)


def timed_passes(step, steps, lib, world, plain_step=None):
    """The step time from a pass without per-launch events (of plain_step
    when given, e.g. a CUDA-graph replay of the same step), the per-kernel
    times from a second pass of `step` with them."""
    ms, _ = timed_pass(plain_step or step, steps, lib, world, False)
    _, prof = timed_pass(step, steps, lib, world, True)
    return ms, prof


KERNEL_TIMES_NOTE = ("per-kernel times from a second timed pass of the same steps with CUDA events around each "
                     "launch group; the step time from the first pass, without them")


def run_blockmap_stress(args, world, rank, dev):
    """The block map at stress size: 2048 sequences of 32768 flags (rate
    0.1), tile classes included; reported in GB/s of algorithmic bytes (flags
    read; tile classes, separator positions, counts and ranges written)."""
    import torch

    import long_context_structured_b200 as sa
    from long_context_structured_b200 import _lib
    B, T, ns, w = 2048, 32768, 4, 256
    g = torch.Generator().manual_seed(rank)
    flags = (torch.rand(B, T, generator=g) < 0.1).to(torch.uint8).to(dev)
    lib = _lib.load()
    for _ in range(args.warmup):
        sa.build_blockmap(flags, B=B, T=T, n_start=ns, window=w, device=dev)
    torch.cuda.synchronize()
    gpu_uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    clocks = ClockSampler(gpu_uuid, int(os.environ.get("LOCAL_RANK", "0")))
    clocks.start()
    time.sleep(0.3)
    el_ms, prof = timed_passes(lambda: sa.build_blockmap(flags, B=B, T=T, n_start=ns, window=w, device=dev),
                               args.steps, lib, world)
    clk = clocks.stop()
    ms = el_ms / args.steps
    nqt = T // 128
    nbytes = B * T + B * nqt * nqt + B * T * 4 + B * 4 + B * nqt * 8
    kms = prof["blockmap"][1] / args.steps
    peaks, peak_src = load_peaks()
    roof = roofline_of("blockmap", ("hbm", nbytes, "B"), kms, peaks, peak_src)
    roof["kernel"] = "sep_scan_kernel + tile_class_kernel"
    roof["traffic"] = None
    if rank == 0:
        print(json.dumps({
            "metric": "block map GB/s at stress size (algorithmic bytes)", "value": roof["achieved"], "unit": "GB/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u8",
            "data": "synthetic (seeded Bernoulli(0.1) separator flags)",
            "config": {"workload": "block map of %d sequences x %d flags (2^26), n_start %d, window %d, tile classes "
                                   "%dx%d per sequence" % (B, T, ns, w, nqt, nqt),
                       "algorithmic_bytes": nbytes,
                       "l2": "no flush: %d MB read and written per step, > 126 MB L2" % (nbytes >> 20)},
            "roofline": roof, "kernels": {"blockmap": {"launches": prof["blockmap"][0], "ms_per_step": round(kms, 5)}},
            "kernel_times": KERNEL_TIMES_NOTE,
            "gpu_launches": prof["blockmap"][0], "clocks": clk, "e2e": None, "cpu_baseline": None}), flush=True)


# ---------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# ---------------------------------------------------------------------------

def _oracle_sample(wl, n_rows, seed):
    """Rows (b, h, i) spread over all batches, heads and positions, seeded."""
    rng = np.random.default_rng(seed)
    bs = rng.integers(0, wl.B, n_rows)
    heads = rng.integers(0, wl.Hq, n_rows)
    pos = rng.integers(0, wl.T, n_rows)
    return np.stack([bs, heads, pos], axis=1).astype(np.int64)


def _pairs_of_rows(wl, rows, is_sep):
    """Kept (q, k) pairs of the sampled rows (same counting as unmasked_pairs)."""
    b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
    if wl.segmented:
        s, t = i // wl.seg_S, i % wl.seg_S
        is_long = np.isin(h, np.array(wl.long_heads, dtype=np.int64))
        extra = np.where(s > 0, np.where(is_long, wl.seg_R, wl.seg_M), 0)
        return int((t + 1 + extra).sum())
    n = np.minimum(i + 1, wl.n_start + wl.window + 1)
    if is_sep is not None:
        f = is_sep.astype(np.int64).copy()
        f[:, : wl.n_start] = 0
        pre = np.concatenate([np.zeros((wl.B, 1), np.int64), np.cumsum(f, axis=1)], axis=1)
        n = n + pre[b, np.clip(i - wl.window, 0, wl.T)]
    if wl.topk > 0:
        n = n + np.minimum(wl.topk, np.maximum(0, i - wl.window - wl.n_start))
    return int(n.sum())


def _oracle_rows(O, wl, inp, rows, nthreads):
    p = O.params_of(wl)
    if wl.segmented:
        O.segment_rows(p, wl.seg_S, wl.seg_M, wl.seg_R, wl.retr_block, inp["is_long"], inp["q"], inp["k"],
                       inp["v"], rows, nthreads=nthreads)
    else:
        O.fwd_rows(p, inp["q"], inp["k"], inp["v"], inp["is_sep"], rows, nthreads=nthreads)


def cpu_rows_of(args) -> int:
    return args.cpu_rows if args.cpu_rows else CPU_ROWS.get(args.workload, 32768)


def cpu_sample_rows(wl, n_rows):
    """The CPU-oracle sample of a forward workload: seeded rows over all
    batches, heads and positions, grouped by (batch, head)."""
    rows = _oracle_sample(wl, n_rows, 1234)
    return rows[np.lexsort((rows[:, 2], rows[:, 1], rows[:, 0]))]


def cpu_baseline(wl, inp, n_rows, decode=False):
    from oracle import oracle as O
    O.build()
    if decode:  # the decoded rows (b, h, T-1), repeated to a bounded sample
        base = np.array([(b, h, wl.T - 1) for b in range(wl.B) for h in range(wl.Hq)], dtype=np.int64)
        rows = np.tile(base, (max(1, n_rows // (16 * len(base))), 1))
    else:
        rows = cpu_sample_rows(wl, n_rows)
    nthreads = O.nthreads_default()
    t0 = time.perf_counter()
    _oracle_rows(O, wl, inp, rows, nthreads)
    dt = time.perf_counter() - t0
    flops = 4.0 * wl.d * _pairs_of_rows(wl, rows, inp["is_sep"])
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": nthreads, "kind": "oracle",
            "sample": "%d %s rows (b, h, i) of the same workload, all heads, fp64, %.1f s" % (
                len(rows), "decoded" if decode else "seeded", dt),
            "seconds": round(dt, 2)}


def bwd_sample(wl):
    """A bounded sample of a backward workload for the CPU oracle: the same
    mask parameters on one kv-head group of one sequence, T cut to 4096."""
    return wl.scaled(B=1, Hq=wl.Hq // wl.Hkv, Hkv=1, T=min(wl.T, 4096))


def cpu_baseline_bwd(wl):
    from oracle import oracle as O
    O.build()
    sw = bwd_sample(wl)
    inp = synth.make_inputs(sw, seed=0)
    g = np.random.default_rng(3)
    do = g.standard_normal(inp["q"].shape).astype(np.float32)
    if sw.dtype == "bf16":
        do = (do.view(np.uint32) >> 16).astype(np.uint16)
    nthreads = O.nthreads_default()
    t0 = time.perf_counter()
    O.bwd(O.params_of(sw), inp["q"], inp["k"], inp["v"], inp["is_sep"], do, nthreads=nthreads)
    dt = time.perf_counter() - t0
    flops = float(BWD_FLOPS_PER_PAIR_D) * sw.d * unmasked_pairs(sw, inp["is_sep"])
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
            "sample": "backward of one kv-head group (%d query heads), B=1, T=%d, same mask parameters, fp64, "
                      "%.1f s (the oracle's backward runs one thread per kv head)" % (sw.Hq, sw.T, dt),
            "seconds": round(dt, 2)}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import oracle as O
    O.build()
    decode = args.workload in DECODE_ALIASES
    if args.workload in TREE_ALIASES:
        cfg = TREE_WORKLOADS[TREE_ALIASES[args.workload]]
        t0 = time.perf_counter()
        for _ in range(args.warmup + args.steps):
            cpu = cpu_baseline_tree(cfg, n_rows=8)
        line = {"impl": "reference", "metric": METRIC, "value": cpu["value"], "unit": "TFLOP/s", "n_gpus": 1,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round((time.perf_counter() - t0) * 1e3 / (args.warmup + args.steps), 3),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic (seeded N(0,1))", "config": {"workload": "tree_cross_128k (oracle sample)"},
                "cpu_baseline": cpu,
                "e2e": {"value": cpu["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    if args.workload in BWD_ALIASES:
        wl = synth.WORKLOADS[BWD_ALIASES[args.workload]]
        t0 = time.perf_counter()
        for _ in range(args.warmup + args.steps):
            cpu = cpu_baseline_bwd(wl)
        line = {"impl": "reference", "metric": METRIC, "value": cpu["value"], "unit": "TFLOP/s", "n_gpus": 1,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round((time.perf_counter() - t0) * 1e3 / (args.warmup + args.steps), 3),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic (seeded N(0,1))", "config": config_dict(bwd_sample(wl), 0, backward=True),
                "cpu_baseline": cpu,
                "e2e": {"value": cpu["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    wl = synth.WORKLOADS[(DECODE_ALIASES if decode else WORKLOAD_ALIASES).get(args.workload, args.workload)]
    inp = synth.make_inputs(wl, seed=0)
    nthreads = O.nthreads_default()
    # the CPU-baseline sample, one (batch, head) group per step, groups in
    # turn: each step pays one head's set-up for that head's rows, as the
    # baseline does, so the two figures measure the same thing
    sample = cpu_sample_rows(wl, cpu_rows_of(args))
    keys = sample[:, 0] * wl.Hq + sample[:, 1]
    groups = [sample[keys == kk] for kk in np.unique(keys)]

    def step(s):
        if decode:  # the decoded row of every sequence, one head per step
            rows = np.array([(b, s % wl.Hq, wl.T - 1) for b in range(wl.B)], dtype=np.int64)
        else:
            rows = groups[s % len(groups)]
        _oracle_rows(O, wl, inp, rows, nthreads)
        return _pairs_of_rows(wl, rows, inp["is_sep"])

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
        "data": "synthetic (seeded N(0,1)%s)" % ("; keys 0-3 x8" if wl.sink_scale != 1.0 else ""),
        "config": config_dict(wl, int(decode_keys(wl, inp["is_sep"]).sum()) * wl.Hq if decode
                              else unmasked_pairs(wl, inp["is_sep"]), decode=decode),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": nthreads, "kind": "oracle",
                         "sample": ("each step: the decoded rows of one head (heads cycle)" if decode else
                                    "each step: the rows of one (batch, head) of the %d-row CPU-baseline sample "
                                    "(groups in turn)" % len(sample)) + ", fp64 C oracle"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(WORKLOAD_ALIASES) + sorted(WORKLOAD_ALIASES.values()) + sorted(DECODE_ALIASES)
                    + sorted(BWD_ALIASES) + sorted(TREE_ALIASES) + sorted(STREAM_ALIASES) + sorted(STRESS_ALIASES)
                    + sorted(EXTRA_WORKLOADS))
    ap.add_argument("--cpu-rows", type=int, default=0,
                    help="rows in the CPU-oracle baseline sample (default: 6144 on the top-k workload, else 32768)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--heads", type=int, default=0, help="override the head count (profiling captures only)")
    ap.add_argument("--split", choices=["none", "heads"], default="none",
                    help="none: an independent layer per rank (weak scaling); heads: one layer split over the "
                         "ranks by kv-head groups (strong scaling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    args.workload = {v: k for k, v in WORKLOAD_ALIASES.items()}.get(args.workload, args.workload)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
