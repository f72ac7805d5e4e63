"""Seeded synthetic inputs for the structured-attention workloads.

This module only draws numbers.  It holds none of the attention arithmetic:
no mask rule, no logit, no softmax.  Both the CUDA path and the CPU oracle are
fed from the arrays it returns, so neither side can bias the other's inputs.

The workloads stand in for the shapes the source pages evaluate on (a
Llama-2-7B attention layer for LM-Infinite, a Llama-3-8B GQA layer for SepLLM,
a LLaMA2-7B layer for segmented execution); the pages' datasets and trained
weights are not used.  Values are N(0, 1) unless a workload says otherwise.

Arrays come back as numpy:  bf16 tensors as ``uint16`` bit patterns (exactly
the values both sides see), fp32 tensors as ``float32``, separator flags as
``uint8``.  Layout is ``[B, H, T, d]`` with the head dimension contiguous.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and mask parameters of one synthetic workload."""

    name: str
    B: int
    Hq: int
    Hkv: int
    T: int
    d: int
    dtype: str                 # "bf16" or "f32"
    n_start: int = 0
    window: int = 0
    L_pretrain: int = 0        # 0 disables the distance cap
    rope_theta: float = 0.0    # 0 disables RoPE
    rope_pos_scale: float = 1.0  # position interpolation: rotary positions multiplied by this
    alibi: bool = False        # clipped ALiBi bias in place of the rotation (rope_theta 0)
    topk: int = 0
    sep_rate: float = 0.0      # Bernoulli flag rate (c1-style) ...
    sep_vocab: int = 0         # ... or token-id derived flags (c3-style) when > 0
    sep_ids: int = 0
    sink_scale: float = 1.0    # keys 0..3 scaled by this (attention-sink mimic)
    plant: int = 0             # planted key/query clusters per head (top-k workload)
    plant_cos: float = 0.9
    plant_run: int = 32
    # segmented execution
    seg_S: int = 0
    seg_M: int = 0
    seg_R: int = 0
    retr_block: int = 64
    long_heads: tuple = ()

    @property
    def segmented(self) -> bool:
        return self.seg_S > 0

    def is_long_mask(self) -> np.ndarray:
        m = np.zeros(self.Hq, dtype=np.uint8)
        for h in self.long_heads:
            m[h] = 1
        return m

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads.  Sizes, rates and mask parameters follow the
# configuration list that accompanies the pages; the separator vocabulary
# (128,256 ids, 9 separator ids, 10% rate) is Llama-3's tokenizer size.
WORKLOADS = {
    "c1_f32_sep": Workload(
        name="c1_f32_sep", B=1, Hq=1, Hkv=1, T=1024, d=64, dtype="f32",
        n_start=4, window=128, sep_rate=0.08),
    "c2_lminf_16k": Workload(
        name="c2_lminf_16k", B=1, Hq=32, Hkv=32, T=16384, d=128, dtype="bf16",
        n_start=4, window=4096, L_pretrain=4096, rope_theta=10000.0,
        sink_scale=8.0),
    "c3_sepllm_gqa_8k": Workload(
        name="c3_sepllm_gqa_8k", B=4, Hq=32, Hkv=8, T=8192, d=128, dtype="bf16",
        n_start=4, window=256, L_pretrain=0, rope_theta=500000.0,
        sep_vocab=128256, sep_ids=9, sep_rate=0.10),
    "c4_lminf_topk_32k": Workload(
        name="c4_lminf_topk_32k", B=1, Hq=32, Hkv=32, T=32768, d=128, dtype="bf16",
        n_start=4, window=4096, L_pretrain=4096, rope_theta=10000.0, topk=5,
        plant=64),
    "c5_segmented_32k": Workload(
        name="c5_segmented_32k", B=1, Hq=32, Hkv=32, T=32768, d=128, dtype="bf16",
        rope_theta=10000.0, seg_S=2048, seg_M=512, seg_R=1024, retr_block=64,
        long_heads=tuple(range(24, 32))),
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _bf16_bits(x: torch.Tensor) -> np.ndarray:
    """Round fp32 to bf16 (round-to-nearest-even, torch's cast) and return the bits."""
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _normal(g: torch.Generator, shape) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32)


def _inverse_rotate_half(x: np.ndarray, pos: float, theta: float) -> np.ndarray:
    """Undo a rotate-half rotary rotation by ``pos`` (fp64).

    Used only to *shape* planted query vectors so that, after the attention's
    own rotation, they point along a chosen direction.  Neither the oracle nor
    the CUDA path calls this; if it were wrong the planted keys would simply
    not be found, which the top-k tests check.
    """
    d = x.shape[-1]
    h = d // 2
    c = np.arange(h, dtype=np.float64)
    ang = -pos * np.power(theta, -2.0 * c / d)
    cs, sn = np.cos(ang), np.sin(ang)
    a, b = x[..., :h], x[..., h:]
    return np.concatenate([a * cs - b * sn, b * cs + a * sn], axis=-1)


def separator_flags(wl: Workload, seed: int) -> Optional[np.ndarray]:
    """Separator flags ``[B, T]`` (uint8) or None when the workload has none."""
    if wl.sep_rate <= 0.0:
        return None
    g = _gen(seed * 7919 + 17)
    if wl.sep_vocab > 0:
        # Token ids: with prob. sep_rate uniform over a seeded separator-id
        # set, otherwise uniform over the remaining ids; flag = id in set.
        sep_set = torch.randperm(wl.sep_vocab, generator=g)[: wl.sep_ids]
        sep_sorted = torch.sort(sep_set).values
        pick_sep = torch.rand(wl.B, wl.T, generator=g) < wl.sep_rate
        which = torch.randint(0, wl.sep_ids, (wl.B, wl.T), generator=g)
        other = torch.randint(0, wl.sep_vocab - wl.sep_ids, (wl.B, wl.T), generator=g)
        # map [0, V - n) onto the ids not in the set, keeping order
        shifted = other.clone()
        for s in sep_sorted.tolist():
            shifted = shifted + (shifted >= s).to(shifted.dtype)
        ids = torch.where(pick_sep, sep_set[which], shifted)
        flags = torch.isin(ids, sep_set)
        return flags.to(torch.uint8).numpy()
    flags = torch.rand(wl.B, wl.T, generator=g) < wl.sep_rate
    return flags.to(torch.uint8).numpy()


def make_inputs(wl: Workload, seed: int = 0) -> dict:
    """Q, K, V (and flags / long-head mask) for ``wl``.

    Returns a dict with numpy arrays ``q`` ``[B,Hq,T,d]``, ``k`` and ``v``
    ``[B,Hkv,T,d]`` (uint16 bf16 bits or float32), ``is_sep`` ``[B,T]`` or
    None, ``is_long`` ``[Hq]`` (segmented workloads) and the recipe metadata.
    """
    g = _gen(seed)
    q = _normal(g, (wl.B, wl.Hq, wl.T, wl.d))
    k = _normal(g, (wl.B, wl.Hkv, wl.T, wl.d))
    v = _normal(g, (wl.B, wl.Hkv, wl.T, wl.d))
    if wl.sink_scale != 1.0:
        k[:, :, : min(4, wl.T), :] *= wl.sink_scale
    meta = {}
    if wl.plant > 0:
        q, k, meta = _plant(wl, q, k, seed)
    out = {"workload": wl, "seed": seed, "meta": meta}
    if wl.dtype == "bf16":
        out["q"], out["k"], out["v"] = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    else:
        out["q"], out["k"], out["v"] = q.numpy(), k.numpy(), v.numpy()
    out["is_sep"] = separator_flags(wl, seed)
    out["is_long"] = wl.is_long_mask() if wl.segmented else None
    return out


def _plant(wl: Workload, q: torch.Tensor, k: torch.Tensor, seed: int):
    """Plant, per head, ``wl.plant`` keys aligned (cosine ``plant_cos``) with
    runs of ``plant_run`` later queries, measured after the query's rotation
    to the capped distance.  Key positions are uniform in
    ``[n_start, T - w - 1024)``; each run starts uniformly in
    ``(j + w, T - run]``.  The key keeps its norm; the queries keep theirs.
    """
    g = _gen(seed * 104729 + 3)
    B, H, T, d = q.shape
    rep = wl.Hq // wl.Hkv
    lo, hi = wl.n_start, T - wl.window - 1024
    if hi <= lo:
        raise ValueError("sequence too short to plant clusters")
    pos_cap = float(wl.L_pretrain if wl.L_pretrain > 0 else 0)
    planted = []
    for b in range(B):
        for h in range(H):
            hk = h // rep
            for _ in range(wl.plant):
                j = int(torch.randint(lo, hi, (1,), generator=g))
                u = torch.randn(d, generator=g, dtype=torch.float64).numpy()
                u /= np.linalg.norm(u)
                r = torch.randn(d, generator=g, dtype=torch.float64).numpy()
                r -= r.dot(u) * u
                r /= np.linalg.norm(r)
                kj = k[b, hk, j].numpy().astype(np.float64)
                newk = np.linalg.norm(kj) * (wl.plant_cos * u + math.sqrt(1.0 - wl.plant_cos ** 2) * r)
                k[b, hk, j] = torch.from_numpy(newk.astype(np.float32))
                start = int(torch.randint(j + wl.window + 1, T - wl.plant_run + 1, (1,), generator=g))
                qs = q[b, h, start:start + wl.plant_run].numpy().astype(np.float64)
                target = np.linalg.norm(qs, axis=-1, keepdims=True) * u[None, :]
                if wl.rope_theta > 0:
                    target = _inverse_rotate_half(target, pos_cap, wl.rope_theta)
                q[b, h, start:start + wl.plant_run] = torch.from_numpy(target.astype(np.float32))
                planted.append((b, h, j, start))
    meta = {"planted": planted}
    return q, k, meta


def sample_rows(wl: Workload, n_per_head: int, seed: int = 1, extra=()) -> np.ndarray:
    """A seeded row sample ``[(b, h, i)]`` covering every (b, h), the tile and
    window boundaries, the sequence ends, plus ``extra`` rows."""
    g = _gen(seed * 31337 + 11)
    rows = set()
    bnd = [0, 1, wl.n_start, wl.n_start + 1, 127, 128, 129, wl.T - 1, wl.T - 2]
    for x in (wl.window, wl.window + 1, wl.window + wl.n_start, wl.window + 127, wl.window + 128):
        bnd.append(x)
    if wl.segmented:
        for s in range(0, wl.T, wl.seg_S):
            bnd += [s, s + 1, s + wl.seg_S - 1]
    bnd = [x for x in bnd if 0 <= x < wl.T]
    for b in range(wl.B):
        for h in range(wl.Hq):
            for i in bnd:
                rows.add((b, h, i))
            for i in torch.randint(0, wl.T, (n_per_head,), generator=g).tolist():
                rows.add((b, h, int(i)))
    for r in extra:
        rows.add(tuple(int(x) for x in r))
    return np.array(sorted(rows), dtype=np.int64).reshape(-1, 3)
