"""Structured-mask causal attention for B200 (sm_100a).

Python binding of ``libsattn.so``.  Every computation runs in the library's
CUDA kernels; this module only marshals arguments: it reads shapes and
strides from torch tensors, allocates the caller-side workspace with torch,
and passes raw device pointers and the current CUDA stream through the C ABI.

Public calls (names follow the C ABI):
    fwd(q, k, v, ...)            -> (O, lse)
    topk_select(q, k, ...)       -> (idx, logit)
    build_blockmap(is_sep, ...)  -> dict(cls, sep_pos, sep_count, qtile_sep_range)
    build_blockmap_noalloc(...)  -> the same, scratch inside the library (no workspace)
    segment_fwd(q, k, v, ...)    -> (O, lse, prefix_blocks)
    segment_bwd(q, k, v, o, lse, prefix_blocks, do, ...) -> (dq, dk, dv)
    stream_status(workspace)     -> device status code

``fwd`` and ``segment_fwd`` also accept host (CPU) tensors: the inputs are
then copied to the device, the call runs there, and the outputs are copied
back -- the end-to-end path a host application uses.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _lib
from ._lib import DTYPE_BF16, DTYPE_F32, SattnError, SattnParams

__all__ = ["fwd", "topk_select", "build_blockmap", "build_blockmap_noalloc", "segment_fwd", "segment_bwd",
           "SegmentStream", "stream_status", "workspace_size",
           "segment_workspace_size", "params", "SattnError", "version", "TILE", "selftest_wait_timeout",
           "decode_fwd"]

TILE = 128
_ws_cache: dict = {}


def version() -> int:
    return _lib.load().sattn_version()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    if t.dtype == torch.float32:
        return DTYPE_F32
    raise TypeError("q/k/v must be bfloat16 or float32, got %s" % t.dtype)


def _strides(t: Optional[torch.Tensor]):
    if t is None:
        return (0, 0, 0)
    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError("expected a [B, H, T, d] tensor with a contiguous head dimension")
    return (t.stride(0), t.stride(1), t.stride(2))


def params(q, k, v=None, o=None, *, n_start=0, window=0, L_pretrain=0, topk=0, rope_theta=0.0,
           with_separators=False, rope_pos_scale=1.0, alibi=False) -> SattnParams:
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    p = SattnParams()
    p.B, p.Hq, p.Hkv, p.T, p.d = B, Hq, Hkv, T, d
    p.dtype = _dtype_code(q)
    for name, t in (("q_stride", q), ("k_stride", k), ("v_stride", v), ("o_stride", o if o is not None else q)):
        s = _strides(t)
        arr = getattr(p, name)
        arr[0], arr[1], arr[2] = s
    p.n_start, p.window, p.L_pretrain, p.topk = int(n_start), int(window), int(L_pretrain), int(topk)
    p.with_separators = 1 if with_separators else 0
    p.rope_theta = float(rope_theta)
    p.rope_pos_scale = float(rope_pos_scale)
    p.alibi = 1 if alibi else 0
    return p


def workspace_size(p: SattnParams) -> int:
    n = ctypes.c_size_t(0)
    _lib.check(_lib.load().sattn_workspace_size(ctypes.byref(p), ctypes.byref(n)), "sattn_workspace_size")
    return int(n.value)


def segment_workspace_size(p: SattnParams, S, M, R, retr_block, is_long) -> int:
    n = ctypes.c_size_t(0)
    il = None if is_long is None else (ctypes.c_uint8 * len(is_long))(*[int(x) for x in is_long])
    _lib.check(_lib.load().sattn_segment_workspace_size(ctypes.byref(p), S, M, R, retr_block, il, ctypes.byref(n)),
               "sattn_segment_workspace_size")
    return int(n.value)


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor]) -> torch.Tensor:
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError("workspace too small: need %d bytes" % nbytes)
        return workspace
    key = (str(device), nbytes)
    ws = _ws_cache.get(key)
    if ws is None:
        _ws_cache.clear()  # keep one buffer per process
        ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def _to_dev(t, device):
    if t is None:
        return None
    return t.to(device, non_blocking=True)


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, n_start: int = 0, window: int = 0,
        L_pretrain: int = 0, rope_theta: float = 0.0, topk: int = 0, is_sep: Optional[torch.Tensor] = None,
        topk_idx: Optional[torch.Tensor] = None, topk_logit: Optional[torch.Tensor] = None,
        out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
        workspace: Optional[torch.Tensor] = None, rope_pos_scale: float = 1.0, alibi: bool = False):
    """Structured-mask attention forward.  Returns (O [B,Hq,T,d], lse [B,Hq,T] fp32).
    rope_pos_scale < 1 is position interpolation (rotary positions scaled);
    alibi adds the (clipped) ALiBi bias instead of rotating (rope_theta = 0)."""
    if not q.is_cuda:
        return _host_call(fwd, (q, k, v), dict(n_start=n_start, window=window, L_pretrain=L_pretrain,
                                               rope_theta=rope_theta, topk=topk, is_sep=is_sep,
                                               topk_idx=topk_idx, topk_logit=topk_logit,
                                               rope_pos_scale=rope_pos_scale, alibi=alibi))
    B, Hq, T, d = q.shape
    if out is None:
        out = torch.empty((B, Hq, T, d), dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    if is_sep is not None:
        is_sep = is_sep.to(torch.uint8).contiguous()
    p = params(q, k, v, out, n_start=n_start, window=window, L_pretrain=L_pretrain, topk=topk,
               rope_theta=rope_theta, with_separators=is_sep is not None, rope_pos_scale=rope_pos_scale,
               alibi=alibi)
    nbytes = workspace_size(p)
    ws = _workspace(nbytes, q.device, workspace)
    rc = _lib.load().sattn_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(is_sep), _ptr(topk_idx),
                               _ptr(topk_logit), _ptr(out), _ptr(lse), _ptr(ws), nbytes, _stream_ptr(q.device))
    _lib.check(rc, "sattn_fwd")
    return out, lse


def topk_select(q: torch.Tensor, k: torch.Tensor, *, topk: int, n_start: int = 0, window: int = 0,
                L_pretrain: int = 0, rope_theta: float = 0.0, is_sep: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None, rope_pos_scale: float = 1.0, alibi: bool = False):
    """Per-head top-k middle tokens.  Returns (idx [B,Hq,T,k] int32, logit [B,Hq,T,k] fp32)."""
    B, Hq, T, d = q.shape
    idx = torch.empty((B, Hq, T, topk), dtype=torch.int32, device=q.device)
    logit = torch.empty((B, Hq, T, topk), dtype=torch.float32, device=q.device)
    if is_sep is not None:
        is_sep = is_sep.to(torch.uint8).contiguous()
    p = params(q, k, k, q, n_start=n_start, window=window, L_pretrain=L_pretrain, topk=topk,
               rope_theta=rope_theta, with_separators=is_sep is not None, rope_pos_scale=rope_pos_scale,
               alibi=alibi)
    nbytes = workspace_size(p)
    ws = _workspace(nbytes, q.device, workspace)
    rc = _lib.load().sattn_topk_select(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(is_sep), _ptr(idx), _ptr(logit),
                                       _ptr(ws), nbytes, _stream_ptr(q.device))
    _lib.check(rc, "sattn_topk_select")
    return idx, logit


def build_blockmap(is_sep: Optional[torch.Tensor], *, B: int, T: int, n_start: int, window: int,
                   device="cuda", with_classes: bool = True, workspace: Optional[torch.Tensor] = None):
    """Block map + separator compaction for [B, T] flags (None = no separators)."""
    nqt = (T + TILE - 1) // TILE
    dummy = torch.empty((B, 1, T, 64), dtype=torch.bfloat16, device=device)
    p = params(dummy, dummy, dummy, dummy, n_start=n_start, window=window, with_separators=True)
    if is_sep is not None:
        is_sep = is_sep.to(torch.uint8).contiguous()
    cls = torch.empty((B, nqt, nqt), dtype=torch.uint8, device=device) if with_classes else None
    sep_pos = torch.empty((B, T), dtype=torch.int32, device=device)
    sep_count = torch.empty((B,), dtype=torch.int32, device=device)
    ranges = torch.empty((B, nqt, 2), dtype=torch.int32, device=device)
    nbytes = workspace_size(p)
    ws = _workspace(nbytes, device, workspace)
    rc = _lib.load().sattn_build_blockmap(ctypes.byref(p), _ptr(is_sep), _ptr(cls), _ptr(sep_pos), _ptr(sep_count),
                                          _ptr(ranges), _ptr(ws), nbytes, _stream_ptr(sep_pos.device))
    _lib.check(rc, "sattn_build_blockmap")
    return {"cls": cls, "sep_pos": sep_pos, "sep_count": sep_count, "qtile_sep_range": ranges}


def build_blockmap_noalloc(is_sep: Optional[torch.Tensor], *, B: int, T: int, n_start: int, window: int,
                           device="cuda", with_classes: bool = True):
    """``build_blockmap`` through ``sattn_build_blockmap_noalloc``: the library
    keeps the scratch in its own fixed device array, so no workspace is
    passed (the outputs are still allocated here, by the caller)."""
    nqt = (T + TILE - 1) // TILE
    dummy = torch.empty((B, 1, T, 64), dtype=torch.bfloat16, device=device)
    p = params(dummy, dummy, dummy, dummy, n_start=n_start, window=window, with_separators=True)
    if is_sep is not None:
        is_sep = is_sep.to(torch.uint8).contiguous()
    cls = torch.empty((B, nqt, nqt), dtype=torch.uint8, device=device) if with_classes else None
    sep_pos = torch.empty((B, T), dtype=torch.int32, device=device)
    sep_count = torch.empty((B,), dtype=torch.int32, device=device)
    ranges = torch.empty((B, nqt, 2), dtype=torch.int32, device=device)
    rc = _lib.load().sattn_build_blockmap_noalloc(ctypes.byref(p), _ptr(is_sep), _ptr(cls), _ptr(sep_pos),
                                                  _ptr(sep_count), _ptr(ranges), _stream_ptr(sep_pos.device))
    _lib.check(rc, "sattn_build_blockmap_noalloc")
    return {"cls": cls, "sep_pos": sep_pos, "sep_count": sep_count, "qtile_sep_range": ranges}


def segment_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, S: int, M: int, R: int, retr_block: int,
                is_long, rope_theta: float = 0.0, out: Optional[torch.Tensor] = None,
                lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                rope_pos_scale: float = 1.0):
    """Segmented execution of one layer.  Returns (O, lse, prefix_blocks [B,Hq,T/S,R/retr_block])."""
    if not q.is_cuda:
        return _host_call(segment_fwd, (q, k, v), dict(S=S, M=M, R=R, retr_block=retr_block, is_long=is_long,
                                                       rope_theta=rope_theta, rope_pos_scale=rope_pos_scale))
    B, Hq, T, d = q.shape
    if out is None:
        out = torch.empty((B, Hq, T, d), dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    nb = R // retr_block if retr_block > 0 else 0
    prefix = torch.empty((B, Hq, T // S, max(nb, 1)), dtype=torch.int32, device=q.device)
    il_list = [int(x) for x in (is_long.tolist() if hasattr(is_long, "tolist") else is_long)]
    il = (ctypes.c_uint8 * Hq)(*il_list)
    p = params(q, k, v, out, rope_theta=rope_theta, rope_pos_scale=rope_pos_scale)
    nbytes = segment_workspace_size(p, S, M, R, retr_block, il_list)
    ws = _workspace(nbytes, q.device, workspace)
    rc = _lib.load().sattn_segment_fwd(ctypes.byref(p), S, M, R, retr_block, il, _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                       _ptr(lse), _ptr(prefix), _ptr(ws), nbytes, _stream_ptr(q.device))
    _lib.check(rc, "sattn_segment_fwd")
    return out, lse, prefix[..., :nb]


class SegmentStream:
    """Segmented execution of one layer one segment at a time, the carried
    part (every earlier token's K and V, their rotated keys, the previous
    segment's last query) in a device state buffer.  ``step(q, k, v)`` takes
    the next segment's [B, H, S, d] inputs and returns its (O, lse,
    prefix_blocks [B, Hq, R / retr_block]); steps 0 .. N-1 give what
    ``segment_fwd`` gives on the concatenated segments."""

    def __init__(self, *, B: int, Hq: int, Hkv: int, d: int, capacity: int, S: int, M: int, R: int,
                 retr_block: int, is_long, rope_theta: float = 0.0, rope_pos_scale: float = 1.0, device="cuda"):
        self.B, self.Hq, self.Hkv, self.d, self.capacity = B, Hq, Hkv, d, capacity
        self.S, self.M, self.R, self.retr_block = S, M, R, retr_block
        self.rope_theta, self.rope_pos_scale = float(rope_theta), float(rope_pos_scale)
        self.device = torch.device(device)
        il = [int(x) for x in (is_long.tolist() if hasattr(is_long, "tolist") else is_long)]
        if len(il) != Hq:
            raise ValueError("is_long needs one flag per query head")
        self.is_long = (ctypes.c_uint8 * Hq)(*il)
        p = self._params()
        n = ctypes.c_size_t(0)
        L = _lib.load()
        _lib.check(L.sattn_segment_state_size(ctypes.byref(p), S, M, R, retr_block, ctypes.byref(n)),
                   "sattn_segment_state_size")
        self.state = torch.empty(int(n.value), dtype=torch.uint8, device=self.device)
        _lib.check(L.sattn_segment_step_workspace_size(ctypes.byref(p), S, M, R, retr_block, self.is_long,
                                                       ctypes.byref(n)), "sattn_segment_step_workspace_size")
        self.workspace = torch.empty(max(int(n.value), 256), dtype=torch.uint8, device=self.device)
        self.reset()

    def _params(self, q=None, k=None, v=None, o=None) -> SattnParams:
        if q is None:
            p = SattnParams()
            p.B, p.Hq, p.Hkv, p.d = self.B, self.Hq, self.Hkv, self.d
            p.dtype = _lib.DTYPE_BF16
            for name, H in (("q_stride", self.Hq), ("k_stride", self.Hkv), ("v_stride", self.Hkv),
                            ("o_stride", self.Hq)):
                arr = getattr(p, name)
                arr[0], arr[1], arr[2] = H * self.S * self.d, self.S * self.d, self.d
            p.rope_theta, p.rope_pos_scale = self.rope_theta, self.rope_pos_scale
        else:
            p = params(q, k, v, o, rope_theta=self.rope_theta, rope_pos_scale=self.rope_pos_scale)
        p.T = self.capacity
        return p

    def reset(self):
        """Start a new sequence (no segment taken)."""
        p = self._params()
        _lib.check(_lib.load().sattn_segment_state_reset(ctypes.byref(p), self.S, self.M, self.R, self.retr_block,
                                                         _ptr(self.state), self.state.numel(),
                                                         _stream_ptr(self.device)), "sattn_segment_state_reset")
        self.seg = 0

    def step(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: Optional[torch.Tensor] = None,
             lse: Optional[torch.Tensor] = None, seg: Optional[int] = None):
        """The next segment (or segment ``seg``; a step that is not the next
        one writes nothing and leaves an error in the status word)."""
        B, Hq, S, d = q.shape
        if S != self.S:
            raise ValueError("a step takes one segment of S = %d positions" % self.S)
        if out is None:
            out = torch.empty((B, Hq, S, d), dtype=q.dtype, device=q.device)
        if lse is None:
            lse = torch.empty((B, Hq, S), dtype=torch.float32, device=q.device)
        nb = self.R // self.retr_block
        prefix = torch.empty((B, Hq, max(nb, 1)), dtype=torch.int32, device=q.device)
        p = self._params(q, k, v, out)
        s = self.seg if seg is None else int(seg)
        rc = _lib.load().sattn_segment_step(ctypes.byref(p), self.S, self.M, self.R, self.retr_block, self.is_long, s,
                                            _ptr(q), _ptr(k), _ptr(v), _ptr(self.state), self.state.numel(),
                                            _ptr(out), _ptr(lse), _ptr(prefix), _ptr(self.workspace),
                                            self.workspace.numel(), _stream_ptr(q.device))
        _lib.check(rc, "sattn_segment_step")
        if seg is None:
            self.seg += 1
        return out, lse, prefix[..., :nb]

    def status(self) -> int:
        """Synchronise and read the status word of the last step."""
        return stream_status(self.workspace)


def segment_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
                prefix_blocks: torch.Tensor, do: torch.Tensor, *, S: int, M: int, R: int, retr_block: int, is_long,
                rope_theta: float = 0.0, rope_pos_scale: float = 1.0, workspace: Optional[torch.Tensor] = None,
                grads: Optional[tuple] = None):
    """Backward pass of ``segment_fwd``: gradients of sum(do * o), the
    forward's retrieval (``prefix_blocks``) held fixed.  Returns (dq, dk, dv)
    shaped and strided like q, k, v."""
    if do.stride() != o.stride() or do.dtype != o.dtype or do.shape != o.shape:
        raise ValueError("do must match o in shape, dtype and strides")
    dq, dk, dv = grads if grads is not None else (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    for g, x in ((dq, q), (dk, k), (dv, v)):
        if g.stride() != x.stride():
            raise ValueError("gradient buffers must share the strides of their inputs")
    il_list = [int(x) for x in (is_long.tolist() if hasattr(is_long, "tolist") else is_long)]
    il = (ctypes.c_uint8 * len(il_list))(*il_list)
    p = params(q, k, v, o, rope_theta=rope_theta, rope_pos_scale=rope_pos_scale)
    n = ctypes.c_size_t(0)
    L = _lib.load()
    _lib.check(L.sattn_segment_bwd_workspace_size(ctypes.byref(p), S, M, R, retr_block, ctypes.byref(n)),
               "sattn_segment_bwd_workspace_size")
    nbytes = int(n.value)
    ws = _workspace(nbytes, q.device, workspace)
    pb = prefix_blocks.to(torch.int32).contiguous()
    rc = L.sattn_segment_bwd(ctypes.byref(p), S, M, R, retr_block, il, _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                             _ptr(lse), _ptr(pb), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), nbytes,
                             _stream_ptr(q.device))
    _lib.check(rc, "sattn_segment_bwd")
    return dq, dk, dv


def decode_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, n_start: int = 0, window: int = 0,
               L_pretrain: int = 0, rope_theta: float = 0.0, is_sep: Optional[torch.Tensor] = None,
               out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None, rope_pos_scale: float = 1.0, alibi: bool = False,
               topk: int = 0, return_topk: bool = False):
    """One decoding step: q [B, Hq, 1, d] is the query of the cache's last
    position (k, v [B, Hkv, T, d]).  Returns (O [B, Hq, 1, d], lse [B, Hq]);
    with topk > 0 the query's top-k middle tokens join its key set, and
    return_topk adds their (idx [B, Hq, topk] int32, logit [B, Hq, topk])."""
    B, Hq, one, d = q.shape
    if one != 1:
        raise ValueError("decode_fwd takes one query per (batch, head): q is [B, Hq, 1, d]")
    T = k.shape[2]
    if out is None:
        out = torch.empty((B, Hq, 1, d), dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if is_sep is not None:
        is_sep = is_sep.to(torch.uint8).contiguous()
    p = params(q, k, v, out, n_start=n_start, window=window, L_pretrain=L_pretrain, rope_theta=rope_theta,
               topk=topk, with_separators=is_sep is not None, rope_pos_scale=rope_pos_scale, alibi=alibi)
    p.T = T
    n = ctypes.c_size_t(0)
    L = _lib.load()
    _lib.check(L.sattn_decode_workspace_size(ctypes.byref(p), ctypes.byref(n)), "sattn_decode_workspace_size")
    nbytes = int(n.value)
    ws = _workspace(nbytes, q.device, workspace)
    idx = z = None
    if return_topk:
        if topk < 1:
            raise ValueError("return_topk needs topk > 0")
        idx = torch.empty((B, Hq, topk), dtype=torch.int32, device=q.device)
        z = torch.empty((B, Hq, topk), dtype=torch.float32, device=q.device)
    rc = L.sattn_decode_topk_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(is_sep), _ptr(out), _ptr(lse),
                                 _ptr(idx), _ptr(z), _ptr(ws), nbytes, _stream_ptr(q.device))
    _lib.check(rc, "sattn_decode_topk_fwd")
    return (out, lse, idx, z) if return_topk else (out, lse)


def bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
        do: torch.Tensor, *, n_start: int = 0, window: int = 0, L_pretrain: int = 0, rope_theta: float = 0.0,
        topk: int = 0, is_sep: Optional[torch.Tensor] = None, topk_idx: Optional[torch.Tensor] = None,
        workspace: Optional[torch.Tensor] = None, rope_pos_scale: float = 1.0, alibi: bool = False,
        grads: Optional[tuple] = None):
    """Backward pass of ``fwd``: gradients of sum(do * o) for the forward's
    inputs and outputs.  ``topk_idx`` is the forward's selection (needed when
    topk > 0).  Returns (dq, dk, dv), shaped and strided like q, k, v (written
    into ``grads`` when given)."""
    if do.stride() != o.stride() or do.dtype != o.dtype or do.shape != o.shape:
        raise ValueError("do must match o in shape, dtype and strides")
    dq, dk, dv = grads if grads is not None else (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    for g, x in ((dq, q), (dk, k), (dv, v)):
        if g.stride() != x.stride():
            raise ValueError("gradient buffers must share the strides of their inputs")
    if is_sep is not None:
        is_sep = is_sep.to(torch.uint8).contiguous()
    if topk_idx is not None:
        topk_idx = topk_idx.to(torch.int32).contiguous()
    p = params(q, k, v, o, n_start=n_start, window=window, L_pretrain=L_pretrain, topk=topk, rope_theta=rope_theta,
               with_separators=is_sep is not None, rope_pos_scale=rope_pos_scale, alibi=alibi)
    n = ctypes.c_size_t(0)
    L = _lib.load()
    _lib.check(L.sattn_bwd_workspace_size(ctypes.byref(p), ctypes.byref(n)), "sattn_bwd_workspace_size")
    nbytes = int(n.value)
    ws = _workspace(nbytes, q.device, workspace)
    rc = L.sattn_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(is_sep), _ptr(topk_idx), _ptr(o), _ptr(lse),
                     _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), nbytes, _stream_ptr(q.device))
    _lib.check(rc, "sattn_bwd")
    return dq, dk, dv


def tree_cross_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, n_chunks: int, chunk_len: int, depth: int,
                   alpha_leaf: int = 1, rope_theta: float = 0.0, rope_pos_scale: float = 1.0,
                   out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, with_index: bool = False):
    """SharedLLM tree cross-attention: queries q [B, Hq, T, d] over the
    compressed context k, v [B, Hkv, n_chunks * chunk_len, d].  Returns
    (O, lse) or, with ``with_index``, (O, lse, kept offsets within a chunk)."""
    B, Hq, T, d = q.shape
    if k.shape[2] != n_chunks * chunk_len or v.shape[2] != k.shape[2]:
        raise ValueError("k, v must hold n_chunks * chunk_len context rows")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    p = params(q, k, v, out, rope_theta=rope_theta, rope_pos_scale=rope_pos_scale)
    n = ctypes.c_size_t(0)
    L = _lib.load()
    _lib.check(L.sattn_tree_cross_workspace_size(ctypes.byref(p), n_chunks, chunk_len, depth, alpha_leaf,
                                                 ctypes.byref(n)), "sattn_tree_cross_workspace_size")
    nbytes = int(n.value)
    ws = _workspace(nbytes, q.device, workspace)
    idx = torch.full((chunk_len,), -1, dtype=torch.int32, device=q.device) if with_index else None
    rc = L.sattn_tree_cross_fwd(ctypes.byref(p), n_chunks, chunk_len, depth, alpha_leaf, _ptr(q), _ptr(k), _ptr(v),
                                _ptr(out), _ptr(lse), _ptr(idx), _ptr(ws), nbytes, _stream_ptr(q.device))
    _lib.check(rc, "sattn_tree_cross_fwd")
    if with_index:
        return out, lse, idx
    return out, lse


class StreamKV:
    """SepLLM's streaming KV cache (Initial | Separator | Past | Local) for B
    sequences, its state in device memory.  ``append`` adds one token per
    sequence (compacting on the device when the capacity is reached);
    ``decode`` is one step of the newest tokens' queries over the cache with
    rolled positions."""

    def __init__(self, B: int, Hkv: int, d: int, a: int, s: int, w: int, c: int, device="cuda"):
        self.cfg = _lib.StreamConfig(B, Hkv, d, a, s, w, c)
        self.device = torch.device(device)
        n = ctypes.c_size_t(0)
        L = _lib.load()
        _lib.check(L.sattn_stream_state_size(ctypes.byref(self.cfg), ctypes.byref(n)), "sattn_stream_state_size")
        self.nbytes = int(n.value)
        self.state = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=self.device)
        off = (-self.state.data_ptr()) % 256
        self.state = self.state[off:off + self.nbytes]
        self.position = 0
        self.reset()

    def reset(self):
        _lib.check(_lib.load().sattn_stream_reset(ctypes.byref(self.cfg), _ptr(self.state), self.nbytes,
                                                  _stream_ptr(self.device)), "sattn_stream_reset")
        self.position = 0

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, is_sep: Optional[torch.Tensor] = None):
        """k_new, v_new [B, Hkv, d] bf16 (keys unrotated); is_sep [B] (0/1)."""
        k_new, v_new = k_new.contiguous(), v_new.contiguous()
        if is_sep is not None:
            is_sep = is_sep.to(torch.uint8).contiguous()
        rc = _lib.load().sattn_stream_append(ctypes.byref(self.cfg), _ptr(self.state), self.nbytes, _ptr(k_new),
                                             _ptr(v_new), _ptr(is_sep), self.position, _stream_ptr(self.device))
        _lib.check(rc, "sattn_stream_append")
        self.position += 1

    def read(self):
        """(sizes [B, 4] Initial/Separator/Past/Local, stream position per slot [B, c]) as numpy."""
        import numpy as np
        sizes = np.zeros((self.cfg.B, 4), dtype=np.int32)
        pos = np.zeros((self.cfg.B, self.cfg.c), dtype=np.int32)
        rc = _lib.load().sattn_stream_read(ctypes.byref(self.cfg), _ptr(self.state), self.nbytes,
                                           sizes.ctypes.data_as(ctypes.c_void_p), pos.ctypes.data_as(ctypes.c_void_p),
                                           _stream_ptr(self.device))
        _lib.check(rc, "sattn_stream_read")
        return sizes, pos

    def decode(self, q: torch.Tensor, rope_theta: float = 0.0, rope_pos_scale: float = 1.0,
               out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None):
        """q [B, Hq, 1, d] bf16 -> (O [B, Hq, 1, d], lse [B, Hq])."""
        B, Hq, one, d = q.shape
        if out is None:
            out = torch.empty_like(q)
        if lse is None:
            lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        p = _lib.SattnParams()
        p.B, p.Hq, p.Hkv, p.T, p.d = B, Hq, self.cfg.Hkv, self.cfg.c, d
        p.dtype = _dtype_code(q)
        for name, t in (("q_stride", q), ("o_stride", out)):
            st = _strides(t)
            arr = getattr(p, name)
            arr[0], arr[1], arr[2] = st
        p.rope_theta = float(rope_theta)
        p.rope_pos_scale = float(rope_pos_scale)
        n = ctypes.c_size_t(0)
        L = _lib.load()
        _lib.check(L.sattn_stream_decode_workspace_size(ctypes.byref(self.cfg), ctypes.byref(p), ctypes.byref(n)),
                   "sattn_stream_decode_workspace_size")
        nbytes = int(n.value)
        ws = _workspace(nbytes, q.device, workspace)
        rc = L.sattn_stream_decode(ctypes.byref(self.cfg), ctypes.byref(p), _ptr(self.state), self.nbytes, _ptr(q),
                                   _ptr(out), _ptr(lse), _ptr(ws), nbytes, _stream_ptr(q.device))
        _lib.check(rc, "sattn_stream_decode")
        return out, lse


def stream_status(workspace: Optional[torch.Tensor] = None, device="cuda") -> int:
    """Synchronise the current stream and read the device status word of the
    workspace (the cached one when None)."""
    if workspace is None:
        if not _ws_cache:
            return 0
        workspace = next(iter(_ws_cache.values()))
    st = ctypes.c_int32(0)
    _lib.check(_lib.load().sattn_stream_status(_stream_ptr(workspace.device), _ptr(workspace), ctypes.byref(st)),
               "sattn_stream_status")
    return int(st.value)


_copy_streams: dict = {}


def _copy_stream_pair(dev):
    """(host-to-device stream, device-to-host stream) of a device."""
    st = _copy_streams.get(dev)
    if st is None:
        st = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
        _copy_streams[dev] = st
    return st


def selftest_wait_timeout(limit_ms: float = 20.0, device="cuda") -> tuple:
    """Run the library's bounded-wait failure path: a kernel waits on a
    barrier nothing arrives at and gives up after ``limit_ms``.  Returns
    (status, site) read back from a fresh workspace's status word; the
    expected result is (SATTN_ERR_TIMEOUT, 99) with the CUDA context intact."""
    ws = torch.empty(256, dtype=torch.uint8, device=device)
    st = _stream_ptr(ws.device)
    _lib.check(_lib.load().sattn_selftest_wait_timeout(_ptr(ws), 256, int(limit_ms * 1e6), st),
               "sattn_selftest_wait_timeout")
    status = stream_status(ws)
    site = int(ws[4:8].view(torch.int32).item())
    return status, site


def _host_chunks(B: int, Hkv: int, n: int):
    """About n independent pieces of a problem, as (b0, b1, kv0, kv1): batch
    ranges, each cut into groups of kv heads (whole GQA groups) when there
    are fewer sequences than pieces."""
    nb = min(n, B)
    nh = min(max(1, n // nb), Hkv)
    return [(B * i // nb, B * (i + 1) // nb, Hkv * j // nh, Hkv * (j + 1) // nh)
            for i in range(nb) for j in range(nh)]


def _host_call(fn, tensors, kw, n_chunks: int = 8):
    """Host tensors in, host tensors out: the end-to-end path.

    Sequences and groups of kv heads are independent, so the problem is cut
    into about n_chunks pieces: one copy stream moves piece c+1 to the device
    while the compute stream runs piece c, and a second copy stream brings
    each piece's results back as soon as they are ready (the two directions
    overlap).  Outputs land in pinned host memory; the result equals the
    one-piece call bit for bit."""
    dev = torch.device("cuda", torch.cuda.current_device())
    q, k, v = tensors
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    rep = Hq // Hkv
    compute = torch.cuda.current_stream(dev)
    copy, back = _copy_stream_pair(dev)
    copy.wait_stream(compute)  # device buffers below are allocated on the compute stream
    dq, dk, dv = (torch.empty(t.shape, dtype=t.dtype, device=dev) for t in (q, k, v))
    kw = dict(kw)
    side = {name: kw.pop(name) for name in ("is_sep", "topk_idx", "topk_logit") if kw.get(name) is not None}
    dside = {name: torch.empty(t.shape, dtype=t.dtype, device=dev) for name, t in side.items()}
    outs_host = None
    res_keep = []
    for b0, b1, x0, x1 in _host_chunks(B, Hkv, n_chunks):
        sl_q = (slice(b0, b1), slice(x0 * rep, x1 * rep))
        sl_kv = (slice(b0, b1), slice(x0, x1))
        sl_side = (slice(b0, b1),)
        with torch.cuda.stream(copy):
            for src, dst, sl in ((q, dq, sl_q), (k, dk, sl_kv), (v, dv, sl_kv)):
                dst[sl].copy_(src[sl], non_blocking=True)
            for name, t in side.items():
                if name == "is_sep":
                    if x0 == 0:  # flags are per sequence, shared by the head pieces
                        dside[name][sl_side].copy_(t[sl_side], non_blocking=True)
                else:
                    dside[name][sl_q].copy_(t[sl_q], non_blocking=True)
            ready = torch.cuda.Event()
            ready.record(copy)
        compute.wait_event(ready)
        ckw = dict(kw)
        for name, t in dside.items():
            ckw[name] = t[sl_side] if name == "is_sep" else t[sl_q]
        if "is_long" in ckw:
            ckw["is_long"] = list(ckw["is_long"])[x0 * rep:x1 * rep]
        res = fn(dq[sl_q], dk[sl_kv], dv[sl_kv], **ckw)
        done = torch.cuda.Event()
        done.record(compute)
        if outs_host is None:
            shapes = [(B, Hq) + tuple(r.shape[2:]) for r in res]
            outs_host = tuple(torch.empty(sh, dtype=r.dtype, pin_memory=True) for sh, r in zip(shapes, res))
        back.wait_event(done)
        with torch.cuda.stream(back):
            for oh, r in zip(outs_host, res):
                oh[sl_q].copy_(r, non_blocking=True)
        res_keep.append(res)  # device results stay alive until the copies finish
    back.synchronize()
    copy.synchronize()
    compute.synchronize()
    return outs_host
