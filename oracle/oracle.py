"""ctypes front end of the fp64 CPU oracle (``sattn_oracle.c``).

TEST INFRASTRUCTURE ONLY.  The product library never imports this module;
only the tests, the smoke check and the CPU-baseline leg of the benchmark do.
It builds ``liboracle.so`` with gcc on first use (or via :func:`build`).

Parity status of each function (pins live in ``tests/test_oracle_pins.py``):
  decode_bf16     pinned: hand-computed IEEE values
  rope / logit    pinned: 2-D rotation closed form, relative-position
                  identity, cap = shifted-distance identity
  mask_row        pinned: hand-written golden masks from the pages'
                  definitions, closed-form set sizes (brute force T <= 12)
  fwd_rows        pinned: full causal / sliding window equal torch SDPA;
                  rows sum to one; invariance outside the kept set;
                  top-k with k >= #middle equals full causal; planted keys
  blockmap        pinned: numpy nonzero / searchsorted, interval geometry
  segment_rows    pinned: S = T gives causal; R = whole previous segment
                  gives causal over two segments; effective-context count
  bwd, bwd_dq_rows, bwd_dkv_keys
                  pinned: central finite differences of the pinned forward,
                  autograd through fp64 SDPA, sum dV = sum dO; the rows and
                  keys entries equal the full backward bit for bit
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sattn_oracle.c")
_LIB = os.environ.get("SATTN_ORACLE_LIB") or os.path.join(_HERE, "liboracle.so")
_SRC = os.environ.get("SATTN_ORACLE_SRC") or _SRC
_lock = threading.Lock()
_lib = None


class OracleParams(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
        ("T", ctypes.c_int32), ("d", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("n_start", ctypes.c_int32), ("window", ctypes.c_int32),
        ("L_pretrain", ctypes.c_int32), ("topk", ctypes.c_int32),
        ("rope_theta", ctypes.c_double), ("rope_pos_scale", ctypes.c_double),
        ("alibi", ctypes.c_int32),
    ]


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` (plain C, fp64, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            P = ctypes.POINTER
            L.oracle_decode_bf16.restype = ctypes.c_double
            L.oracle_decode_bf16.argtypes = [ctypes.c_uint16]
            L.oracle_rope.restype = None
            L.oracle_rope.argtypes = [P(ctypes.c_double), ctypes.c_int, ctypes.c_double,
                                      ctypes.c_double, P(ctypes.c_double)]
            L.oracle_logit.restype = ctypes.c_double
            L.oracle_logit.argtypes = [P(ctypes.c_double), P(ctypes.c_double), ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double]
            L.oracle_mask_row.restype = ctypes.c_int64
            L.oracle_mask_row.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_void_p, ctypes.c_void_p]
            L.oracle_fwd_rows.restype = ctypes.c_int
            L.oracle_fwd_rows.argtypes = [P(OracleParams)] + [ctypes.c_void_p] * 4 + [
                ctypes.c_int64] + [ctypes.c_void_p] * 7 + [ctypes.c_int]
            L.oracle_tree_index.restype = ctypes.c_int
            L.oracle_tree_index.argtypes = [ctypes.c_int] * 3 + [ctypes.c_void_p]
            L.oracle_tree_cross.restype = ctypes.c_int
            L.oracle_tree_cross.argtypes = [P(OracleParams)] + [ctypes.c_int] * 4 + [ctypes.c_void_p] * 5 + [
                ctypes.c_int]
            L.oracle_bwd.restype = ctypes.c_int
            L.oracle_bwd.argtypes = [P(OracleParams)] + [ctypes.c_void_p] * 9 + [ctypes.c_int]
            L.oracle_bwd_dq_rows.restype = ctypes.c_int
            L.oracle_bwd_dq_rows.argtypes = [P(OracleParams)] + [ctypes.c_void_p] * 6 + [
                ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
            L.oracle_bwd_dkv_keys.restype = ctypes.c_int
            L.oracle_bwd_dkv_keys.argtypes = [P(OracleParams)] + [ctypes.c_void_p] * 6 + [
                ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
            L.oracle_blockmap.restype = ctypes.c_int
            L.oracle_blockmap.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p] * 5
            L.oracle_segment_rows.restype = ctypes.c_int
            L.oracle_segment_rows.argtypes = [P(OracleParams)] + [ctypes.c_int] * 4 + [
                ctypes.c_void_p] * 4 + [ctypes.c_int64] + [ctypes.c_void_p] * 4 + [ctypes.c_int]
            L.oracle_segment_bwd.restype = ctypes.c_int
            L.oracle_segment_bwd.argtypes = [P(OracleParams)] + [ctypes.c_int] * 4 + [ctypes.c_void_p] * 8 + [
                ctypes.c_int]
            L.oracle_segment_blocks.restype = ctypes.c_int
            L.oracle_segment_blocks.argtypes = [P(OracleParams)] + [ctypes.c_int] * 3 + [
                ctypes.c_void_p] * 5
            L.oracle_segment_keys.restype = ctypes.c_int
            L.oracle_segment_keys.argtypes = [P(OracleParams)] + [ctypes.c_int] * 4 + [
                ctypes.c_void_p] * 3 + [ctypes.c_int] * 3 + [ctypes.c_void_p] * 3
            _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype=None):
    if a is None:
        return None
    return np.ascontiguousarray(a if dtype is None else a.astype(dtype, copy=False))


def nthreads_default() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def params(B, Hq, Hkv, T, d, dtype="bf16", n_start=0, window=0, L_pretrain=0, topk=0,
           rope_theta=0.0, rope_pos_scale=1.0, alibi=False) -> OracleParams:
    return OracleParams(B, Hq, Hkv, T, d, 0 if dtype == "bf16" else 1, n_start, window,
                        L_pretrain, topk, float(rope_theta), float(rope_pos_scale), int(bool(alibi)))


def params_of(wl) -> OracleParams:
    return params(wl.B, wl.Hq, wl.Hkv, wl.T, wl.d, wl.dtype, wl.n_start, wl.window,
                  wl.L_pretrain, wl.topk, wl.rope_theta, wl.rope_pos_scale, wl.alibi)


def _inputs(p: OracleParams, q, k, v):
    if p.dtype == 0:
        return _c(q, np.uint16), _c(k, np.uint16), _c(v, np.uint16)
    return _c(q, np.float32), _c(k, np.float32), _c(v, np.float32)


def decode_bf16(bits: int) -> float:
    return lib().oracle_decode_bf16(int(bits) & 0xFFFF)


def rope(x, pos, theta):
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty_like(x)
    P = ctypes.POINTER(ctypes.c_double)
    lib().oracle_rope(x.ctypes.data_as(P), x.shape[-1], float(pos), float(theta), out.ctypes.data_as(P))
    return out


def logit(q, k, i, j, L, theta) -> float:
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    P = ctypes.POINTER(ctypes.c_double)
    return lib().oracle_logit(q.ctypes.data_as(P), k.ctypes.data_as(P), q.shape[-1], int(i), int(j),
                              int(L), float(theta))


def mask_row(T, i, n_start, w, is_sep=None):
    m = np.zeros(T, dtype=np.uint8)
    s = _c(is_sep, np.uint8)
    cnt = lib().oracle_mask_row(T, i, n_start, w, _ptr(s), _ptr(m))
    return m, int(cnt)


def fwd_rows(p: OracleParams, q, k, v, is_sep, rows, forced_topk=None, nthreads=None):
    """Rows ``[(b, h, i)]`` -> (O [n,d], lse [n], topk_idx [n,k], topk_z [n,k], counts [n])."""
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    n = rows.shape[0]
    q, k, v = _inputs(p, q, k, v)
    s = _c(is_sep, np.uint8)
    O = np.zeros((n, p.d), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    kk = max(p.topk, 1)
    tki = np.full((n, kk), -1, dtype=np.int32)
    tkz = np.full((n, kk), -np.inf, dtype=np.float64)
    cnt = np.zeros(n, dtype=np.int64)
    f = _c(forced_topk, np.int32)
    rc = lib().oracle_fwd_rows(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(s), n, _ptr(rows),
                               _ptr(f), _ptr(O), _ptr(lse), _ptr(tki), _ptr(tkz), _ptr(cnt),
                               nthreads or nthreads_default())
    if rc != 0:
        raise RuntimeError("oracle_fwd_rows failed: %d" % rc)
    return O, lse, tki[:, : p.topk], tkz[:, : p.topk], cnt


def bwd(p: OracleParams, q, k, v, is_sep, dO, forced_topk=None, nthreads=None):
    """Gradients of sum(dO * O): (dQ [B,Hq,T,d], dK [B,Hkv,T,d], dV [B,Hkv,T,d]) in float64.
    dO has the inputs' encoding; forced_topk [B,Hq,T,k] fixes the top-k sets."""
    q, k, v = _inputs(p, q, k, v)
    g = _c(dO, np.uint16 if p.dtype == 0 else np.float32)
    assert g.size == q.size
    s = _c(is_sep, np.uint8)
    f = _c(forced_topk, np.int32)
    dQ = np.zeros((p.B, p.Hq, p.T, p.d), dtype=np.float64)
    dK = np.zeros((p.B, p.Hkv, p.T, p.d), dtype=np.float64)
    dV = np.zeros((p.B, p.Hkv, p.T, p.d), dtype=np.float64)
    rc = lib().oracle_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(s), _ptr(f), _ptr(g), _ptr(dQ),
                          _ptr(dK), _ptr(dV), nthreads or nthreads_default())
    if rc != 0:
        raise RuntimeError("oracle_bwd failed: %d" % rc)
    return dQ, dK, dV


def bwd_dq_rows(p: OracleParams, q, k, v, is_sep, dO, rows, forced_topk=None, nthreads=None):
    """dQ of the rows ``[(b, h, i)]`` alone -> [n, d] float64: the same row
    arithmetic as ``bwd`` (a row's dq depends on that row only), for sizes
    where the full backward is too slow."""
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    q, k, v = _inputs(p, q, k, v)
    g = _c(dO, np.uint16 if p.dtype == 0 else np.float32)
    assert g.size == q.size
    s = _c(is_sep, np.uint8)
    f = _c(forced_topk, np.int32)
    dq = np.zeros((rows.shape[0], p.d), dtype=np.float64)
    rc = lib().oracle_bwd_dq_rows(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(s), _ptr(f), _ptr(g),
                                  rows.shape[0], _ptr(rows), _ptr(dq), nthreads or nthreads_default())
    if rc != 0:
        raise RuntimeError("oracle_bwd_dq_rows failed: %d" % rc)
    return dq


def bwd_dkv_keys(p: OracleParams, q, k, v, is_sep, dO, keys, forced_topk=None, nthreads=None):
    """dK and dV of the keys ``[(b, g, j)]`` (kv head g) alone -> ([n, d], [n, d])
    float64: key j's terms of ``bwd``'s key-side sums over every row of the
    query-head group, summed in the same order, for sizes where the full
    backward is too slow."""
    keys = np.ascontiguousarray(keys, dtype=np.int64).reshape(-1, 3)
    q, k, v = _inputs(p, q, k, v)
    g = _c(dO, np.uint16 if p.dtype == 0 else np.float32)
    assert g.size == q.size
    s = _c(is_sep, np.uint8)
    f = _c(forced_topk, np.int32)
    dk = np.zeros((keys.shape[0], p.d), dtype=np.float64)
    dv = np.zeros((keys.shape[0], p.d), dtype=np.float64)
    rc = lib().oracle_bwd_dkv_keys(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(s), _ptr(f), _ptr(g),
                                   keys.shape[0], _ptr(keys), _ptr(dk), _ptr(dv), nthreads or nthreads_default())
    if rc != 0:
        raise RuntimeError("oracle_bwd_dkv_keys failed: %d" % rc)
    return dk, dv


def tree_index(chunk_len, depth, alpha_leaf) -> np.ndarray:
    """Kept offsets of one context chunk of the tree cross-attention."""
    n = lib().oracle_tree_index(chunk_len, depth, alpha_leaf, None)
    if n < 1:
        raise RuntimeError("oracle_tree_index failed: %d" % n)
    out = np.zeros(n, dtype=np.int32)
    lib().oracle_tree_index(chunk_len, depth, alpha_leaf, _ptr(out))
    return out


def tree_cross(p: OracleParams, n_chunks, chunk_len, depth, alpha_leaf, q, k, v, nthreads=None):
    """Tree cross-attention: (O [B,Hq,T,d], lse [B,Hq,T]) in float64."""
    q, k, v = _inputs(p, q, k, v)
    O = np.zeros((p.B, p.Hq, p.T, p.d), dtype=np.float64)
    lse = np.zeros((p.B, p.Hq, p.T), dtype=np.float64)
    rc = lib().oracle_tree_cross(ctypes.byref(p), n_chunks, chunk_len, depth, alpha_leaf, _ptr(q), _ptr(k), _ptr(v),
                                 _ptr(O), _ptr(lse), nthreads or nthreads_default())
    if rc != 0:
        raise RuntimeError("oracle_tree_cross failed: %d" % rc)
    return O, lse


def all_rows(B, H, T) -> np.ndarray:
    b, h, i = np.meshgrid(np.arange(B), np.arange(H), np.arange(T), indexing="ij")
    return np.stack([b.ravel(), h.ravel(), i.ravel()], axis=1).astype(np.int64)


def blockmap(B, T, n_start, w, BM, BN, is_sep):
    nQT, nKT = -(-T // BM), -(-T // BN)
    cls = np.zeros((B, nQT, nKT), dtype=np.uint8)
    sep_pos = np.zeros((B, T), dtype=np.int32)
    cnt = np.zeros(B, dtype=np.int32)
    rng = np.zeros((B, nQT, 2), dtype=np.int32)
    s = _c(is_sep, np.uint8)
    rc = lib().oracle_blockmap(B, T, n_start, w, BM, BN, _ptr(s), _ptr(cls), _ptr(sep_pos), _ptr(cnt),
                               _ptr(rng))
    if rc != 0:
        raise RuntimeError("oracle_blockmap failed: %d" % rc)
    return cls, sep_pos, cnt, rng


def segment_rows(p: OracleParams, S, M, R, blk, is_long, q, k, v, rows, nthreads=None):
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    n = rows.shape[0]
    q, k, v = _inputs(p, q, k, v)
    il = _c(is_long, np.uint8)
    O = np.zeros((n, p.d), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    cnt = np.zeros(n, dtype=np.int64)
    rc = lib().oracle_segment_rows(ctypes.byref(p), S, M, R, blk, _ptr(il), _ptr(q), _ptr(k), _ptr(v), n,
                                   _ptr(rows), _ptr(O), _ptr(lse), _ptr(cnt), nthreads or nthreads_default())
    if rc != 0:
        raise RuntimeError("oracle_segment_rows failed: %d" % rc)
    return O, lse, cnt


def segment_bwd(p: OracleParams, S, M, R, blk, is_long, q, k, v, dO, nthreads=None):
    """Gradients of sum(dO * O) for segmented execution, the retrieval held
    fixed: (dQ [B,Hq,T,d], dK [B,Hkv,T,d], dV [B,Hkv,T,d]) in float64."""
    il = np.ascontiguousarray(np.asarray(is_long, dtype=np.uint8))
    q, k, v = _inputs(p, q, k, v)
    g = _c(dO, np.uint16 if p.dtype == 0 else np.float32)
    assert g.size == q.size
    dQ = np.zeros((p.B, p.Hq, p.T, p.d), dtype=np.float64)
    dK = np.zeros((p.B, p.Hkv, p.T, p.d), dtype=np.float64)
    dV = np.zeros((p.B, p.Hkv, p.T, p.d), dtype=np.float64)
    rc = lib().oracle_segment_bwd(ctypes.byref(p), S, M, R, blk, _ptr(il), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                  _ptr(dQ), _ptr(dK), _ptr(dV), nthreads or nthreads_default())
    if rc != 0:
        raise RuntimeError("oracle_segment_bwd failed: %d" % rc)
    return dQ, dK, dV


def segment_blocks(p: OracleParams, S, R, blk, is_long, q, k):
    N, nb = p.T // S, R // blk
    q, k, _ = _inputs(p, q, k, k)
    il = _c(is_long, np.uint8)
    out = np.zeros((p.B, p.Hq, N, nb), dtype=np.int32)
    sk = np.zeros((p.B, p.Hq, N, 2), dtype=np.float64)
    rc = lib().oracle_segment_blocks(ctypes.byref(p), S, R, blk, _ptr(il), _ptr(q), _ptr(k), _ptr(out), _ptr(sk))
    if rc != 0:
        raise RuntimeError("oracle_segment_blocks failed: %d" % rc)
    return out, sk


def segment_keys(p: OracleParams, S, M, R, blk, is_long, q, k, b, h, i):
    """(key indices, rotary positions, P) of one row in segmented execution."""
    q, k, _ = _inputs(p, q, k, k)
    il = _c(is_long, np.uint8)
    cap = M + R + S + 1
    kj = np.zeros(cap, dtype=np.int32)
    kp = np.zeros(cap, dtype=np.int32)
    P = np.zeros(1, dtype=np.int32)
    n = lib().oracle_segment_keys(ctypes.byref(p), S, M, R, blk, _ptr(il), _ptr(q), _ptr(k), b, h, i,
                                  _ptr(kj), _ptr(kp), _ptr(P))
    if n < 0:
        raise RuntimeError("oracle_segment_keys failed: %d" % n)
    return kj[:n].copy(), kp[:n].copy(), int(P[0])
