"""ctypes loader for ``libsattn.so`` -- the C ABI declared in ``include/sattn.h``.

Loading fails loudly when the library has not been built; there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsattn.so")

SATTN_OK = 0
SATTN_ERR_INVALID_ARG = -1
SATTN_ERR_UNSUPPORTED = -2
SATTN_ERR_CUDA = -3
SATTN_ERR_TIMEOUT = -4
DTYPE_BF16 = 0
DTYPE_F32 = 1

# every function the header declares, in header order
EXPORTS = (
    "sattn_strerror", "sattn_version", "sattn_workspace_size", "sattn_segment_workspace_size",
    "sattn_build_blockmap", "sattn_topk_select", "sattn_fwd", "sattn_segment_fwd",
    "sattn_segment_bwd_workspace_size", "sattn_segment_bwd", "sattn_segment_state_size", "sattn_segment_state_reset",
    "sattn_segment_step_workspace_size", "sattn_segment_step",
    "sattn_decode_workspace_size", "sattn_decode_fwd", "sattn_decode_topk_fwd", "sattn_bwd_workspace_size",
    "sattn_bwd",
    "sattn_tree_cross_workspace_size", "sattn_tree_cross_fwd", "sattn_stream_state_size", "sattn_stream_reset",
    "sattn_stream_append", "sattn_stream_read", "sattn_stream_decode_workspace_size", "sattn_stream_decode",
    "sattn_stream_status",
    "sattn_build_blockmap_noalloc", "sattn_selftest_wait_timeout", "sattn_profile_enable", "sattn_profile_collect",
)


class StreamConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "Hkv", "d", "a", "s", "w", "c")]


class SattnParams(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("T", ctypes.c_int32),
        ("d", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("q_stride", ctypes.c_int64 * 3), ("k_stride", ctypes.c_int64 * 3),
        ("v_stride", ctypes.c_int64 * 3), ("o_stride", ctypes.c_int64 * 3),
        ("n_start", ctypes.c_int32), ("window", ctypes.c_int32), ("L_pretrain", ctypes.c_int32),
        ("topk", ctypes.c_int32), ("with_separators", ctypes.c_int32), ("rope_theta", ctypes.c_double),
        ("rope_pos_scale", ctypes.c_double), ("alibi", ctypes.c_int32), ("tile_m", ctypes.c_int32),
        ("tile_n", ctypes.c_int32),
    ]


class SattnError(RuntimeError):
    def __init__(self, rc: int, what: str):
        super().__init__("%s failed: %s (%d)" % (what, strerror(rc), rc))
        self.rc = rc


_lib = None
_lock = threading.Lock()


def load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                "libsattn.so is not built (expected at %s); run `python -m long_context_structured_b200.build`"
                % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
        P = ctypes.POINTER(SattnParams)
        L.sattn_strerror.restype = ctypes.c_char_p
        L.sattn_strerror.argtypes = [ctypes.c_int]
        L.sattn_version.restype = ctypes.c_int
        L.sattn_version.argtypes = []
        L.sattn_workspace_size.restype = ctypes.c_int
        L.sattn_workspace_size.argtypes = [P, ctypes.POINTER(sz)]
        L.sattn_segment_workspace_size.restype = ctypes.c_int
        L.sattn_segment_workspace_size.argtypes = [P, i32, i32, i32, i32, vp, ctypes.POINTER(sz)]
        L.sattn_build_blockmap.restype = ctypes.c_int
        L.sattn_build_blockmap.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sattn_topk_select.restype = ctypes.c_int
        L.sattn_topk_select.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sattn_fwd.restype = ctypes.c_int
        L.sattn_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sattn_segment_fwd.restype = ctypes.c_int
        L.sattn_segment_fwd.argtypes = [P, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sattn_segment_bwd_workspace_size.restype = ctypes.c_int
        L.sattn_segment_bwd_workspace_size.argtypes = [P, i32, i32, i32, i32, ctypes.POINTER(sz)]
        L.sattn_segment_bwd.restype = ctypes.c_int
        L.sattn_segment_bwd.argtypes = [P, i32, i32, i32, i32] + [vp] * 11 + [vp, sz, vp]
        L.sattn_segment_state_size.restype = ctypes.c_int
        L.sattn_segment_state_size.argtypes = [P, i32, i32, i32, i32, ctypes.POINTER(sz)]
        L.sattn_segment_state_reset.restype = ctypes.c_int
        L.sattn_segment_state_reset.argtypes = [P, i32, i32, i32, i32, vp, sz, vp]
        L.sattn_segment_step_workspace_size.restype = ctypes.c_int
        L.sattn_segment_step_workspace_size.argtypes = [P, i32, i32, i32, i32, vp, ctypes.POINTER(sz)]
        L.sattn_segment_step.restype = ctypes.c_int
        L.sattn_segment_step.argtypes = [P, i32, i32, i32, i32, vp, i32, vp, vp, vp, vp, sz, vp, vp, vp, vp, sz, vp]
        L.sattn_decode_workspace_size.restype = ctypes.c_int
        L.sattn_decode_workspace_size.argtypes = [P, ctypes.POINTER(sz)]
        L.sattn_decode_fwd.restype = ctypes.c_int
        L.sattn_decode_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sattn_decode_topk_fwd.restype = ctypes.c_int
        L.sattn_decode_topk_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sattn_bwd_workspace_size.restype = ctypes.c_int
        L.sattn_bwd_workspace_size.argtypes = [P, ctypes.POINTER(sz)]
        L.sattn_bwd.restype = ctypes.c_int
        L.sattn_bwd.argtypes = [P] + [vp] * 12 + [sz, vp]
        L.sattn_tree_cross_workspace_size.restype = ctypes.c_int
        L.sattn_tree_cross_workspace_size.argtypes = [P, i32, i32, i32, i32, ctypes.POINTER(sz)]
        L.sattn_tree_cross_fwd.restype = ctypes.c_int
        L.sattn_tree_cross_fwd.argtypes = [P, i32, i32, i32, i32] + [vp] * 7 + [sz, vp]
        SC = ctypes.POINTER(StreamConfig)
        L.sattn_stream_state_size.restype = ctypes.c_int
        L.sattn_stream_state_size.argtypes = [SC, ctypes.POINTER(sz)]
        L.sattn_stream_reset.restype = ctypes.c_int
        L.sattn_stream_reset.argtypes = [SC, vp, sz, vp]
        L.sattn_stream_append.restype = ctypes.c_int
        L.sattn_stream_append.argtypes = [SC, vp, sz, vp, vp, vp, ctypes.c_int64, vp]
        L.sattn_stream_read.restype = ctypes.c_int
        L.sattn_stream_read.argtypes = [SC, vp, sz, vp, vp, vp]
        L.sattn_stream_decode_workspace_size.restype = ctypes.c_int
        L.sattn_stream_decode_workspace_size.argtypes = [SC, P, ctypes.POINTER(sz)]
        L.sattn_stream_decode.restype = ctypes.c_int
        L.sattn_stream_decode.argtypes = [SC, P, vp, sz, vp, vp, vp, vp, sz, vp]
        L.sattn_stream_status.restype = ctypes.c_int
        L.sattn_stream_status.argtypes = [vp, vp, ctypes.POINTER(i32)]
        L.sattn_build_blockmap_noalloc.restype = ctypes.c_int
        L.sattn_build_blockmap_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp]
        L.sattn_selftest_wait_timeout.restype = ctypes.c_int
        L.sattn_selftest_wait_timeout.argtypes = [vp, sz, ctypes.c_uint64, vp]
        L.sattn_profile_enable.restype = ctypes.c_int
        L.sattn_profile_enable.argtypes = [ctypes.c_int]
        L.sattn_profile_collect.restype = ctypes.c_int
        L.sattn_profile_collect.argtypes = [ctypes.c_char_p, ctypes.POINTER(i32), ctypes.POINTER(ctypes.c_double), i32,
                                            ctypes.POINTER(i32)]
        _lib = L
        return _lib


def strerror(rc: int) -> str:
    return load().sattn_strerror(int(rc)).decode()


def check(rc: int, what: str) -> None:
    if rc != SATTN_OK:
        raise SattnError(rc, what)
