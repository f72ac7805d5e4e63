"""sattn_build_blockmap_noalloc: the block map for callers that cannot
allocate device memory or pass a workspace (e.g. an extension inside a host
framework that owns all device memory, or a loop where an allocation and the
synchronisation it may bring are not allowed).  Its scratch is a fixed device
array inside the library.

Checked through the C ABI against sattn_build_blockmap (the workspace
version) on two calls in a row with different inputs, so a stale array from
the first call cannot hide.  Outputs are integers: they must match exactly.
This file is collected last so a failure here leaves every other test run.
"""
import ctypes

import numpy as np
import pytest
import torch

from long_context_structured_b200 import _lib

pytestmark = pytest.mark.gpu

MAX_BYTES = 1 << 22


def _scratch_bytes(B, T, window):
    """The scratch size the header states for the no-alloc block map."""
    up16 = lambda x: (x + 15) // 16 * 16
    nqt = (T + 127) // 128
    bt = min(nqt, (window + 127) // 128)
    kc = min((nqt + 15) // 16, bt // 16 + 2)
    return up16(B * 8 * (T // 32 + 1)) + B * up16(nqt) + B * 16 * nqt * kc


def _params(B, T, n_start, window):
    p = _lib.SattnParams()
    p.B, p.Hq, p.Hkv, p.T, p.d, p.dtype = B, 1, 1, T, 64, _lib.DTYPE_BF16
    for name in ("q_stride", "k_stride", "v_stride", "o_stride"):
        arr = getattr(p, name)
        arr[0], arr[1], arr[2] = T * 64, T * 64, 64
    p.n_start, p.window, p.with_separators = n_start, window, 1
    return p


def _outputs(B, T, dev):
    nqt = (T + 127) // 128
    return (torch.full((B, nqt, nqt), 7, dtype=torch.uint8, device=dev),
            torch.full((B, T), -7, dtype=torch.int32, device=dev),
            torch.full((B,), -7, dtype=torch.int32, device=dev),
            torch.full((B, nqt, 2), -7, dtype=torch.int32, device=dev))


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _run_both(lib, B, T, n_start, window, flags, dev):
    p = _params(B, T, n_start, window)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    f = torch.from_numpy(flags).to(dev)
    ref = _outputs(B, T, dev)
    n = ctypes.c_size_t(0)
    assert lib.sattn_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 0
    ws = torch.empty(n.value, dtype=torch.uint8, device=dev)
    assert lib.sattn_build_blockmap(ctypes.byref(p), _ptr(f), *map(_ptr, ref), _ptr(ws), n.value, stream) == 0
    got = _outputs(B, T, dev)
    assert lib.sattn_build_blockmap_noalloc(ctypes.byref(p), _ptr(f), *map(_ptr, got), stream) == 0
    torch.cuda.synchronize(dev)
    for a, b in zip(ref, got):
        assert torch.equal(a, b)


def test_noalloc_matches_workspace_version_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    lib = _lib.load()
    rng = np.random.default_rng(20)
    # first call: c3-like sizes; second: a different shape and rate, so the
    # scratch left by the first call cannot be reused by accident
    flags1 = (rng.random((4, 8192)) < 0.10).astype(np.uint8)
    _run_both(lib, 4, 8192, 4, 256, flags1, dev)
    flags2 = (rng.random((3, 1000)) < 0.4).astype(np.uint8)
    _run_both(lib, 3, 1000, 2, 37, flags2, dev)


@pytest.mark.parametrize("T,window", [(40000, 128), (4096, 5000)])
def test_noalloc_largest_accepted_batch(T, window):
    """The largest batch whose scratch fits the 4 MiB array runs and matches
    the workspace version; one sequence more is refused on the host."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    lib = _lib.load()
    B = 1
    while _scratch_bytes(B + 1, T, window) <= MAX_BYTES:
        B += 1
    rng = np.random.default_rng(T + window)
    flags = (rng.random((B, T)) < 0.1).astype(np.uint8)
    _run_both(lib, B, T, 4, window, flags, dev)
    p = _params(B + 1, T, 4, window)
    fake = ctypes.c_void_p(0x100000)  # never dereferenced: the size check fails first
    assert lib.sattn_build_blockmap_noalloc(ctypes.byref(p), None, None, fake, fake, fake, None) == \
        _lib.SATTN_ERR_UNSUPPORTED


def test_noalloc_rejects_oversize_before_launch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = _lib.load()
    T, w = 40000, 128
    B = 1
    while _scratch_bytes(B, T, w) <= MAX_BYTES:
        B += 1
    assert _scratch_bytes(B - 1, T, w) <= MAX_BYTES < _scratch_bytes(B, T, w)
    p = _params(B, T, 4, w)
    fake = ctypes.c_void_p(0x100000)  # never dereferenced: the size check fails first
    assert lib.sattn_build_blockmap_noalloc(ctypes.byref(p), None, None, fake, fake, fake, None) == \
        _lib.SATTN_ERR_UNSUPPORTED
