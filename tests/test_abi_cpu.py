"""The C-ABI library on a machine without a GPU: it loads, exports every
function ``include/sattn.h`` declares, and its host-side validation and
workspace sizing work without touching the device."""
import ctypes
import os
import re

import pytest

from long_context_structured_b200 import _lib
import long_context_structured_b200 as sa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    text = open(os.path.join(ROOT, "include", "sattn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sattn_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        import long_context_structured_b200.build as b
        b.build()
    return _lib.load()


def test_exports_every_header_function(lib):
    names = _header_functions()
    assert set(names) == set(_lib.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_strerror(lib):
    assert lib.sattn_version() == 10000
    for rc in (0, -1, -2, -3, -4):
        assert len(_lib.strerror(rc)) > 0
    assert _lib.strerror(-99) == "unknown status"


def _p(B=1, Hq=2, Hkv=2, T=256, d=128, dtype=_lib.DTYPE_BF16, **kw):
    p = _lib.SattnParams()
    p.B, p.Hq, p.Hkv, p.T, p.d, p.dtype = B, Hq, Hkv, T, d, dtype
    for name in ("q_stride", "k_stride", "v_stride", "o_stride"):
        H = Hq if name in ("q_stride", "o_stride") else Hkv
        arr = getattr(p, name)
        arr[0], arr[1], arr[2] = H * T * d, T * d, d
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def _ws(lib, p):
    n = ctypes.c_size_t(0)
    rc = lib.sattn_workspace_size(ctypes.byref(p), ctypes.byref(n))
    return rc, n.value


def test_workspace_size_and_validation(lib):
    rc, n = _ws(lib, _p())
    assert rc == 0 and n > 0
    rc_sep, n_sep = _ws(lib, _p(with_separators=1))
    assert rc_sep == 0 and n_sep > n
    rc_tk, n_tk = _ws(lib, _p(topk=5, window=64, L_pretrain=64))
    assert rc_tk == 0 and n_tk > n
    # rejected on the host
    assert _ws(lib, _p(d=96))[0] == _lib.SATTN_ERR_UNSUPPORTED
    assert _ws(lib, _p(Hq=3, Hkv=2))[0] == _lib.SATTN_ERR_INVALID_ARG
    assert _ws(lib, _p(window=-1))[0] == _lib.SATTN_ERR_INVALID_ARG
    assert _ws(lib, _p(topk=17))[0] == _lib.SATTN_ERR_UNSUPPORTED
    assert _ws(lib, _p(window=100, L_pretrain=50))[0] == _lib.SATTN_ERR_UNSUPPORTED
    # top-k with the window below the cap is taken, except with the ALiBi bias
    assert _ws(lib, _p(window=30, L_pretrain=50, topk=2))[0] == 0
    assert _ws(lib, _p(window=30, L_pretrain=50, topk=2, alibi=1, rope_theta=0.0))[0] == _lib.SATTN_ERR_UNSUPPORTED
    # tiles: 128 x 128 (or 0, the default) only
    assert _ws(lib, _p(tile_m=128, tile_n=128))[0] == 0
    assert _ws(lib, _p(tile_m=64))[0] == _lib.SATTN_ERR_UNSUPPORTED
    assert _ws(lib, _p(tile_n=256))[0] == _lib.SATTN_ERR_UNSUPPORTED
    # separators with the window below the cap are taken
    assert _ws(lib, _p(window=30, L_pretrain=50, with_separators=1))[0] == 0
    assert _ws(lib, _p(dtype=7))[0] == _lib.SATTN_ERR_INVALID_ARG
    assert _ws(lib, _p(rope_theta=float("nan")))[0] == _lib.SATTN_ERR_INVALID_ARG
    # fp32 has no tensor-core restrictions on the cap
    assert _ws(lib, _p(dtype=_lib.DTYPE_F32, window=30, L_pretrain=50, topk=2))[0] == 0
    p = _p()
    p.q_stride[2] = 100  # 200-byte rows: not 16-byte aligned for bf16
    assert _ws(lib, p)[0] == _lib.SATTN_ERR_INVALID_ARG


def test_workspace_grows_with_problem(lib):
    sizes = [_ws(lib, _p(T=T))[1] for T in (128, 1024, 8192)]
    assert sizes[0] < sizes[1] < sizes[2]


def test_segment_workspace(lib):
    n = ctypes.c_size_t(0)
    il = (ctypes.c_uint8 * 4)(0, 0, 1, 1)
    p = _p(Hq=4, Hkv=4, T=1024)
    assert lib.sattn_segment_workspace_size(ctypes.byref(p), 256, 64, 128, 64, il, ctypes.byref(n)) == 0
    n_half = n.value
    assert lib.sattn_segment_workspace_size(ctypes.byref(p), 256, 64, 128, 64, None, ctypes.byref(n)) == 0
    assert n.value > n_half  # all heads long needs more prefix room
    assert lib.sattn_segment_workspace_size(ctypes.byref(p), 100, 64, 128, 64, il, ctypes.byref(n)) == -1
    assert lib.sattn_segment_workspace_size(ctypes.byref(p), 256, 64, 100, 64, il, ctypes.byref(n)) == -1


def test_segment_stream_sizes_and_validation(lib):
    """The carried state holds K, V and rotated K of every position of the
    capacity plus the table; the step's workspace holds one segment's
    queries and prefix.  Bad shapes and out-of-range steps are refused on the
    host before any launch."""
    n = ctypes.c_size_t(0)
    il = (ctypes.c_uint8 * 4)(0, 0, 1, 1)
    p = _p(Hq=4, Hkv=2, T=1024, rope_theta=1e4)
    assert lib.sattn_segment_state_size(ctypes.byref(p), 256, 64, 128, 64, ctypes.byref(n)) == 0
    kv = 2 * 1024 * 128 * 2  # one of K, V, rotated K: B * Hkv * T * d bf16
    assert n.value >= 3 * kv + 1024 * 64 * 8
    assert lib.sattn_segment_step_workspace_size(ctypes.byref(p), 256, 64, 128, 64, il, ctypes.byref(n)) == 0
    assert n.value >= 4 * 256 * 128 * 2  # the segment's rotated queries
    assert lib.sattn_segment_state_size(ctypes.byref(p), 100, 64, 128, 64, ctypes.byref(n)) == -1  # S % 128
    assert lib.sattn_segment_state_size(ctypes.byref(p), 384, 64, 128, 64, ctypes.byref(n)) == -1  # T % S
    assert lib.sattn_segment_state_size(ctypes.byref(p), 256, 64, 100, 64, ctypes.byref(n)) == -1  # R % blk
    fake = ctypes.c_void_p(0x100000)  # never dereferenced: validation fails first
    big = ctypes.c_size_t(1 << 40).value
    for seg in (-1, 4):  # capacity 1024 = 4 segments
        assert lib.sattn_segment_step(ctypes.byref(p), 256, 64, 128, 64, il, seg, fake, fake, fake, fake, big,
                                      fake, fake, fake, fake, big, None) == -1
    assert lib.sattn_segment_step(ctypes.byref(p), 256, 64, 128, 64, None, 0, fake, fake, fake, fake, big,
                                  fake, fake, fake, fake, big, None) == -1  # is_long required
    pa = _p(Hq=4, Hkv=2, T=1024, alibi=1)
    assert lib.sattn_segment_state_size(ctypes.byref(pa), 256, 64, 128, 64, ctypes.byref(n)) == -2


def test_entry_points_reject_bad_arguments_before_launch(lib):
    p = _p()
    rc, n = _ws(lib, p)
    fake = ctypes.c_void_p(0x100000)  # never dereferenced: validation fails first
    # null tensors
    assert lib.sattn_fwd(ctypes.byref(p), None, fake, fake, None, None, None, fake, fake, fake, n, None) == -1
    # workspace too small
    assert lib.sattn_fwd(ctypes.byref(p), fake, fake, fake, None, None, None, fake, fake, fake, n - 1, None) == -1
    # misaligned workspace
    assert lib.sattn_fwd(ctypes.byref(p), fake, fake, fake, None, None, None, fake, fake, ctypes.c_void_p(0x100010), n,
                         None) == -1
    # separators without room for them
    assert lib.sattn_fwd(ctypes.byref(p), fake, fake, fake, fake, None, None, fake, fake, fake, n, None) == -1
    # only one of topk_idx / topk_logit
    assert lib.sattn_fwd(ctypes.byref(p), fake, fake, fake, None, fake, None, fake, fake, fake, n, None) == -1
    # misaligned tensor
    assert lib.sattn_fwd(ctypes.byref(p), ctypes.c_void_p(0x100008), fake, fake, None, None, None, fake, fake, fake, n,
                         None) == -1
    # top-k selection needs topk >= 1
    assert lib.sattn_topk_select(ctypes.byref(p), fake, fake, None, fake, fake, fake, n, None) == -1
    # blockmap outputs required
    assert lib.sattn_build_blockmap(ctypes.byref(p), None, None, None, fake, fake, fake, n, None) == -1
    # segment: host head mask required
    assert lib.sattn_segment_fwd(ctypes.byref(p), 128, 0, 0, 64, None, fake, fake, fake, fake, fake, fake, fake, n,
                                 None) == -1
    # status query needs a workspace
    st = ctypes.c_int32(0)
    assert lib.sattn_stream_status(None, None, ctypes.byref(st)) == -1


def test_python_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(ImportError):
        _lib.load()


def _noalloc_scratch_bytes(B, T, window):
    """The scratch of sattn_build_blockmap_noalloc as the header states it."""
    up16 = lambda x: (x + 15) // 16 * 16
    nqt = (T + 127) // 128
    bt = min(nqt, (window + 127) // 128)
    kc = min((nqt + 15) // 16, bt // 16 + 2)
    return up16(8 * B * (T // 32 + 1)) + B * up16(nqt) + B * 16 * nqt * kc


@pytest.mark.parametrize("T,window", [(40000, 128), (8192, 256), (4096, 5000), (1000, 37)])
def test_noalloc_refuses_oversize_on_the_host(lib, T, window):
    """The no-alloc block map refuses, on the host and before it touches any
    device, the first batch size whose scratch (the header's formula) no
    longer fits its 4 MiB array.  Only the refused size is called here: an
    accepted size would launch, and it is checked with real device buffers
    in the GPU tests."""
    B = 1
    while _noalloc_scratch_bytes(B + 1, T, window) <= 1 << 22:
        B += 1
    assert _noalloc_scratch_bytes(B, T, window) <= 1 << 22 < _noalloc_scratch_bytes(B + 1, T, window)
    fake = ctypes.c_void_p(0x100000)  # never dereferenced: the size check returns first
    big = lib.sattn_build_blockmap_noalloc(ctypes.byref(_p(B=B + 1, T=T, n_start=4, window=window,
                                                           with_separators=1)), None, None, fake, fake, fake, None)
    assert big == _lib.SATTN_ERR_UNSUPPORTED
