"""Out-of-bounds write check for every entry point (a stand-in for a memory
sanitizer, which is not available here).

Every output and every workspace is placed inside a larger device buffer
whose surrounding bytes hold a known pattern (4 KB on each side), outputs
with a row stride wider than the head dimension are also checked in the gaps
between rows, and the workspace is given exactly the size its query
returned.  After each call (through the C ABI, with the library's own size
queries) the guard bytes and gaps must be untouched, and the guarded results
must equal those of the Python binding's ordinary call.
"""
import ctypes

import numpy as np
import pytest
import torch

import long_context_structured_b200 as sa
from long_context_structured_b200 import _lib, synth
from _util import to_dev

pytestmark = pytest.mark.gpu

PAT = 0xA5
GUARD = 4096


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


class Guarded:
    """nbytes of device memory, 256-byte aligned, between two guard zones."""

    def __init__(self, nbytes, dev="cuda"):
        self.n = int(nbytes)
        self.raw = torch.full((self.n + 2 * GUARD + 512,), PAT, dtype=torch.uint8, device=dev)
        self.lo = (-self.raw.data_ptr()) % 256 + GUARD
        self.buf = self.raw[self.lo:self.lo + self.n]

    @property
    def ptr(self):
        return ctypes.c_void_p(self.buf.data_ptr())

    def view(self, dtype, shape, strides=None):
        t = self.buf.view(dtype)
        return torch.as_strided(t, shape, strides) if strides is not None else t.view(shape)

    def check(self, name):
        torch.cuda.synchronize()
        raw = self.raw.cpu().numpy()
        assert (raw[:self.lo] == PAT).all(), "%s: bytes before the buffer were written" % name
        assert (raw[self.lo + self.n:] == PAT).all(), "%s: bytes after the buffer were written" % name


def padded(shape, d, dtype, dev="cuda", fill=None, src=None):
    """[B, H, T, d] tensor with token stride d + pad (16 bytes of padding per row)."""
    B, H, T, _ = shape
    esz = torch.tensor([], dtype=dtype).element_size()
    sp = d + 16 // esz
    g = Guarded(B * H * T * sp * esz, dev)
    t = g.view(dtype, (B, H, T, d), (H * T * sp, T * sp, sp, 1))
    if src is not None:
        t.copy_(src)
    return g, t, sp


def gaps_untouched(g, shape, d, sp, dtype, name):
    B, H, T, _ = shape
    itype = {2: torch.int16, 4: torch.int32}[torch.tensor([], dtype=dtype).element_size()]
    rows = g.buf.view(itype).view(B, H, T, sp)[..., d:].cpu().numpy()
    pat = np.full(1, PAT * (0x0101 if itype == torch.int16 else 0x01010101), dtype=np.int64).astype(
        np.int16 if itype == torch.int16 else np.int32)[0]
    assert (rows == pat).all(), "%s: the gaps between rows were written" % name


def _stream(dev="cuda"):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _ws(query, *args):
    n = ctypes.c_size_t(0)
    assert query(*args, ctypes.byref(n)) == 0
    return Guarded(max(int(n.value), 256)), int(n.value)


def _inputs(cfg, dtype="bf16", seed=3):
    wl = synth.Workload(name="canary", dtype=dtype, **cfg)
    inp = synth.make_inputs(wl, seed=seed)
    return wl, inp, to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), to_dev(inp["is_sep"])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fwd_and_topk_select(dtype):
    L = _lib.load()
    cfg = dict(B=1, Hq=4, Hkv=2, T=700, d=128 if dtype == "bf16" else 64, n_start=4, window=128, L_pretrain=128,
               rope_theta=1e4, topk=3, sep_rate=0.1)
    wl, inp, q, k, v, sep = _inputs(cfg, dtype)
    tdt = q.dtype
    shape = (wl.B, wl.Hq, wl.T, wl.d)
    go, O, sp = padded(shape, wl.d, tdt)
    p = sa.params(q, k, v, O, n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain, topk=wl.topk,
                  rope_theta=wl.rope_theta, with_separators=True)
    ws, nb = _ws(L.sattn_workspace_size, ctypes.byref(p))
    gl = Guarded(wl.B * wl.Hq * wl.T * 4)
    rc = L.sattn_fwd(ctypes.byref(p), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                     ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(sep.data_ptr()), None, None, go.ptr, gl.ptr,
                     ws.ptr, nb, _stream())
    assert rc == 0
    for g, name in ((go, "O"), (gl, "lse"), (ws, "workspace")):
        g.check(name)
    gaps_untouched(go, shape, wl.d, sp, tdt, "O")
    O_ref, l_ref = sa.fwd(q, k, v, n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain, topk=wl.topk,
                          rope_theta=wl.rope_theta, is_sep=sep)
    assert torch.equal(O, O_ref) and torch.equal(gl.view(torch.float32, (wl.B, wl.Hq, wl.T)), l_ref)
    if dtype != "bf16":
        return
    # the selection alone
    gi = Guarded(wl.B * wl.Hq * wl.T * wl.topk * 4)
    gz = Guarded(wl.B * wl.Hq * wl.T * wl.topk * 4)
    ws.raw.fill_(PAT)
    rc = L.sattn_topk_select(ctypes.byref(p), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                             ctypes.c_void_p(sep.data_ptr()), gi.ptr, gz.ptr, ws.ptr, nb, _stream())
    assert rc == 0
    for g, name in ((gi, "idx"), (gz, "logit"), (ws, "workspace")):
        g.check(name)
    idx_ref, z_ref = sa.topk_select(q, k, topk=wl.topk, n_start=wl.n_start, window=wl.window,
                                    L_pretrain=wl.L_pretrain, rope_theta=wl.rope_theta, is_sep=sep)
    assert torch.equal(gi.view(torch.int32, idx_ref.shape), idx_ref)


def test_blockmap_both_entries():
    L = _lib.load()
    B, T = 3, 1000
    flags = (np.random.default_rng(1).random((B, T)) < 0.2).astype(np.uint8)
    f = torch.from_numpy(flags).cuda()
    nqt = (T + 127) // 128
    dummy = torch.empty((B, 1, T, 64), dtype=torch.bfloat16, device="cuda")
    p = sa.params(dummy, dummy, dummy, dummy, n_start=4, window=37, with_separators=True)
    ref = sa.build_blockmap(f, B=B, T=T, n_start=4, window=37)
    for noalloc in (False, True):
        outs = [Guarded(B * nqt * nqt), Guarded(B * T * 4), Guarded(B * 4), Guarded(B * nqt * 2 * 4)]
        if noalloc:
            rc = L.sattn_build_blockmap_noalloc(ctypes.byref(p), ctypes.c_void_p(f.data_ptr()),
                                                *[g.ptr for g in outs], _stream())
        else:
            ws, nb = _ws(L.sattn_workspace_size, ctypes.byref(p))
            rc = L.sattn_build_blockmap(ctypes.byref(p), ctypes.c_void_p(f.data_ptr()), *[g.ptr for g in outs],
                                        ws.ptr, nb, _stream())
            ws.check("workspace")
        assert rc == 0
        for g, name in zip(outs, ("cls", "sep_pos", "sep_count", "ranges")):
            g.check(name)
        assert torch.equal(outs[0].view(torch.uint8, ref["cls"].shape), ref["cls"])
        assert torch.equal(outs[1].view(torch.int32, ref["sep_pos"].shape), ref["sep_pos"])
        assert torch.equal(outs[3].view(torch.int32, ref["qtile_sep_range"].shape), ref["qtile_sep_range"])


def test_segment_fwd():
    L = _lib.load()
    cfg = dict(B=1, Hq=2, Hkv=2, T=1024, d=128, rope_theta=1e4, seg_S=256, seg_M=64, seg_R=128, retr_block=64,
               long_heads=(1,))
    wl, inp, q, k, v, _ = _inputs(cfg)
    shape = (wl.B, wl.Hq, wl.T, wl.d)
    go, O, sp = padded(shape, wl.d, q.dtype)
    gl = Guarded(wl.B * wl.Hq * wl.T * 4)
    N, nb_blk = wl.T // wl.seg_S, wl.seg_R // wl.retr_block
    gp = Guarded(wl.B * wl.Hq * N * nb_blk * 4)
    p = sa.params(q, k, v, O, rope_theta=wl.rope_theta)
    il = (ctypes.c_uint8 * wl.Hq)(*[int(x) for x in inp["is_long"]])
    ws, nb = _ws(L.sattn_segment_workspace_size, ctypes.byref(p), wl.seg_S, wl.seg_M, wl.seg_R, wl.retr_block, il)
    rc = L.sattn_segment_fwd(ctypes.byref(p), wl.seg_S, wl.seg_M, wl.seg_R, wl.retr_block, il,
                             ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                             ctypes.c_void_p(v.data_ptr()), go.ptr, gl.ptr, gp.ptr, ws.ptr, nb, _stream())
    assert rc == 0
    for g, name in ((go, "O"), (gl, "lse"), (gp, "prefix_blocks"), (ws, "workspace")):
        g.check(name)
    gaps_untouched(go, shape, wl.d, sp, q.dtype, "O")
    O_ref, _, pb_ref = sa.segment_fwd(q, k, v, S=wl.seg_S, M=wl.seg_M, R=wl.seg_R, retr_block=wl.retr_block,
                                      is_long=inp["is_long"], rope_theta=wl.rope_theta)
    assert torch.equal(O, O_ref) and torch.equal(gp.view(torch.int32, pb_ref.shape), pb_ref)


def test_decode_fwd():
    L = _lib.load()
    cfg = dict(B=2, Hq=8, Hkv=2, T=900, d=128, n_start=12, window=64, L_pretrain=64, rope_theta=1e4, sep_rate=0.1)
    wl, inp, q, k, v, sep = _inputs(cfg)
    qd = q[:, :, -1:, :].contiguous()
    shape = (wl.B, wl.Hq, 1, wl.d)
    go, O, sp = padded(shape, wl.d, qd.dtype)
    gl = Guarded(wl.B * wl.Hq * 4)
    p = sa.params(qd, k, v, O, n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain,
                  rope_theta=wl.rope_theta, with_separators=True)
    p.T = wl.T
    ws, nb = _ws(L.sattn_decode_workspace_size, ctypes.byref(p))
    rc = L.sattn_decode_fwd(ctypes.byref(p), ctypes.c_void_p(qd.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                            ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(sep.data_ptr()), go.ptr, gl.ptr, ws.ptr,
                            nb, _stream())
    assert rc == 0
    for g, name in ((go, "O"), (gl, "lse"), (ws, "workspace")):
        g.check(name)
    gaps_untouched(go, shape, wl.d, sp, qd.dtype, "O")
    O_ref, _ = sa.decode_fwd(qd, k, v, n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain,
                             rope_theta=wl.rope_theta, is_sep=sep)
    assert torch.equal(O, O_ref)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_bwd(dtype):
    L = _lib.load()
    cfg = dict(B=1, Hq=4, Hkv=2, T=600, d=128 if dtype == "bf16" else 64, n_start=20, window=64, L_pretrain=64,
               rope_theta=1e4, sep_rate=0.1)
    wl, inp, q0, k0, v0, sep = _inputs(cfg, dtype)
    kw = dict(n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain, rope_theta=wl.rope_theta)
    qs, ks = (wl.B, wl.Hq, wl.T, wl.d), (wl.B, wl.Hkv, wl.T, wl.d)
    # inputs with the same padded strides as the gradients they describe
    _, q, _ = padded(qs, wl.d, q0.dtype, src=q0)
    _, k, _ = padded(ks, wl.d, q0.dtype, src=k0)
    _, v, _ = padded(ks, wl.d, q0.dtype, src=v0)
    O, lse = sa.fwd(q, k, v, is_sep=sep, **kw)
    dO = torch.randn(qs, device="cuda").to(q0.dtype)
    dO = dO.contiguous()
    Oc = O.contiguous()
    gq, dQ, spq = padded(qs, wl.d, q0.dtype)
    gk, dK, spk = padded(ks, wl.d, q0.dtype)
    gv, dV, _ = padded(ks, wl.d, q0.dtype)
    p = sa.params(q, k, v, Oc, with_separators=True, **kw)
    ws, nb = _ws(L.sattn_bwd_workspace_size, ctypes.byref(p))
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = L.sattn_bwd(ctypes.byref(p), ptr(q), ptr(k), ptr(v), ptr(sep), None, ptr(Oc), ptr(lse), ptr(dO), gq.ptr,
                     gk.ptr, gv.ptr, ws.ptr, nb, _stream())
    assert rc == 0
    for g, name in ((gq, "dQ"), (gk, "dK"), (gv, "dV"), (ws, "workspace")):
        g.check(name)
    gaps_untouched(gq, qs, wl.d, spq, q0.dtype, "dQ")
    gaps_untouched(gk, ks, wl.d, spk, q0.dtype, "dK")
    ref = sa.bwd(q0, k0, v0, Oc, lse, dO, is_sep=sep, **kw)
    for got, r in zip((dQ, dK, dV), ref):
        assert torch.equal(got, r)


def test_tree_cross_fwd():
    L = _lib.load()
    B, H, Tq, d, n_chunks, chunk_len, depth, alpha = 1, 2, 300, 128, 4, 512, 2, 2
    g = torch.Generator().manual_seed(0)
    mk = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16).cuda()
    q, k, v = mk(B, H, Tq, d), mk(B, H, n_chunks * chunk_len, d), mk(B, H, n_chunks * chunk_len, d)
    shape = (B, H, Tq, d)
    go, O, sp = padded(shape, d, q.dtype)
    gl = Guarded(B * H * Tq * 4)
    O_ref, l_ref, kept = sa.tree_cross_fwd(q, k, v, n_chunks=n_chunks, chunk_len=chunk_len, depth=depth,
                                           alpha_leaf=alpha, rope_theta=1e4, with_index=True)
    n_kept = int((kept >= 0).sum())
    gk = Guarded(n_kept * 4)
    p = sa.params(q, k, v, O, rope_theta=1e4)
    ws, nb = _ws(L.sattn_tree_cross_workspace_size, ctypes.byref(p), n_chunks, chunk_len, depth, alpha)
    rc = L.sattn_tree_cross_fwd(ctypes.byref(p), n_chunks, chunk_len, depth, alpha, ctypes.c_void_p(q.data_ptr()),
                                ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()), go.ptr, gl.ptr, gk.ptr,
                                ws.ptr, nb, _stream())
    assert rc == 0
    for gg, name in ((go, "O"), (gl, "lse"), (gk, "kept_index"), (ws, "workspace")):
        gg.check(name)
    gaps_untouched(go, shape, d, sp, q.dtype, "O")
    assert torch.equal(O, O_ref) and torch.equal(gk.view(torch.int32, (n_kept,)), kept[:n_kept])


def test_stream_cache():
    L = _lib.load()
    cfg = _lib.StreamConfig(2, 2, 128, 4, 8, 16, 40)
    n = ctypes.c_size_t(0)
    assert L.sattn_stream_state_size(ctypes.byref(cfg), ctypes.byref(n)) == 0
    st = Guarded(int(n.value))
    assert L.sattn_stream_reset(ctypes.byref(cfg), st.ptr, int(n.value), _stream()) == 0
    g = torch.Generator().manual_seed(1)
    for pos in range(100):
        kn = torch.randn(2, 2, 128, generator=g).to(torch.bfloat16).cuda()
        vn = torch.randn(2, 2, 128, generator=g).to(torch.bfloat16).cuda()
        sp = (torch.rand(2, generator=g) < 0.3).to(torch.uint8).cuda()
        assert L.sattn_stream_append(ctypes.byref(cfg), st.ptr, int(n.value), ctypes.c_void_p(kn.data_ptr()),
                                     ctypes.c_void_p(vn.data_ptr()), ctypes.c_void_p(sp.data_ptr()), pos,
                                     _stream()) == 0
    st.check("stream state")
    q = torch.randn(2, 4, 1, 128, generator=g).to(torch.bfloat16).cuda()
    shape = (2, 4, 1, 128)
    go, O, spo = padded(shape, 128, q.dtype)
    gl = Guarded(2 * 4 * 4)
    p = _lib.SattnParams()
    p.B, p.Hq, p.Hkv, p.T, p.d, p.dtype = 2, 4, 2, 40, 128, _lib.DTYPE_BF16
    p.q_stride[0], p.q_stride[1], p.q_stride[2] = 4 * 128, 128, 128
    p.o_stride[0], p.o_stride[1], p.o_stride[2] = O.stride(0), O.stride(1), O.stride(2)
    p.rope_theta = 1e4
    nw = ctypes.c_size_t(0)
    assert L.sattn_stream_decode_workspace_size(ctypes.byref(cfg), ctypes.byref(p), ctypes.byref(nw)) == 0
    ws = Guarded(max(int(nw.value), 256))
    assert L.sattn_stream_decode(ctypes.byref(cfg), ctypes.byref(p), st.ptr, int(n.value),
                                 ctypes.c_void_p(q.data_ptr()), go.ptr, gl.ptr, ws.ptr, int(nw.value),
                                 _stream()) == 0
    for gg, name in ((go, "O"), (gl, "lse"), (ws, "workspace"), (st, "stream state")):
        gg.check(name)
    gaps_untouched(go, shape, 128, spo, q.dtype, "O")


def test_decode_topk_fwd():
    L = _lib.load()
    cfg = dict(B=2, Hq=8, Hkv=2, T=1200, d=128, n_start=4, window=64, L_pretrain=200, rope_theta=1e4, topk=5,
               sep_rate=0.1)
    wl, inp, q, k, v, sep = _inputs(cfg)
    qd = q[:, :, -1:, :].contiguous()
    shape = (wl.B, wl.Hq, 1, wl.d)
    go, O, sp = padded(shape, wl.d, qd.dtype)
    gl = Guarded(wl.B * wl.Hq * 4)
    gi = Guarded(wl.B * wl.Hq * wl.topk * 4)
    gz = Guarded(wl.B * wl.Hq * wl.topk * 4)
    p = sa.params(qd, k, v, O, n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain, topk=wl.topk,
                  rope_theta=wl.rope_theta, with_separators=True)
    p.T = wl.T
    ws, nb = _ws(L.sattn_decode_workspace_size, ctypes.byref(p))
    rc = L.sattn_decode_topk_fwd(ctypes.byref(p), ctypes.c_void_p(qd.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                 ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(sep.data_ptr()), go.ptr, gl.ptr,
                                 gi.ptr, gz.ptr, ws.ptr, nb, _stream())
    assert rc == 0
    for g, name in ((go, "O"), (gl, "lse"), (gi, "topk_idx"), (gz, "topk_logit"), (ws, "workspace")):
        g.check(name)
    gaps_untouched(go, shape, wl.d, sp, qd.dtype, "O")
    O_ref, _, idx_ref, z_ref = sa.decode_fwd(qd, k, v, n_start=wl.n_start, window=wl.window,
                                             L_pretrain=wl.L_pretrain, rope_theta=wl.rope_theta, is_sep=sep,
                                             topk=wl.topk, return_topk=True)
    assert torch.equal(O, O_ref)
    assert torch.equal(gi.view(torch.int32, idx_ref.shape), idx_ref)
    assert torch.equal(gz.view(torch.float32, z_ref.shape), z_ref)


def test_fwd_topk_window_below_cap():
    """The two-operand selector instantiation (window below the cap) and the
    separators' extended band."""
    L = _lib.load()
    cfg = dict(B=1, Hq=4, Hkv=2, T=900, d=128, n_start=4, window=64, L_pretrain=256, rope_theta=1e4, topk=4,
               sep_rate=0.1)
    wl, inp, q, k, v, sep = _inputs(cfg)
    shape = (wl.B, wl.Hq, wl.T, wl.d)
    go, O, sp = padded(shape, wl.d, q.dtype)
    gl = Guarded(wl.B * wl.Hq * wl.T * 4)
    p = sa.params(q, k, v, O, n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain, topk=wl.topk,
                  rope_theta=wl.rope_theta, with_separators=True)
    ws, nb = _ws(L.sattn_workspace_size, ctypes.byref(p))
    rc = L.sattn_fwd(ctypes.byref(p), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                     ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(sep.data_ptr()), None, None, go.ptr, gl.ptr,
                     ws.ptr, nb, _stream())
    assert rc == 0
    for g, name in ((go, "O"), (gl, "lse"), (ws, "workspace")):
        g.check(name)
    gaps_untouched(go, shape, wl.d, sp, q.dtype, "O")
    O_ref, l_ref = sa.fwd(q, k, v, n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain, topk=wl.topk,
                          rope_theta=wl.rope_theta, is_sep=sep)
    assert torch.equal(O, O_ref) and torch.equal(gl.view(torch.float32, (wl.B, wl.Hq, wl.T)), l_ref)


def test_segment_step():
    """The carried state and every step's outputs and workspace."""
    L = _lib.load()
    cfg = dict(B=1, Hq=4, Hkv=2, T=768, d=128, rope_theta=1e4, seg_S=256, seg_M=64, seg_R=128, retr_block=64,
               long_heads=(1, 2))
    wl, inp, q, k, v, _ = _inputs(cfg)
    S, N, nb_blk = wl.seg_S, wl.T // wl.seg_S, wl.seg_R // wl.retr_block
    il = (ctypes.c_uint8 * wl.Hq)(*[int(x) for x in inp["is_long"]])
    seg = lambda t, s: t[:, :, s * S:(s + 1) * S].contiguous()
    shape = (wl.B, wl.Hq, S, wl.d)
    go, O, sp = padded(shape, wl.d, q.dtype)
    p = sa.params(seg(q, 0), seg(k, 0), seg(v, 0), O, rope_theta=wl.rope_theta)
    p.T = wl.T  # the capacity
    n = ctypes.c_size_t(0)
    assert L.sattn_segment_state_size(ctypes.byref(p), S, wl.seg_M, wl.seg_R, wl.retr_block, ctypes.byref(n)) == 0
    st = Guarded(int(n.value))
    assert L.sattn_segment_state_reset(ctypes.byref(p), S, wl.seg_M, wl.seg_R, wl.retr_block, st.ptr, int(n.value),
                                       _stream()) == 0
    ws, nb = _ws(L.sattn_segment_step_workspace_size, ctypes.byref(p), S, wl.seg_M, wl.seg_R, wl.retr_block, il)
    O_ref, _, pb_ref = sa.segment_fwd(q, k, v, S=S, M=wl.seg_M, R=wl.seg_R, retr_block=wl.retr_block,
                                      is_long=inp["is_long"], rope_theta=wl.rope_theta)
    for s in range(N):
        gl = Guarded(wl.B * wl.Hq * S * 4)
        gp = Guarded(wl.B * wl.Hq * nb_blk * 4)
        qs, ks, vs = seg(q, s), seg(k, s), seg(v, s)
        rc = L.sattn_segment_step(ctypes.byref(p), S, wl.seg_M, wl.seg_R, wl.retr_block, il, s,
                                  ctypes.c_void_p(qs.data_ptr()), ctypes.c_void_p(ks.data_ptr()),
                                  ctypes.c_void_p(vs.data_ptr()), st.ptr, int(n.value), go.ptr, gl.ptr, gp.ptr,
                                  ws.ptr, nb, _stream())
        assert rc == 0
        for g, name in ((go, "O"), (gl, "lse"), (gp, "prefix_blocks"), (ws, "workspace"), (st, "state")):
            g.check("%s (segment %d)" % (name, s))
        gaps_untouched(go, shape, wl.d, sp, q.dtype, "O")
        assert torch.equal(O, O_ref[:, :, s * S:(s + 1) * S])
        assert torch.equal(gp.view(torch.int32, (wl.B, wl.Hq, nb_blk)), pb_ref[:, :, s])
