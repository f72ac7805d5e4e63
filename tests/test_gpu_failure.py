"""Failure detection on the GPU without a GPU fault.

Every mbarrier wait in the library's kernels is bounded: when the limit
passes, the kernel records SATTN_ERR_TIMEOUT (and the waiting site) in the
workspace's status word and returns normally.  Here a kernel waits on a
barrier that nothing arrives at, with a 20 ms limit; the host reads the
status, and the same process then runs a normal call to show that the CUDA
context is still usable.
"""
import numpy as np
import pytest
import torch

import long_context_structured_b200 as sa
from long_context_structured_b200 import _lib, synth
from _util import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def test_bounded_wait_reports_timeout_and_context_survives():
    status, site = sa.selftest_wait_timeout(limit_ms=20.0)
    assert status == _lib.SATTN_ERR_TIMEOUT
    assert site == 99
    # the context still works: a normal call succeeds with a clean status and
    # the same result as before the timeout
    wl = synth.Workload(name="after_timeout", B=1, Hq=2, Hkv=2, T=300, d=128, dtype="bf16", n_start=4, window=64,
                        L_pretrain=64, rope_theta=1e4)
    inp = synth.make_inputs(wl, seed=2)
    q, k, v = (to_dev(inp[x]) for x in ("q", "k", "v"))
    kw = dict(n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain, rope_theta=wl.rope_theta)
    O1, l1 = sa.fwd(q, k, v, **kw)
    torch.cuda.synchronize()
    assert sa.stream_status() == 0
    assert torch.isfinite(O1.float()).all()
    status2, _ = sa.selftest_wait_timeout(limit_ms=5.0)
    assert status2 == _lib.SATTN_ERR_TIMEOUT
    O2, l2 = sa.fwd(q, k, v, **kw)
    torch.cuda.synchronize()
    assert sa.stream_status() == 0
    assert torch.equal(O1, O2) and torch.equal(l1, l2)


def test_selftest_rejects_bad_arguments_before_launch():
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    L = _lib.load()
    st = torch.cuda.current_stream().cuda_stream
    import ctypes
    assert L.sattn_selftest_wait_timeout(None, 256, 1000, ctypes.c_void_p(st)) == _lib.SATTN_ERR_INVALID_ARG
    assert L.sattn_selftest_wait_timeout(ctypes.c_void_p(ws.data_ptr()), 64, 1000,
                                         ctypes.c_void_p(st)) == _lib.SATTN_ERR_INVALID_ARG
    assert L.sattn_selftest_wait_timeout(ctypes.c_void_p(ws.data_ptr()), 256, 0,
                                         ctypes.c_void_p(st)) == _lib.SATTN_ERR_INVALID_ARG
    assert L.sattn_selftest_wait_timeout(ctypes.c_void_p(ws.data_ptr()), 256, 3 * 10 ** 9,
                                         ctypes.c_void_p(st)) == _lib.SATTN_ERR_INVALID_ARG
