"""Segmented execution one segment at a time with the carried state
(``SegmentStream`` over ``sattn_segment_state_*`` / ``sattn_segment_step``).

Steps 0 .. N-1 are checked bit for bit against the whole-layer
``segment_fwd`` on the concatenated segments (the same kernels on the same
operands: keys rotated at their global positions, the same retrieval, the
same attention kernel per segment length), and the concatenated outputs
against the fp64 oracle's segmented rows.  A step out of order writes
nothing and reports SATTN_ERR_INVALID_ARG in the status word.
"""
import numpy as np
import pytest
import torch

import long_context_structured_b200 as sa
from long_context_structured_b200 import _lib, synth
from _util import BF16_MAX_ABS, BF16_MEAN_ABS, compare, gather_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


CASES = [
    # S a multiple of 256: the two-tile attention kernel
    ("s256_tail64_r128", dict(B=1, Hq=2, Hkv=2, T=1024, d=128, S=256, M=64, R=128, blk=64, long=(0, 1))),
    # S = 384: the one-tile kernel; the tail spans most of the previous segment
    ("s384_tail300_r256", dict(B=2, Hq=4, Hkv=2, T=1536, d=128, S=384, M=300, R=256, blk=32, long=(1, 0, 0, 1))),
    # a tail longer than a segment (reaches two segments back); d = 64
    ("s128_tail200_d64", dict(B=1, Hq=4, Hkv=4, T=768, d=64, S=128, M=200, R=128, blk=64, long=(0, 1, 1, 0))),
    # every head long, position interpolation
    ("all_long_pos_interp", dict(B=1, Hq=2, Hkv=1, T=1024, d=128, S=256, M=0, R=256, blk=64, long=(1, 1),
                                 pos_scale=0.25)),
    # no retrieval, no tail: block-diagonal causal
    ("no_state", dict(B=1, Hq=2, Hkv=2, T=512, d=128, S=128, M=0, R=0, blk=16, long=(0, 1))),
]


def _workload(name, c):
    return synth.Workload(name=name, B=c["B"], Hq=c["Hq"], Hkv=c["Hkv"], T=c["T"], d=c["d"], dtype="bf16",
                          rope_theta=1e4, seg_S=c["S"], seg_M=c["M"], seg_R=c["R"], retr_block=c["blk"],
                          long_heads=tuple(h for h in range(c["Hq"]) if c["long"][h]),
                          rope_pos_scale=c.get("pos_scale", 1.0))


@pytest.mark.parametrize("name,c", CASES, ids=[x[0] for x in CASES])
def test_steps_equal_whole_layer_and_oracle(oracle_mod, name, c):
    wl = _workload(name, c)
    inp = synth.make_inputs(wl, seed=21)
    q, k, v = to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"])
    kw = dict(S=wl.seg_S, M=wl.seg_M, R=wl.seg_R, retr_block=wl.retr_block, is_long=inp["is_long"],
              rope_theta=wl.rope_theta, rope_pos_scale=wl.rope_pos_scale)
    O_ref, lse_ref, pb_ref = sa.segment_fwd(q, k, v, **kw)
    st = sa.SegmentStream(B=wl.B, Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, capacity=wl.T, **kw)
    S, N = wl.seg_S, wl.T // wl.seg_S
    outs, lses, pbs = [], [], []
    for s in range(N):
        sl = slice(s * S, (s + 1) * S)
        # the segment's tensors as separate (contiguous) buffers, as a stream would hand them over
        O, lse, pb = st.step(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(), v[:, :, sl].contiguous())
        outs.append(O)
        lses.append(lse)
        pbs.append(pb)
    torch.cuda.synchronize()
    assert st.status() == 0
    O_all = torch.cat(outs, dim=2)
    lse_all = torch.cat(lses, dim=2)
    assert torch.equal(O_all, O_ref) and torch.equal(lse_all, lse_ref)
    if wl.seg_R > 0:
        assert torch.equal(torch.stack(pbs, dim=2), pb_ref)
    rows = oracle_mod.all_rows(wl.B, wl.Hq, wl.T)
    p = oracle_mod.params_of(wl)
    Oo, lo, _ = oracle_mod.segment_rows(p, wl.seg_S, wl.seg_M, wl.seg_R, wl.retr_block, inp["is_long"],
                                        inp["q"], inp["k"], inp["v"], rows)
    compare("O", gather_rows(O_all, rows), Oo, BF16_MAX_ABS, BF16_MEAN_ABS)
    compare("LSE", gather_rows(lse_all, rows), lo, BF16_MAX_ABS, BF16_MEAN_ABS)


def test_out_of_order_step_writes_nothing():
    wl = _workload("order", CASES[0][1])
    inp = synth.make_inputs(wl, seed=5)
    q, k, v = to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"])
    kw = dict(S=wl.seg_S, M=wl.seg_M, R=wl.seg_R, retr_block=wl.retr_block, is_long=inp["is_long"],
              rope_theta=wl.rope_theta)
    S = wl.seg_S
    seg = lambda t, s: t[:, :, s * S:(s + 1) * S].contiguous()
    st = sa.SegmentStream(B=wl.B, Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, capacity=wl.T, **kw)
    st.step(seg(q, 0), seg(k, 0), seg(v, 0))
    assert st.status() == 0
    state_before = st.state.clone()
    O = torch.full((wl.B, wl.Hq, S, wl.d), 7.0, dtype=torch.bfloat16, device="cuda")
    st.step(seg(q, 2), seg(k, 2), seg(v, 2), out=O, seg=2)  # segment 1 is next
    assert st.status() == _lib.SATTN_ERR_INVALID_ARG
    assert torch.equal(st.state, state_before)
    assert torch.all(O == 7.0)
    # the state goes on from where it was
    O1, lse1, _ = st.step(seg(q, 1), seg(k, 1), seg(v, 1), seg=1)
    assert st.status() == 0
    O_ref, lse_ref, _ = sa.segment_fwd(q, k, v, **kw)
    assert torch.equal(O1, O_ref[:, :, S:2 * S]) and torch.equal(lse1, lse_ref[:, :, S:2 * S])
    # a state that was never reset is refused the same way
    st2 = sa.SegmentStream(B=wl.B, Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, capacity=wl.T, **kw)
    st2.state.zero_()
    st2.step(seg(q, 0), seg(k, 0), seg(v, 0))
    assert st2.status() == _lib.SATTN_ERR_INVALID_ARG


def test_reset_starts_over():
    wl = _workload("reset", CASES[2][1])
    inp = synth.make_inputs(wl, seed=6)
    q, k, v = to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"])
    kw = dict(S=wl.seg_S, M=wl.seg_M, R=wl.seg_R, retr_block=wl.retr_block, is_long=inp["is_long"],
              rope_theta=wl.rope_theta)
    S = wl.seg_S
    st = sa.SegmentStream(B=wl.B, Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, capacity=wl.T, **kw)
    first = [st.step(*(t[:, :, s * S:(s + 1) * S].contiguous() for t in (q, k, v)))[0] for s in range(3)]
    st.reset()
    again = [st.step(*(t[:, :, s * S:(s + 1) * S].contiguous() for t in (q, k, v)))[0] for s in range(3)]
    torch.cuda.synchronize()
    assert st.status() == 0
    assert all(torch.equal(a, b) for a, b in zip(first, again))
