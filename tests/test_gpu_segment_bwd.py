"""GPU parity of the segmented-execution backward pass against the oracle's
fp64 gradients (``oracle_segment_bwd``, pinned by finite differences of the
segmented forward and by the one-segment case against the structured
backward).  The forward runs on the GPU first; its retrieval must equal the
oracle's (the retrieved blocks are constants of the backward pass), then the
gradients are compared element by element with bars relative to each
gradient's largest magnitude: max 2e-2, mean 2e-3 (bf16 operands)."""
import numpy as np
import pytest
import torch

import long_context_structured_b200 as sa
from long_context_structured_b200 import synth
from _util import to_dev
from test_gpu_bwd import BF16_GRAD_MEAN_REL, BF16_GRAD_REL, compare_grad

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


CASES = [
    ("tail_and_prefix", dict(B=1, Hq=2, Hkv=2, T=1024, S=256, M=64, R=128, blk=64, long=(1,))),
    ("tail_longer_than_segment", dict(B=1, Hq=2, Hkv=2, T=768, S=256, M=300, R=256, blk=32, long=(1,))),
    ("no_state", dict(B=1, Hq=2, Hkv=2, T=512, S=128, M=0, R=0, blk=16, long=(1,))),
    ("gqa_mixed_d64", dict(B=2, Hq=4, Hkv=2, T=512, S=128, M=32, R=64, blk=16, long=(1, 2), d=64)),
    ("pos_interp_all_long", dict(B=1, Hq=2, Hkv=1, T=768, S=256, M=0, R=128, blk=32, long=(0, 1), pos_scale=0.5)),
]


@pytest.mark.parametrize("name,cfg", CASES, ids=[c[0] for c in CASES])
def test_segment_bwd_matches_oracle(oracle_mod, name, cfg):
    wl = synth.Workload(name=name, B=cfg["B"], Hq=cfg["Hq"], Hkv=cfg["Hkv"], T=cfg["T"], d=cfg.get("d", 128),
                        dtype="bf16", rope_theta=1e4, seg_S=cfg["S"], seg_M=cfg["M"], seg_R=cfg["R"],
                        retr_block=cfg["blk"], long_heads=cfg["long"], rope_pos_scale=cfg.get("pos_scale", 1.0))
    inp = synth.make_inputs(wl, seed=41)
    q, k, v = (to_dev(inp[x]) for x in ("q", "k", "v"))
    kw = dict(S=wl.seg_S, M=wl.seg_M, R=wl.seg_R, retr_block=wl.retr_block, is_long=inp["is_long"],
              rope_theta=wl.rope_theta, rope_pos_scale=wl.rope_pos_scale)
    O, lse, pb = sa.segment_fwd(q, k, v, **kw)
    g = np.random.default_rng(42)
    dO_h = (g.standard_normal(inp["q"].shape).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    dO = to_dev(dO_h)
    dq, dk, dv = sa.segment_bwd(q, k, v, O, lse, pb, dO, **kw)
    torch.cuda.synchronize()
    p = oracle_mod.params_of(wl)
    if wl.seg_R > 0:
        ref_pb, _ = oracle_mod.segment_blocks(p, wl.seg_S, wl.seg_R, wl.retr_block, inp["is_long"], inp["q"],
                                              inp["k"])
        assert np.array_equal(pb.cpu().numpy(), ref_pb)
    ref = oracle_mod.segment_bwd(p, wl.seg_S, wl.seg_M, wl.seg_R, wl.retr_block, inp["is_long"], inp["q"], inp["k"],
                                 inp["v"], dO_h)
    for gname, t, r in (("dQ", dq, ref[0]), ("dK", dk, ref[1]), ("dV", dv, ref[2])):
        compare_grad(gname, t.float().cpu().numpy().astype(np.float64), r, BF16_GRAD_REL, BF16_GRAD_MEAN_REL)
    again = sa.segment_bwd(q, k, v, O, lse, pb, dO, **kw)
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip((dq, dk, dv), again))
