"""Head-sharded forward on the GPU: each rank's block of kv-head groups run
through the library on its own, the blocks put back in head order, compared
bit for bit with the unsharded call and with the fp64 oracle.

One GPU stands in for the ranks by running their blocks one after another;
the blocks share no data and nothing waits on another rank, so this is the
same arithmetic each rank does on its own GPU.  The all-gather itself is
covered by the world-size-2 gloo test on CPU.
"""
import numpy as np
import pytest
import torch

import long_context_structured_b200 as sa
from long_context_structured_b200 import synth
from long_context_structured_b200.shard import head_shard, sharded_fwd
from _util import BF16_MAX_ABS, BF16_MEAN_ABS, compare, gather_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


CASES = [
    # the SepLLM GQA layer's mask at a small size, 3 ranks over 4 kv heads (uneven)
    ("sep_gqa_uneven", 3, dict(B=2, Hq=8, Hkv=4, T=700, d=128, n_start=4, window=64, rope_theta=5e5, sep_rate=0.1)),
    # capped top-k layer, 2 ranks
    ("topk_capped", 2, dict(B=1, Hq=4, Hkv=4, T=1500, d=128, n_start=4, window=256, L_pretrain=256,
                            rope_theta=1e4, topk=5)),
]


@pytest.mark.parametrize("name,world,cfg", CASES, ids=[c[0] for c in CASES])
def test_sharded_blocks_equal_unsharded(oracle_mod, name, world, cfg):
    wl = synth.Workload(name=name, dtype="bf16", **cfg)
    inp = synth.make_inputs(wl, seed=5)
    q, k, v = to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"])
    kw = dict(n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain, rope_theta=wl.rope_theta,
              topk=wl.topk, is_sep=to_dev(inp["is_sep"]))
    O_ref, lse_ref = sa.fwd(q, k, v, **kw)
    blocks = []
    for r in range(world):
        O, lse, (q0, q1) = sharded_fwd(q, k, v, world=world, rank=r, **kw)
        assert (q0, q1) == head_shard(wl.Hq, wl.Hkv, world, r)[:2]
        blocks.append((O, lse))
    torch.cuda.synchronize()
    assert sa.stream_status() == 0
    O_cat = torch.cat([b[0] for b in blocks], dim=1)
    lse_cat = torch.cat([b[1] for b in blocks], dim=1)
    assert torch.equal(O_cat, O_ref) and torch.equal(lse_cat, lse_ref)
    # and against the oracle on every row (the top-k case on rows whose
    # selection has no near tie is covered by the parity suite; here the
    # GPU's own selection is forced into the oracle)
    rows = oracle_mod.all_rows(wl.B, wl.Hq, wl.T)
    forced = None
    if wl.topk:
        idx, _ = sa.topk_select(q, k, topk=wl.topk, n_start=wl.n_start, window=wl.window,
                                L_pretrain=wl.L_pretrain, rope_theta=wl.rope_theta)
        forced = idx.cpu().numpy()
    p = oracle_mod.params_of(wl)
    Oo, lo, *_ = oracle_mod.fwd_rows(p, inp["q"], inp["k"], inp["v"], inp["is_sep"], rows, forced_topk=forced)
    compare("O", gather_rows(O_cat, rows), Oo, BF16_MAX_ABS, BF16_MEAN_ABS)
    compare("LSE", gather_rows(lse_cat, rows), lo, BF16_MAX_ABS, BF16_MEAN_ABS)
