"""GPU parity of SharedLLM's tree cross-attention against the fp64 oracle.

The kept offsets within a chunk are compared bit-exactly; O and LSE with
the bf16 bars (max-abs 2e-2, mean-abs 2e-3).  Large cases check a seeded
sample of query rows (rows are independent: the oracle runs on those rows'
queries alone).
"""
import numpy as np
import pytest
import torch

import long_context_structured_b200 as sa
from long_context_structured_b200 import _lib
from _util import BF16_MAX_ABS, BF16_MEAN_ABS, compare, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _bits(g, *shape):
    x = g.standard_normal(shape).astype(np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


CASES = [
    # B, Hq, Hkv, T, d, n_chunks, chunk_len, depth, alpha_leaf, theta, sampled rows
    ("pow2_gqa", (1, 4, 2, 300, 128, 8, 512, 3, 1, 1e4, 0)),
    ("odd_chunks_d64", (2, 2, 2, 130, 64, 5, 1000, 2, 2, 5e5, 0)),
    ("depth0_dense_no_rope", (1, 2, 1, 257, 128, 3, 300, 0, 1, 0.0, 0)),
    ("deep_coarse", (1, 2, 2, 64, 128, 16, 777, 6, 3, 1e4, 0)),
    ("long_context_64k_kept", (1, 8, 8, 512, 128, 64, 2048, 3, 1, 1e4, 48)),
]


@pytest.mark.parametrize("name,cfg", CASES, ids=[c[0] for c in CASES])
def test_tree_cross_matches_oracle(oracle_mod, name, cfg):
    B, Hq, Hkv, T, d, n, l, D, alpha, theta, n_sample = cfg
    g = np.random.default_rng(hash(name) % 2 ** 32)
    q, k, v = _bits(g, B, Hq, T, d), _bits(g, B, Hkv, n * l, d), _bits(g, B, Hkv, n * l, d)
    O, lse, idx = sa.tree_cross_fwd(to_dev(q), to_dev(k), to_dev(v), n_chunks=n, chunk_len=l, depth=D,
                                    alpha_leaf=alpha, rope_theta=theta, with_index=True)
    torch.cuda.synchronize()
    assert sa.stream_status() == 0
    ref_idx = oracle_mod.tree_index(l, D, alpha)
    got_idx = idx.cpu().numpy()
    assert np.array_equal(got_idx[: len(ref_idx)], ref_idx)
    assert np.all(got_idx[len(ref_idx):] == -1)
    rows = np.arange(T) if not n_sample else np.sort(g.choice(T, n_sample, replace=False))
    qs = np.ascontiguousarray(q[:, :, rows])
    p = oracle_mod.params(B, Hq, Hkv, len(rows), d, "bf16", rope_theta=theta)
    Oref, lref = oracle_mod.tree_cross(p, n, l, D, alpha, qs, k, v)
    got = O[:, :, torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
    compare("O", got, Oref, BF16_MAX_ABS, BF16_MEAN_ABS)
    gl = lse[:, :, torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64)
    compare("LSE", gl, lref, BF16_MAX_ABS, BF16_MEAN_ABS)


def test_tree_cross_dense_equals_sdpa():
    """Depth 0 at rate 1 without rotation is plain unmasked attention over the
    whole context."""
    torch.manual_seed(3)
    B, H, T, d, n, l = 1, 4, 400, 128, 4, 640
    q = torch.randn(B, H, T, d, device="cuda").bfloat16()
    k = torch.randn(B, H, n * l, d, device="cuda").bfloat16()
    v = torch.randn(B, H, n * l, d, device="cuda").bfloat16()
    O, _ = sa.tree_cross_fwd(q, k, v, n_chunks=n, chunk_len=l, depth=0, alpha_leaf=1)
    ref = torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double())
    compare("O vs SDPA", O.double().cpu().numpy(), ref.cpu().numpy(), BF16_MAX_ABS, BF16_MEAN_ABS)


def test_tree_cross_rejects_bad_arguments():
    q = torch.zeros((1, 1, 8, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 1, 64, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_lib.SattnError):
        sa.tree_cross_fwd(q, k, k, n_chunks=2, chunk_len=32, depth=2, alpha_leaf=0)
    with pytest.raises(_lib.SattnError):
        sa.tree_cross_fwd(q, k, k, n_chunks=2, chunk_len=32, depth=21, alpha_leaf=1)
