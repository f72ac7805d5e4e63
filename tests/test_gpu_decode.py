"""GPU parity of the decoding step against the fp64 oracle.

A decoding step is row i = T-1 of the structured attention: the oracle's
row (b, h, T-1), computed from the materialised 0/1 mask, is the reference.
Bars as for the bf16 prefill: max-abs 2e-2, mean-abs 2e-3 on O and LSE.
"""
import numpy as np
import pytest
import torch

import long_context_structured_b200 as sa
from long_context_structured_b200 import _lib, synth
from _util import BF16_MAX_ABS, BF16_MEAN_ABS, compare, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _decode_and_check(oracle_mod, wl, seed):
    inp = synth.make_inputs(wl, seed=seed)
    q, k, v = (to_dev(inp[x]) for x in ("q", "k", "v"))
    sep = to_dev(inp["is_sep"])
    qd = q[:, :, wl.T - 1:wl.T, :].contiguous()
    O, lse = sa.decode_fwd(qd, k, v, n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain,
                           rope_theta=wl.rope_theta, is_sep=sep, rope_pos_scale=wl.rope_pos_scale, alibi=wl.alibi)
    torch.cuda.synchronize()
    assert sa.stream_status() == 0
    rows = np.array([(b, h, wl.T - 1) for b in range(wl.B) for h in range(wl.Hq)], dtype=np.int64)
    Oref, lref, *_ = oracle_mod.fwd_rows(oracle_mod.params_of(wl), inp["q"], inp["k"], inp["v"], inp["is_sep"],
                                         rows)
    got = O[:, :, 0, :].reshape(-1, wl.d).float().cpu().numpy().astype(np.float64)
    gl = lse.reshape(-1).float().cpu().numpy().astype(np.float64)
    compare("O", got, Oref, BF16_MAX_ABS, BF16_MEAN_ABS)
    compare("LSE", gl, lref, BF16_MAX_ABS, BF16_MEAN_ABS)
    return O, lse


CASES = [
    ("lambda_capped_sinks", dict(B=2, Hq=4, Hkv=4, T=1000, d=128, n_start=4, window=100, L_pretrain=100,
                                 rope_theta=1e4, sink_scale=8.0)),
    ("sep_gqa4_d64", dict(B=3, Hq=8, Hkv=2, T=777, d=64, n_start=4, window=37, rope_theta=5e5, sep_rate=0.1)),
    ("sep_capped_gqa8", dict(B=1, Hq=8, Hkv=1, T=600, d=128, n_start=2, window=50, L_pretrain=50,
                             rope_theta=1e4, sep_rate=0.3)),
    ("full_causal_no_rope", dict(B=1, Hq=2, Hkv=2, T=300, d=128, n_start=0, window=1000)),
    ("all_sinks", dict(B=1, Hq=2, Hkv=1, T=3, d=128, n_start=8, window=1, rope_theta=1e4)),
    ("window0_all_seps", dict(B=1, Hq=2, Hkv=2, T=257, d=128, n_start=1, window=0, sep_rate=1.0)),
    ("one_token", dict(B=2, Hq=2, Hkv=2, T=1, d=64, n_start=0, window=4, rope_theta=1e4)),
    ("pos_interp", dict(B=1, Hq=4, Hkv=1, T=900, d=128, n_start=4, window=64, L_pretrain=64, rope_theta=1e4,
                        sep_rate=0.1, rope_pos_scale=0.25)),
    ("alibi_capped_sep_gqa4", dict(B=2, Hq=8, Hkv=2, T=900, d=128, n_start=4, window=64, L_pretrain=64,
                                   sep_rate=0.1, alibi=True)),
    ("alibi_unclipped_sep_d64", dict(B=1, Hq=4, Hkv=4, T=500, d=64, n_start=2, window=40, sep_rate=0.2,
                                     alibi=True)),
    ("sep_capped_gqa2_d64", dict(B=2, Hq=4, Hkv=2, T=1500, d=64, n_start=4, window=80, L_pretrain=80,
                                 rope_theta=1e4, sep_rate=0.15)),
    # sink spans wider than 8
    ("sinks12_capped", dict(B=1, Hq=4, Hkv=2, T=1000, d=128, n_start=12, window=100, L_pretrain=100,
                            rope_theta=1e4, sink_scale=8.0)),
    ("sinks40_sep_capped_gqa8", dict(B=2, Hq=8, Hkv=1, T=900, d=128, n_start=40, window=64, L_pretrain=64,
                                     rope_theta=1e4, sep_rate=0.1)),
    ("sinks256_d64", dict(B=1, Hq=2, Hkv=2, T=700, d=64, n_start=256, window=30, rope_theta=5e5,
                          sep_rate=0.05)),
]


@pytest.mark.parametrize("name,cfg", CASES, ids=[c[0] for c in CASES])
def test_decode_matches_oracle(oracle_mod, name, cfg):
    wl = synth.Workload(name=name, dtype="bf16", **cfg)
    _decode_and_check(oracle_mod, wl, seed=13)


def test_decode_full_size_lambda(oracle_mod):
    """The 16K-token LM-Infinite layer's last position (32 heads)."""
    _decode_and_check(oracle_mod, synth.WORKLOADS["c2_lminf_16k"], seed=0)


def test_decode_full_size_sepllm_gqa(oracle_mod):
    """The SepLLM GQA layer's last positions (4 sequences, 32 query heads)."""
    _decode_and_check(oracle_mod, synth.WORKLOADS["c3_sepllm_gqa_8k"], seed=0)


def test_decode_deterministic_and_invariant_outside_kept_set():
    wl = synth.Workload(name="inv", B=1, Hq=4, Hkv=2, T=900, d=128, dtype="bf16", n_start=4, window=64,
                        L_pretrain=64, rope_theta=1e4, sep_rate=0.1)
    inp = synth.make_inputs(wl, seed=3)
    q, k, v = (to_dev(inp[x]) for x in ("q", "k", "v"))
    sep = to_dev(inp["is_sep"])
    kw = dict(n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain, rope_theta=wl.rope_theta, is_sep=sep)
    qd = q[:, :, -1:, :].contiguous()
    O1, l1 = sa.decode_fwd(qd, k, v, **kw)
    O2, l2 = sa.decode_fwd(qd, k, v, **kw)
    assert torch.equal(O1, O2) and torch.equal(l1, l2)
    # change K and V at positions the last row does not keep
    i = wl.T - 1
    flags = inp["is_sep"][0]
    kept = np.zeros(wl.T, dtype=bool)
    kept[: wl.n_start] = True
    kept[max(0, i - wl.window):] = True
    kept |= (flags != 0) & (np.arange(wl.T) < i - wl.window) & (np.arange(wl.T) >= wl.n_start)
    drop = torch.from_numpy(np.nonzero(~kept)[0]).cuda()
    k2, v2 = k.clone(), v.clone()
    k2[:, :, drop] = 3.0
    v2[:, :, drop] = -7.0
    O3, l3 = sa.decode_fwd(qd, k2, v2, **kw)
    assert torch.equal(O1, O3) and torch.equal(l1, l3)


def test_decode_rejects_unsupported():
    q = torch.zeros((1, 3, 1, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 1, 10, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_lib.SattnError):
        sa.decode_fwd(q, k, k)  # Hq / Hkv = 3


# ---------------------------------------------------------------------------
# top-k middle tokens during decoding
# ---------------------------------------------------------------------------

TOPK_CASES = [
    # capped (w = L) with planted clusters, GQA
    ("topk_capped_planted_gqa2", dict(B=2, Hq=4, Hkv=2, T=2048, d=128, n_start=4, window=256, L_pretrain=256,
                                      rope_theta=1e4, topk=5, plant=3)),
    # window below the cap: candidates on both sides of it; separators excluded
    ("topk_window_below_cap_sep_gqa8_d64", dict(B=1, Hq=8, Hkv=1, T=1500, d=64, n_start=2, window=60,
                                                L_pretrain=300, rope_theta=5e5, topk=8, sep_rate=0.15)),
    # uncapped, k = 16, separators
    ("topk16_uncapped_sep", dict(B=2, Hq=2, Hkv=2, T=900, d=128, n_start=4, window=100, rope_theta=1e4,
                                 topk=16, sep_rate=0.1)),
    # clipped ALiBi past the cap
    ("topk_alibi_capped_gqa4", dict(B=1, Hq=8, Hkv=2, T=1200, d=128, n_start=4, window=64, L_pretrain=64,
                                    topk=3, alibi=True)),
    # fewer candidates than k: all of them, then -1 / -inf padding
    ("topk_few_candidates", dict(B=1, Hq=2, Hkv=1, T=40, d=128, n_start=4, window=30, L_pretrain=30,
                                 rope_theta=1e4, topk=8)),
    # no candidate at all
    ("topk_no_candidates", dict(B=1, Hq=2, Hkv=2, T=20, d=64, n_start=4, window=30, L_pretrain=30,
                                rope_theta=1e4, topk=4)),
]


def _decode_topk_and_check(oracle_mod, wl, seed):
    from _util import TOPK_EXT, topk_agreement
    inp = synth.make_inputs(wl, seed=seed)
    q, k, v = (to_dev(inp[x]) for x in ("q", "k", "v"))
    sep = to_dev(inp["is_sep"])
    qd = q[:, :, wl.T - 1:wl.T, :].contiguous()
    O, lse, idx, z = sa.decode_fwd(qd, k, v, n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain,
                                   rope_theta=wl.rope_theta, is_sep=sep, alibi=wl.alibi, topk=wl.topk,
                                   return_topk=True)
    torch.cuda.synchronize()
    assert sa.stream_status() == 0
    rows = np.array([(b, h, wl.T - 1) for b in range(wl.B) for h in range(wl.Hq)], dtype=np.int64)
    # the selection: the oracle's own, bit-exact up to the near-tie rule
    p_ext = oracle_mod.params_of(wl.scaled(topk=wl.topk + TOPK_EXT))
    _, _, ref_idx, ref_z, _ = oracle_mod.fwd_rows(p_ext, inp["q"], inp["k"], inp["v"], inp["is_sep"], rows)
    gi = idx.reshape(-1, wl.topk).cpu().numpy()
    n_exact, n_exempt, bad = topk_agreement(gi, ref_idx, ref_z, wl.topk)
    assert not bad, "rows differ beyond the near-tie rule: %s" % bad[:10]
    gz = z.reshape(-1, wl.topk).cpu().numpy().astype(np.float64)
    same = np.all(gi == ref_idx[:, : wl.topk], axis=1)
    fin = np.isfinite(ref_z[same, : wl.topk])
    assert np.allclose(gz[same][fin], ref_z[same, : wl.topk][fin], rtol=1e-5, atol=1e-4)
    assert np.all(np.isneginf(gz[gi < 0]))
    # the step against the oracle's row with the GPU's selection
    Oref, lref, *_ = oracle_mod.fwd_rows(oracle_mod.params_of(wl), inp["q"], inp["k"], inp["v"], inp["is_sep"],
                                         rows, forced_topk=gi)
    got = O[:, :, 0, :].reshape(-1, wl.d).float().cpu().numpy().astype(np.float64)
    gl = lse.reshape(-1).float().cpu().numpy().astype(np.float64)
    compare("O", got, Oref, BF16_MAX_ABS, BF16_MEAN_ABS)
    compare("LSE", gl, lref, BF16_MAX_ABS, BF16_MEAN_ABS)
    # the step without return_topk is the same call
    O2, lse2 = sa.decode_fwd(qd, k, v, n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain,
                             rope_theta=wl.rope_theta, is_sep=sep, alibi=wl.alibi, topk=wl.topk)
    assert torch.equal(O2, O) and torch.equal(lse2, lse)
    return gi


@pytest.mark.parametrize("name,cfg", TOPK_CASES, ids=[c[0] for c in TOPK_CASES])
def test_decode_topk_matches_oracle(oracle_mod, name, cfg):
    wl = synth.Workload(name=name, dtype="bf16", **cfg)
    gi = _decode_topk_and_check(oracle_mod, wl, seed=23)
    if name == "topk_no_candidates":
        assert np.all(gi == -1)
    if name == "topk_few_candidates":
        n_cand = wl.T - 1 - wl.window - wl.n_start
        assert np.all(gi[:, :n_cand] >= 0) and np.all(gi[:, n_cand:] == -1)


def test_decode_topk_full_size():
    """The 32K-token top-k layer's last position (32 heads, k = 5, planted
    clusters), against the oracle."""
    from oracle import oracle as O
    O.build()
    _decode_topk_and_check(O, synth.WORKLOADS["c4_lminf_topk_32k"], seed=0)


def test_decode_topk_alibi_below_cap_rejected():
    q = torch.zeros((1, 2, 1, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((1, 2, 300, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_lib.SattnError):
        sa.decode_fwd(q, kv, kv, n_start=4, window=30, L_pretrain=100, topk=2, alibi=True)


def _padded(t, pad=8):
    """The same values in a [B, H, T, d] view whose rows are d + pad apart."""
    B, H, T, d = t.shape
    buf = torch.full((B, H, T, d + pad), 5.0, dtype=t.dtype, device=t.device)
    buf[..., :d] = t
    return buf[..., :d]


@pytest.mark.parametrize("name,cfg", [TOPK_CASES[0], TOPK_CASES[1], CASES[0]], ids=lambda x: x if isinstance(x, str) else "")
def test_decode_strided_cache_equals_contiguous(name, cfg):
    """A cache whose rows are not adjacent is staged piece by piece instead
    of by one bulk copy per chunk; the step is the same bit for bit."""
    wl = synth.Workload(name=name, dtype="bf16", **cfg)
    inp = synth.make_inputs(wl, seed=31)
    q, k, v = (to_dev(inp[x]) for x in ("q", "k", "v"))
    sep = to_dev(inp["is_sep"])
    qd = q[:, :, wl.T - 1:wl.T, :].contiguous()
    kw = dict(n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain, rope_theta=wl.rope_theta, is_sep=sep,
              alibi=wl.alibi, topk=wl.topk)
    kp, vp = _padded(k), _padded(v)
    assert kp.stride(2) == wl.d + 8 and not kp.is_contiguous()
    if wl.topk > 0:
        a = sa.decode_fwd(qd, k, v, return_topk=True, **kw)
        b = sa.decode_fwd(qd, kp, vp, return_topk=True, **kw)
    else:
        a = sa.decode_fwd(qd, k, v, **kw)
        b = sa.decode_fwd(qd, kp, vp, **kw)
    torch.cuda.synchronize()
    assert sa.stream_status() == 0
    for x, y in zip(a, b):
        assert torch.equal(x, y)
