"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs.

Bars: block maps, separator lists, top-k selections and retrieved prefix
blocks bit-exact (top-k / retrieval rows exempt only where the oracle's k-th
and (k+1)-th logits are within 1e-4 relative, and then only inside that tied
run: ``_util.topk_row_verdict``); O and LSE within max-abs 2e-2 and mean-abs
2e-3 for bf16 inputs, 1e-4 for the fp32 path.
"""
import numpy as np
import pytest
import torch

import long_context_structured_b200 as sa
from long_context_structured_b200 import _lib, synth
from _util import (BF16_MAX_ABS, BF16_MEAN_ABS, F32_MAX_ABS, TOPK_EXT, compare, gather_rows, to_dev,
                   topk_agreement)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _status_ok():
    assert sa.stream_status() == 0, "device status word reports a failure"


def _run_fwd(wl, inp, **kw):
    q, k, v = to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"])
    sep = to_dev(inp["is_sep"])
    O, lse = sa.fwd(q, k, v, n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain,
                    rope_theta=wl.rope_theta, topk=wl.topk, is_sep=sep, rope_pos_scale=wl.rope_pos_scale,
                    alibi=wl.alibi, **kw)
    torch.cuda.synchronize()
    _status_ok()
    return O, lse


def _check_fwd_rows(oracle_mod, wl, inp, O, lse, rows, forced=None):
    p = oracle_mod.params_of(wl)
    Oref, lref, *_ = oracle_mod.fwd_rows(p, inp["q"], inp["k"], inp["v"], inp["is_sep"], rows, forced_topk=forced)
    Og = gather_rows(O, rows)
    lg = gather_rows(lse, rows)
    if wl.dtype == "f32":
        compare("O", Og, Oref, F32_MAX_ABS)
        compare("LSE", lg, lref, F32_MAX_ABS)
    else:
        compare("O", Og, Oref, BF16_MAX_ABS, BF16_MEAN_ABS)
        compare("LSE", lg, lref, BF16_MAX_ABS, BF16_MEAN_ABS)


# ---------------------------------------------------------------------------
# block map (integer, bit-exact)
# ---------------------------------------------------------------------------

# Shapes reach both class paths (16-byte pieces when the tile count is a
# multiple of 16, bytes otherwise), band tables as wide as the whole row
# (window >= T), sinks over several tiles, a last flag word that is cut short
# and rows whose flags are not 16-byte aligned (T % 16 != 0).
@pytest.mark.parametrize("B,T,ns,w,rate", [(1, 1024, 4, 128, 0.08), (3, 1000, 4, 37, 0.2), (2, 300, 0, 0, 0.5),
                                           (1, 129, 7, 300, 1.0), (4, 8192, 4, 256, 0.10), (2, 777, 2, 5, 0.0),
                                           (2, 4096, 250, 700, 0.3), (1, 6149, 3, 5000, 0.05),
                                           (2, 16384, 0, 20000, 0.1), (2, 4096, 4, 0, 1.0), (2, 4112, 4, 128, 0.2),
                                           (1, 2048, 200, 100, 0.0)])
def test_blockmap_bitexact(oracle_mod, B, T, ns, w, rate):
    rng = np.random.default_rng(B * 1000 + T)
    flags = (rng.random((B, T)) < rate).astype(np.uint8)
    out = sa.build_blockmap(to_dev(flags), B=B, T=T, n_start=ns, window=w)
    torch.cuda.synchronize()
    cls, pos, cnt, rng_ = oracle_mod.blockmap(B, T, ns, w, 128, 128, flags)
    assert np.array_equal(out["sep_count"].cpu().numpy(), cnt)
    assert np.array_equal(out["sep_pos"].cpu().numpy(), pos)
    assert np.array_equal(out["qtile_sep_range"].cpu().numpy(), rng_)
    assert np.array_equal(out["cls"].cpu().numpy(), cls)


def test_blockmap_stress_launch_sampled(oracle_mod):
    """The block map at 2048 sequences x 32768 flags (2^26, the stress size
    the benchmark times), checked on sampled sequences: each sequence is
    computed independently, so the oracle runs on those alone."""
    B, T, ns, w = 2048, 32768, 4, 256
    g = torch.Generator().manual_seed(0)
    flags = (torch.rand(B, T, generator=g) < 0.1).to(torch.uint8)
    out = sa.build_blockmap(flags.cuda(), B=B, T=T, n_start=ns, window=w)
    torch.cuda.synchronize()
    for b in (0, 1337, B - 1):
        f = flags[b:b + 1].numpy()
        cls, pos, cnt, rng_ = oracle_mod.blockmap(1, T, ns, w, 128, 128, f)
        assert int(out["sep_count"][b]) == int(cnt[0])
        assert np.array_equal(out["sep_pos"][b].cpu().numpy(), pos[0])
        assert np.array_equal(out["qtile_sep_range"][b].cpu().numpy(), rng_[0])
        assert np.array_equal(out["cls"][b].cpu().numpy(), cls[0])


def test_blockmap_c3_token_flags(oracle_mod):
    wl = synth.WORKLOADS["c3_sepllm_gqa_8k"]
    flags = synth.separator_flags(wl, 0)
    out = sa.build_blockmap(to_dev(flags), B=wl.B, T=wl.T, n_start=wl.n_start, window=wl.window)
    cls, pos, cnt, rng_ = oracle_mod.blockmap(wl.B, wl.T, wl.n_start, wl.window, 128, 128, flags)
    assert np.array_equal(out["sep_count"].cpu().numpy(), cnt)
    assert np.array_equal(out["sep_pos"].cpu().numpy(), pos)
    assert np.array_equal(out["qtile_sep_range"].cpu().numpy(), rng_)
    assert np.array_equal(out["cls"].cpu().numpy(), cls)


def _tile_class_bruteforce(oracle_mod, T, ns, w, flags, t, u):
    """Class of tile (t, u) from the oracle's materialised mask rows."""
    i0, i1 = t * 128, min(T, t * 128 + 128)
    j0, j1 = u * 128, min(T, u * 128 + 128)
    kept = np.stack([oracle_mod.mask_row(T, i, ns, w, flags)[0][j0:j1] for i in range(i0, i1)])
    return 2 if kept.all() else (1 if kept.any() else 0)


@pytest.mark.parametrize("noalloc", [False, True], ids=["workspace", "noalloc"])
def test_blockmap_long_row_properties(oracle_mod, noalloc):
    """One sequence of 400,003 flags: the separator word prefix (8 bytes per
    32 positions, 100 KB) no longer fits the scan kernel's shared-memory
    stage, so it is read from global memory.  The brute-force block map is
    quadratic in T, so the check is by properties: separator positions
    against numpy's nonzero, counts, per-tile ranges against prefix counts,
    and sampled tiles (sink, diagonal, band edge, far) against the oracle's
    mask rows."""
    B, T, ns, w = 1, 400003, 4, 128
    rng = np.random.default_rng(400003)
    flags = (rng.random((B, T)) < 0.08).astype(np.uint8)
    if noalloc:
        out = sa.build_blockmap_noalloc(to_dev(flags), B=B, T=T, n_start=ns, window=w)
    else:
        out = sa.build_blockmap(to_dev(flags), B=B, T=T, n_start=ns, window=w)
    torch.cuda.synchronize()
    f = flags[0]
    ref_pos = np.flatnonzero(f[ns:]) + ns
    cnt = int(out["sep_count"][0])
    assert cnt == len(ref_pos)
    pos = out["sep_pos"][0].cpu().numpy()
    assert np.array_equal(pos[:cnt], ref_pos) and np.all(pos[cnt:] == -1)
    nQT = -(-T // 128)
    t = np.arange(nQT)
    last = np.minimum(T - 1, t * 128 + 127)
    full_end = np.searchsorted(ref_pos, t * 128 - w, side="left")
    end = np.searchsorted(ref_pos, last - w, side="left")
    rng_ = out["qtile_sep_range"][0].cpu().numpy()
    assert np.array_equal(rng_[:, 0], full_end) and np.array_equal(rng_[:, 1], end)
    cls = out["cls"][0].cpu().numpy()
    assert cls.shape == (nQT, nQT)
    assert np.all(np.triu(cls, 1) == 0)  # above the diagonal nothing is kept
    srng = np.random.default_rng(5)
    tiles = []
    for tq in [0, 1, 2, 1000, nQT // 2, nQT - 2, nQT - 1] + list(srng.integers(3, nQT, 4)):
        for u in {0, tq, tq - 1, tq - 2, int(srng.integers(0, max(1, tq - 2)))}:
            if 0 <= u <= tq:
                tiles.append((int(tq), int(u)))
    for tq, u in tiles:
        assert cls[tq, u] == _tile_class_bruteforce(oracle_mod, T, ns, w, f, tq, u), (tq, u)


def test_fwd_long_row_separators_sampled(oracle_mod):
    """The forward on a 400,003-token SepLLM-mask sequence (about 32K
    separators, word prefix in global memory), sampled rows."""
    wl = synth.Workload(name="long_row", B=1, Hq=1, Hkv=1, T=400003, d=128, dtype="bf16", n_start=4,
                        window=128, rope_theta=5e5, sep_rate=0.08)
    inp = synth.make_inputs(wl, seed=2)
    O, lse = _run_fwd(wl, inp)
    rows = synth.sample_rows(wl, 24, seed=6)
    _check_fwd_rows(oracle_mod, wl, inp, O, lse, rows)


# ---------------------------------------------------------------------------
# fp32 path
# ---------------------------------------------------------------------------

def test_c1_f32_full(oracle_mod):
    wl = synth.WORKLOADS["c1_f32_sep"]
    inp = synth.make_inputs(wl, seed=0)
    O, lse = _run_fwd(wl, inp)
    rows = oracle_mod.all_rows(wl.B, wl.Hq, wl.T)
    _check_fwd_rows(oracle_mod, wl, inp, O, lse, rows)


@pytest.mark.parametrize("cfg", [
    dict(B=1, Hq=2, Hkv=1, T=300, d=64, n_start=2, window=20, L_pretrain=40, rope_theta=1e4, topk=3, sep_rate=0.1),
    dict(B=2, Hq=2, Hkv=2, T=200, d=128, n_start=0, window=199, rope_theta=5e5),
    # clipped ALiBi: separators at their own (unclipped) distance; top-k past the cap; window below the cap
    dict(B=1, Hq=4, Hkv=2, T=300, d=64, n_start=3, window=20, sep_rate=0.15, alibi=True),
    dict(B=1, Hq=4, Hkv=1, T=250, d=128, n_start=2, window=30, L_pretrain=30, topk=3, sep_rate=0.1, alibi=True),
    dict(B=1, Hq=2, Hkv=2, T=260, d=64, n_start=4, window=20, L_pretrain=60, sep_rate=0.1, alibi=True),
])
def test_f32_features(oracle_mod, cfg):
    wl = synth.Workload(name="f32", dtype="f32", **cfg)
    inp = synth.make_inputs(wl, seed=5)
    O, lse = _run_fwd(wl, inp)
    _check_fwd_rows(oracle_mod, wl, inp, O, lse, oracle_mod.all_rows(wl.B, wl.Hq, wl.T))


# ---------------------------------------------------------------------------
# bf16 tensor-core path, small shapes, every row
# ---------------------------------------------------------------------------

SMALL = [
    ("dense_one_tile", dict(B=1, Hq=1, Hkv=1, T=128, d=128, n_start=0, window=127)),
    ("causal_ragged_rope", dict(B=1, Hq=2, Hkv=2, T=300, d=128, n_start=0, window=1000, rope_theta=1e4)),
    ("lambda_capped_gqa", dict(B=1, Hq=2, Hkv=1, T=1000, d=128, n_start=4, window=100, L_pretrain=100,
                               rope_theta=1e4, sink_scale=8.0)),
    ("sep_d64", dict(B=2, Hq=4, Hkv=2, T=700, d=64, n_start=1, window=37, rope_theta=1e4, sep_rate=0.1)),
    ("sep_capped_q2", dict(B=1, Hq=2, Hkv=2, T=513, d=128, n_start=4, window=64, L_pretrain=64, rope_theta=1e4,
                           sep_rate=0.3)),
    ("window0_sep", dict(B=1, Hq=2, Hkv=2, T=400, d=128, n_start=0, window=0, sep_rate=0.5)),
    ("all_separators", dict(B=1, Hq=1, Hkv=1, T=200, d=128, n_start=4, window=3, sep_rate=1.0)),
    ("tiny_T", dict(B=1, Hq=1, Hkv=1, T=5, d=128, n_start=4, window=2, rope_theta=1e4)),
    ("all_sinks", dict(B=1, Hq=1, Hkv=1, T=3, d=128, n_start=8, window=1)),
    ("window_uncapped_long", dict(B=1, Hq=1, Hkv=1, T=900, d=128, n_start=4, window=200, L_pretrain=300,
                                  rope_theta=1e4)),
    ("pos_interp_capped_sinks", dict(B=1, Hq=2, Hkv=2, T=1000, d=128, n_start=4, window=100, L_pretrain=100,
                                     rope_theta=1e4, sink_scale=8.0, rope_pos_scale=0.25)),
    ("pos_interp_sep_gqa", dict(B=2, Hq=4, Hkv=2, T=700, d=64, n_start=2, window=40, rope_theta=5e5,
                                sep_rate=0.15, rope_pos_scale=0.5)),
    # clipped ALiBi (LM-Infinite, section 方法): band keys -m (i - j), keys past the cap -m L
    ("alibi_causal_h8", dict(B=1, Hq=8, Hkv=2, T=700, d=128, n_start=0, window=1000, alibi=True)),
    ("alibi_lambda_capped", dict(B=1, Hq=4, Hkv=1, T=1000, d=128, n_start=4, window=100, L_pretrain=100,
                                 sink_scale=8.0, alibi=True)),
    ("alibi_sep_capped_d64", dict(B=2, Hq=4, Hkv=2, T=600, d=64, n_start=4, window=64, L_pretrain=64,
                                  sep_rate=0.2, alibi=True)),
    ("alibi_window_below_cap", dict(B=1, Hq=2, Hkv=2, T=800, d=128, n_start=4, window=50, L_pretrain=200,
                                    sink_scale=8.0, alibi=True)),
    ("alibi_sep_capped_even", dict(B=1, Hq=2, Hkv=1, T=1024, d=128, n_start=4, window=128, L_pretrain=128,
                                   sep_rate=0.1, alibi=True)),
    # separators with the window below the cap: those with w < i - j <= L
    # are uncapped and ride in the band tiles, the farther ones capped
    ("sep_window_below_cap", dict(B=1, Hq=2, Hkv=2, T=900, d=128, n_start=4, window=64, L_pretrain=128,
                                  rope_theta=1e4, sep_rate=0.1)),
    ("sep_window_below_cap_d64_gqa", dict(B=2, Hq=4, Hkv=2, T=700, d=64, n_start=2, window=30, L_pretrain=200,
                                          rope_theta=5e5, sep_rate=0.2)),
    ("alibi_sep_window_below_cap", dict(B=1, Hq=4, Hkv=1, T=800, d=128, n_start=4, window=40, L_pretrain=150,
                                        sep_rate=0.15, alibi=True)),
    ("sep_window0_capped", dict(B=1, Hq=2, Hkv=2, T=600, d=128, n_start=4, window=0, L_pretrain=100,
                                rope_theta=1e4, sep_rate=0.5)),
    # sink spans wider than 8: the 16-slot sink logits (9..16) and the
    # global-memory ones (> 16) in prep and in the attention epilogue
    ("sinks12_capped", dict(B=1, Hq=2, Hkv=1, T=1000, d=128, n_start=12, window=100, L_pretrain=100,
                            rope_theta=1e4, sink_scale=8.0)),
    ("sinks16_sep_d64", dict(B=2, Hq=4, Hkv=2, T=700, d=64, n_start=16, window=40, rope_theta=5e5,
                             sep_rate=0.1)),
    ("sinks40_sep_capped", dict(B=1, Hq=2, Hkv=2, T=900, d=128, n_start=40, window=64, L_pretrain=64,
                                rope_theta=1e4, sep_rate=0.1, sink_scale=8.0)),
    ("sinks200_capped_d64", dict(B=1, Hq=2, Hkv=1, T=700, d=64, n_start=200, window=64, L_pretrain=64,
                                 rope_theta=1e4)),
    ("sinks256_uncapped", dict(B=1, Hq=1, Hkv=1, T=600, d=128, n_start=256, window=30, rope_theta=1e4,
                               sep_rate=0.05)),
]


@pytest.mark.parametrize("name,cfg", SMALL, ids=[s[0] for s in SMALL])
def test_bf16_small(oracle_mod, name, cfg):
    wl = synth.Workload(name=name, dtype="bf16", **cfg)
    inp = synth.make_inputs(wl, seed=7)
    O, lse = _run_fwd(wl, inp)
    _check_fwd_rows(oracle_mod, wl, inp, O, lse, oracle_mod.all_rows(wl.B, wl.Hq, wl.T))


def test_bf16_topk_small(oracle_mod):
    wl = synth.Workload(name="topk_small", B=1, Hq=2, Hkv=2, T=2048, d=128, dtype="bf16", n_start=4, window=256,
                        L_pretrain=256, rope_theta=1e4, topk=5, plant=2)
    inp = synth.make_inputs(wl, seed=11)
    q, k = to_dev(inp["q"]), to_dev(inp["k"])
    idx, z = sa.topk_select(q, k, topk=wl.topk, n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain,
                            rope_theta=wl.rope_theta)
    torch.cuda.synchronize()
    _status_ok()
    rows = oracle_mod.all_rows(wl.B, wl.Hq, wl.T)
    p_ext = oracle_mod.params_of(wl.scaled(topk=wl.topk + TOPK_EXT))
    _, _, ref_idx, ref_z, _ = oracle_mod.fwd_rows(p_ext, inp["q"], inp["k"], inp["v"], None, rows)
    gi = idx.cpu().numpy().reshape(-1, wl.topk)
    n_exact, n_exempt, bad = topk_agreement(gi, ref_idx, ref_z, wl.topk)
    assert not bad, "rows differ beyond the near-tie rule: %s" % bad[:10]
    # logits of agreeing rows match the oracle's in fp32
    gz = z.cpu().numpy().reshape(-1, wl.topk).astype(np.float64)
    same = np.all(gi == ref_idx[:, : wl.topk], axis=1)
    fin = np.isfinite(ref_z[same, : wl.topk])
    assert np.allclose(gz[same][fin], ref_z[same, : wl.topk][fin], rtol=1e-5, atol=1e-4)
    # attention with the selection inside the call
    O, lse = _run_fwd(wl, inp)
    _check_fwd_rows(oracle_mod, wl, inp, O, lse, rows, forced=gi)


def test_bf16_topk_alibi(oracle_mod):
    """Top-k with the clipped ALiBi bias: every candidate is past the cap
    (L = w), so the ranking is by q.k and the gathered keys carry -m L."""
    wl = synth.Workload(name="topk_alibi", B=1, Hq=4, Hkv=2, T=1536, d=128, dtype="bf16", n_start=4, window=128,
                        L_pretrain=128, topk=4, plant=2, alibi=True)
    inp = synth.make_inputs(wl, seed=12)
    q, k = to_dev(inp["q"]), to_dev(inp["k"])
    idx, _ = sa.topk_select(q, k, topk=wl.topk, n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain,
                            alibi=True)
    torch.cuda.synchronize()
    _status_ok()
    rows = oracle_mod.all_rows(wl.B, wl.Hq, wl.T)
    _, _, ref_idx, ref_z, _ = oracle_mod.fwd_rows(oracle_mod.params_of(wl.scaled(topk=wl.topk + TOPK_EXT)),
                                                  inp["q"], inp["k"], inp["v"], None, rows)
    gi = idx.cpu().numpy().reshape(-1, wl.topk)
    _, _, bad = topk_agreement(gi, ref_idx, ref_z, wl.topk)
    assert not bad, "rows differ beyond the near-tie rule: %s" % bad[:10]
    O, lse = _run_fwd(wl, inp)
    _check_fwd_rows(oracle_mod, wl, inp, O, lse, rows, forced=gi)


TOPK_CASES = [
    # LM-Infinite top-k together with SepLLM separators (candidates exclude
    # the separators the mask already keeps), the capped rule with w = L
    ("topk_separators", dict(B=1, Hq=4, Hkv=2, T=4096, d=128, n_start=4, window=512, L_pretrain=512,
                             rope_theta=1e4, topk=5, plant=4, sep_rate=0.1)),
    ("topk_d64", dict(B=2, Hq=2, Hkv=1, T=2048, d=64, n_start=4, window=256, L_pretrain=256, rope_theta=1e4,
                      topk=5, plant=3)),
    ("topk_d64_separators_k8", dict(B=1, Hq=2, Hkv=2, T=1500, d=64, n_start=2, window=128, L_pretrain=128,
                                    rope_theta=5e5, topk=8, plant=2, sep_rate=0.2)),
    ("topk_sinks40", dict(B=1, Hq=2, Hkv=1, T=2048, d=128, n_start=40, window=256, L_pretrain=256,
                          rope_theta=1e4, topk=4, plant=2, sink_scale=8.0)),
    ("topk_uncapped_k16_separators", dict(B=1, Hq=2, Hkv=2, T=1200, d=128, n_start=4, window=100,
                                          rope_theta=1e4, topk=16, sep_rate=0.05)),
    # the window below the cap: candidates with w < i - j <= L scored with the
    # uncapped pair, the farther ones capped, key tiles straddling i - L both
    # ways; long rows (sampled threshold), short rows (every tile sampled)
    ("topk_window_below_cap_sep", dict(B=1, Hq=4, Hkv=2, T=4096, d=128, n_start=4, window=256, L_pretrain=512,
                                       rope_theta=1e4, topk=5, plant=4, sep_rate=0.1)),
    ("topk_window_below_cap_d64_k8", dict(B=2, Hq=2, Hkv=1, T=2048, d=64, n_start=4, window=100, L_pretrain=300,
                                          rope_theta=5e5, topk=8, plant=2)),
    ("topk_window_below_cap_short", dict(B=1, Hq=2, Hkv=2, T=1000, d=128, n_start=2, window=50, L_pretrain=200,
                                         rope_theta=1e4, topk=4, sep_rate=0.05)),
]


@pytest.mark.parametrize("name,cfg", TOPK_CASES, ids=[c[0] for c in TOPK_CASES])
def test_bf16_topk_selection_unforced(oracle_mod, name, cfg):
    """The GPU selection against the oracle's own selection on every row
    (bit-exact up to the near-tie rule), then the forward with the selection
    made inside the call against the oracle forced to the GPU's picks."""
    wl = synth.Workload(name=name, dtype="bf16", **cfg)
    inp = synth.make_inputs(wl, seed=17)
    q, k = to_dev(inp["q"]), to_dev(inp["k"])
    sep = to_dev(inp["is_sep"])
    idx, z = sa.topk_select(q, k, topk=wl.topk, n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain,
                            rope_theta=wl.rope_theta, is_sep=sep)
    torch.cuda.synchronize()
    _status_ok()
    rows = oracle_mod.all_rows(wl.B, wl.Hq, wl.T)
    p_ext = oracle_mod.params_of(wl.scaled(topk=wl.topk + TOPK_EXT))
    _, _, ref_idx, ref_z, _ = oracle_mod.fwd_rows(p_ext, inp["q"], inp["k"], inp["v"], inp["is_sep"], rows)
    gi = idx.cpu().numpy().reshape(-1, wl.topk)
    n_exact, n_exempt, bad = topk_agreement(gi, ref_idx, ref_z, wl.topk)
    print("%s: %d rows exact, %d exempt" % (name, n_exact, n_exempt))
    assert not bad, "rows differ beyond the near-tie rule: %s" % bad[:10]
    assert n_exempt <= max(2, len(rows) // 100)
    if inp["is_sep"] is not None:  # no separator is ever picked
        flags = inp["is_sep"]
        b_of = rows[:, 0]
        picked = gi >= 0
        assert not np.any(flags[b_of[:, None].repeat(wl.topk, 1)[picked], gi[picked]])
    gz = z.cpu().numpy().reshape(-1, wl.topk).astype(np.float64)
    same = np.all(gi == ref_idx[:, : wl.topk], axis=1)
    fin = np.isfinite(ref_z[same, : wl.topk])
    assert np.allclose(gz[same][fin], ref_z[same, : wl.topk][fin], rtol=1e-5, atol=1e-4)
    O, lse = _run_fwd(wl, inp)
    _check_fwd_rows(oracle_mod, wl, inp, O, lse, rows, forced=gi)


def test_alibi_rejects_unsupported():
    q = torch.zeros((1, 2, 256, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_lib.SattnError):
        sa.fwd(q, q, q, window=8, rope_theta=1e4, alibi=True)  # ALiBi replaces the rotation
    with pytest.raises(_lib.SattnError):
        sa.fwd(q, q, q, window=8, topk=2, alibi=True)          # uncapped bias would reorder top-k
    with pytest.raises(_lib.SattnError):
        sa.fwd(q, q, q, window=8, L_pretrain=16, topk=2, alibi=True)


# ---------------------------------------------------------------------------
# properties on the GPU
# ---------------------------------------------------------------------------

def test_full_causal_matches_sdpa():
    torch.manual_seed(0)
    B, H, T, d = 1, 4, 1000, 128
    q = torch.randn(B, H, T, d, device="cuda").bfloat16()
    k = torch.randn(B, H, T, d, device="cuda").bfloat16()
    v = torch.randn(B, H, T, d, device="cuda").bfloat16()
    O, lse = sa.fwd(q, k, v, n_start=0, window=T)
    ref = torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double(), is_causal=True)
    compare("O vs SDPA", O.double().cpu().numpy(), ref.cpu().numpy(), BF16_MAX_ABS, BF16_MEAN_ABS)


def test_invariant_outside_kept_set():
    wl = synth.Workload(name="inv", B=1, Hq=1, Hkv=1, T=1500, d=128, dtype="bf16", n_start=4, window=100,
                        L_pretrain=100, rope_theta=1e4, sep_rate=0.05)
    inp = synth.make_inputs(wl, seed=3)
    O0, l0 = _run_fwd(wl, inp)
    i = 1400
    flags = inp["is_sep"][0]
    keep = np.zeros(wl.T, bool)
    keep[: wl.n_start] = True
    keep[i - wl.window: i + 1] = True
    keep[np.flatnonzero(flags[: i])] = True
    inp2 = dict(inp)
    v2 = inp["v"].copy()
    k2 = inp["k"].copy()
    out_idx = np.flatnonzero(~keep[: i])
    v2[0, 0, out_idx] ^= np.uint16(0x0123)
    k2[0, 0, out_idx] ^= np.uint16(0x0101)
    inp2["v"], inp2["k"] = v2, k2
    O1, l1 = _run_fwd(wl, inp2)
    assert torch.equal(O0[0, 0, i], O1[0, 0, i]) and torch.equal(l0[0, 0, i], l1[0, 0, i])


def test_deterministic():
    wl = synth.Workload(name="det", B=1, Hq=2, Hkv=2, T=2000, d=128, dtype="bf16", n_start=4, window=500,
                        L_pretrain=500, rope_theta=1e4, topk=3)
    inp = synth.make_inputs(wl, seed=4)
    a = _run_fwd(wl, inp)
    b = _run_fwd(wl, inp)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("B,Hq,Hkv,sep", [(1, 8, 8, 0.0), (1, 8, 2, 0.1), (3, 4, 2, 0.1)])
def test_host_tensors_end_to_end(B, Hq, Hkv, sep):
    """The host-tensor path (pieces copied, computed and copied back on two
    streams) gives the device path's result bit for bit."""
    wl = synth.Workload(name="e2e", B=B, Hq=Hq, Hkv=Hkv, T=600, d=128, dtype="bf16", n_start=4, window=128,
                        L_pretrain=0 if sep else 128, rope_theta=1e4, sep_rate=sep)
    inp = synth.make_inputs(wl, seed=9)
    Od, ld = _run_fwd(wl, inp)
    qh, kh, vh = (to_dev(inp[x], device="cpu") for x in ("q", "k", "v"))
    sep_h = None if inp["is_sep"] is None else torch.from_numpy(inp["is_sep"])
    Oh, lh = sa.fwd(qh, kh, vh, n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain,
                    rope_theta=wl.rope_theta, is_sep=sep_h)
    assert Oh.device.type == "cpu" and Oh.is_pinned()
    assert torch.equal(Oh, Od.cpu()) and torch.equal(lh, ld.cpu())


def test_host_tensors_segmented():
    wl = synth.Workload(name="e2e_seg", B=1, Hq=4, Hkv=4, T=1024, d=128, dtype="bf16", rope_theta=1e4,
                        seg_S=256, seg_M=64, seg_R=128, retr_block=32, long_heads=(1, 3))
    inp = synth.make_inputs(wl, seed=4)
    q, k, v = (to_dev(inp[x]) for x in ("q", "k", "v"))
    kw = dict(S=wl.seg_S, M=wl.seg_M, R=wl.seg_R, retr_block=wl.retr_block, is_long=list(inp["is_long"]),
              rope_theta=wl.rope_theta)
    Od, ld, pd = sa.segment_fwd(q, k, v, **kw)
    Oh, lh, ph = sa.segment_fwd(q.cpu(), k.cpu(), v.cpu(), **kw)
    assert torch.equal(Oh, Od.cpu()) and torch.equal(lh, ld.cpu()) and torch.equal(ph, pd.cpu())


# ---------------------------------------------------------------------------
# full-size workloads on sampled rows
# ---------------------------------------------------------------------------

def test_c2_full_size_sampled(oracle_mod):
    wl = synth.WORKLOADS["c2_lminf_16k"]
    inp = synth.make_inputs(wl, seed=0)
    O, lse = _run_fwd(wl, inp)
    rows = synth.sample_rows(wl, 48, seed=1)
    _check_fwd_rows(oracle_mod, wl, inp, O, lse, rows)


def test_c3_full_size_sampled(oracle_mod):
    wl = synth.WORKLOADS["c3_sepllm_gqa_8k"]
    inp = synth.make_inputs(wl, seed=0)
    O, lse = _run_fwd(wl, inp)
    rows = synth.sample_rows(wl, 12, seed=2)
    _check_fwd_rows(oracle_mod, wl, inp, O, lse, rows)


def test_c4_topk_full_size_sampled(oracle_mod):
    wl = synth.WORKLOADS["c4_lminf_topk_32k"]
    inp = synth.make_inputs(wl, seed=0)
    q, k = to_dev(inp["q"]), to_dev(inp["k"])
    idx, z = sa.topk_select(q, k, topk=wl.topk, n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain,
                            rope_theta=wl.rope_theta)
    torch.cuda.synchronize()
    _status_ok()
    planted_rows = [(b, h, s + x) for (b, h, j, s) in inp["meta"]["planted"][::16] for x in (0, 31)]
    rows = synth.sample_rows(wl, 6, seed=3, extra=planted_rows)
    p_ext = oracle_mod.params_of(wl.scaled(topk=wl.topk + TOPK_EXT))
    _, _, ref_idx, ref_z, _ = oracle_mod.fwd_rows(p_ext, inp["q"], inp["k"], inp["v"], None, rows)
    gi = gather_rows(idx, rows).astype(np.int64)
    n_exact, n_exempt, bad = topk_agreement(gi, ref_idx, ref_z, wl.topk)
    assert not bad, "rows differ beyond the near-tie rule: %s" % [(tuple(rows[r]), v) for r, v in bad[:10]]
    O, lse = _run_fwd(wl, inp)
    _check_fwd_rows(oracle_mod, wl, inp, O, lse, rows, forced=gi.astype(np.int32))


def test_c5_segmented_full_size(oracle_mod):
    wl = synth.WORKLOADS["c5_segmented_32k"]
    inp = synth.make_inputs(wl, seed=0)
    q, k, v = to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"])
    O, lse, pb = sa.segment_fwd(q, k, v, S=wl.seg_S, M=wl.seg_M, R=wl.seg_R, retr_block=wl.retr_block,
                                is_long=inp["is_long"], rope_theta=wl.rope_theta,
                                rope_pos_scale=wl.rope_pos_scale)
    torch.cuda.synchronize()
    _status_ok()
    p = oracle_mod.params_of(wl)
    ref_pb, kth = oracle_mod.segment_blocks(p, wl.seg_S, wl.seg_R, wl.retr_block, inp["is_long"], inp["q"], inp["k"])
    got_pb = pb.cpu().numpy()
    diff = np.argwhere(np.any(got_pb != ref_pb, axis=-1))
    for (b, h, s) in diff:
        a, c = kth[b, h, s]
        assert abs(a - c) <= 1e-4 * max(abs(a), abs(c)), "prefix blocks differ at (%d,%d,%d) without a tie" % (b, h, s)
    assert len(diff) <= 2
    rows = synth.sample_rows(wl, 24, seed=4)
    Oref, lref, _ = oracle_mod.segment_rows(p, wl.seg_S, wl.seg_M, wl.seg_R, wl.retr_block, inp["is_long"],
                                            inp["q"], inp["k"], inp["v"], rows)
    compare("O", gather_rows(O, rows), Oref, BF16_MAX_ABS, BF16_MEAN_ABS)
    compare("LSE", gather_rows(lse, rows), lref, BF16_MAX_ABS, BF16_MEAN_ABS)


@pytest.mark.parametrize("cfg", [
    dict(T=1024, S=256, M=64, R=128, blk=64, long=(0, 1)),
    dict(T=768, S=256, M=300, R=256, blk=32, long=(1, 1)),
    dict(T=512, S=128, M=0, R=0, blk=16, long=(0, 1)),
    dict(T=1024, S=256, M=64, R=128, blk=64, long=(1, 0), pos_scale=0.25),
])
def test_segmented_small_all_rows(oracle_mod, cfg):
    wl = synth.Workload(name="seg", B=1, Hq=2, Hkv=2, T=cfg["T"], d=128, dtype="bf16", rope_theta=1e4,
                        seg_S=cfg["S"], seg_M=cfg["M"], seg_R=cfg["R"], retr_block=cfg["blk"],
                        long_heads=tuple(h for h in range(2) if cfg["long"][h]),
                        rope_pos_scale=cfg.get("pos_scale", 1.0))
    inp = synth.make_inputs(wl, seed=12)
    q, k, v = to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"])
    O, lse, pb = sa.segment_fwd(q, k, v, S=wl.seg_S, M=wl.seg_M, R=wl.seg_R, retr_block=wl.retr_block,
                                is_long=inp["is_long"], rope_theta=wl.rope_theta,
                                rope_pos_scale=wl.rope_pos_scale)
    torch.cuda.synchronize()
    _status_ok()
    p = oracle_mod.params_of(wl)
    if wl.seg_R > 0:
        ref_pb, _ = oracle_mod.segment_blocks(p, wl.seg_S, wl.seg_R, wl.retr_block, inp["is_long"], inp["q"], inp["k"])
        assert np.array_equal(pb.cpu().numpy(), ref_pb)
    rows = oracle_mod.all_rows(1, 2, wl.T)
    Oref, lref, _ = oracle_mod.segment_rows(p, wl.seg_S, wl.seg_M, wl.seg_R, wl.retr_block, inp["is_long"],
                                            inp["q"], inp["k"], inp["v"], rows)
    compare("O", gather_rows(O, rows), Oref, BF16_MAX_ABS, BF16_MEAN_ABS)
    compare("LSE", gather_rows(lse, rows), lref, BF16_MAX_ABS, BF16_MEAN_ABS)
