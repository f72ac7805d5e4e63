"""GPU parity of the backward pass against the oracle's fp64 gradients.

The forward runs on the GPU first (its O and LSE are inputs of the backward,
as in training); the top-k sets are the GPU selection, handed to the oracle
as forced sets.  Gradients are compared element by element with a bar
relative to the gradient's largest magnitude (sums over many rows make dK and
dV grow with the number of rows that keep a key): fp32 1e-4.
"""
import numpy as np
import pytest
import torch

import long_context_structured_b200 as sa
from long_context_structured_b200 import _lib, synth
from _util import to_dev

pytestmark = pytest.mark.gpu

F32_GRAD_REL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def compare_grad(name, got, ref, rel, mean_rel=None):
    scale = max(1.0, float(np.abs(ref).max()))
    err = np.abs(got - ref)
    mx, mn = float(err.max()) / scale, float(err.mean()) / scale
    msg = "%s: max-abs/scale %.3e (bar %.1e), mean-abs/scale %.3e, scale %.3g" % (name, mx, rel, mn, scale)
    print(msg)
    assert np.isfinite(got).all() and mx <= rel and (mean_rel is None or mn <= mean_rel), msg


def _kw(wl):
    return dict(n_start=wl.n_start, window=wl.window, L_pretrain=wl.L_pretrain, rope_theta=wl.rope_theta,
                rope_pos_scale=wl.rope_pos_scale, alibi=wl.alibi)


def _run(oracle_mod, wl, seed, rel, mean_rel=None):
    inp = synth.make_inputs(wl, seed=seed)
    q, k, v = (to_dev(inp[x]) for x in ("q", "k", "v"))
    sep = to_dev(inp["is_sep"])
    g = np.random.default_rng(seed + 100)
    if wl.dtype == "f32":
        dO_h = g.standard_normal(inp["q"].shape).astype(np.float32)
    else:
        dO_h = (g.standard_normal(inp["q"].shape).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    dO = to_dev(dO_h)
    idx = None
    if wl.topk > 0:
        idx, z = sa.topk_select(q, k, topk=wl.topk, is_sep=sep, **_kw(wl))
        O, lse = sa.fwd(q, k, v, topk=wl.topk, is_sep=sep, topk_idx=idx, topk_logit=z, **_kw(wl))
    else:
        O, lse = sa.fwd(q, k, v, is_sep=sep, **_kw(wl))
    dq, dk, dv = sa.bwd(q, k, v, O, lse, dO, topk=wl.topk, is_sep=sep, topk_idx=idx, **_kw(wl))
    torch.cuda.synchronize()
    assert sa.stream_status() == 0
    forced = None if idx is None else idx.cpu().numpy()
    ref = oracle_mod.bwd(oracle_mod.params_of(wl), inp["q"], inp["k"], inp["v"], inp["is_sep"], dO_h,
                         forced_topk=forced)
    for name, t, r in (("dQ", dq, ref[0]), ("dK", dk, ref[1]), ("dV", dv, ref[2])):
        compare_grad(name, t.float().cpu().numpy().astype(np.float64), r, rel, mean_rel)
    return (dq, dk, dv), (q, k, v, O, lse, dO, sep, idx)


F32_CASES = [
    ("lambda_capped_gqa", dict(B=1, Hq=4, Hkv=2, T=300, d=128, n_start=4, window=40, L_pretrain=40,
                               rope_theta=1e4, sink_scale=8.0)),
    ("sep_topk_cap_above_window_pi", dict(B=2, Hq=2, Hkv=1, T=257, d=64, n_start=2, window=20, L_pretrain=40,
                                          rope_theta=1e4, topk=3, sep_rate=0.1, rope_pos_scale=0.5)),
    ("alibi_sep", dict(B=1, Hq=4, Hkv=4, T=200, d=128, n_start=3, window=30, L_pretrain=30, sep_rate=0.15,
                       alibi=True)),
    ("causal_no_rope", dict(B=1, Hq=2, Hkv=2, T=150, d=64, n_start=0, window=1000)),
    ("tiny", dict(B=1, Hq=1, Hkv=1, T=3, d=64, n_start=4, window=1, rope_theta=1e4)),
]


@pytest.mark.parametrize("name,cfg", F32_CASES, ids=[c[0] for c in F32_CASES])
def test_bwd_f32(oracle_mod, name, cfg):
    wl = synth.Workload(name=name, dtype="f32", **cfg)
    _run(oracle_mod, wl, 21, F32_GRAD_REL)


def test_bwd_f32_sinks40(oracle_mod):
    wl = synth.Workload(name="f32_sinks40", B=1, Hq=2, Hkv=1, T=300, d=64, dtype="f32", n_start=40, window=20,
                        L_pretrain=20, rope_theta=1e4, sep_rate=0.1, sink_scale=8.0)
    _run(oracle_mod, wl, 22, F32_GRAD_REL)


def test_bwd_f32_sepllm_config(oracle_mod):
    """The fp32 SepLLM-mask layer (T=1024, d=64, separators at rate 0.08)."""
    _run(oracle_mod, synth.WORKLOADS["c1_f32_sep"], 0, F32_GRAD_REL)


def test_bwd_f32_deterministic(oracle_mod):
    wl = synth.Workload(name="det", B=1, Hq=2, Hkv=1, T=300, d=128, dtype="f32", n_start=4, window=30,
                        L_pretrain=30, rope_theta=1e4, sep_rate=0.1)
    grads, (q, k, v, O, lse, dO, sep, idx) = _run(oracle_mod, wl, 5, F32_GRAD_REL)
    again = sa.bwd(q, k, v, O, lse, dO, is_sep=sep, **_kw(wl))
    assert all(torch.equal(a, b) for a, b in zip(grads, again))


BF16_GRAD_REL, BF16_GRAD_MEAN_REL = 2e-2, 2e-3

BF16_CASES = [
    ("causal_no_rope", dict(B=1, Hq=2, Hkv=2, T=300, d=128, n_start=0, window=1000)),
    ("lambda_capped_sinks_gqa", dict(B=1, Hq=4, Hkv=2, T=700, d=128, n_start=4, window=100, L_pretrain=100,
                                     rope_theta=1e4, sink_scale=8.0)),
    ("sep_uncapped_d64", dict(B=2, Hq=4, Hkv=2, T=600, d=64, n_start=1, window=37, rope_theta=1e4, sep_rate=0.1)),
    ("sep_capped", dict(B=1, Hq=2, Hkv=2, T=513, d=128, n_start=4, window=64, L_pretrain=64, rope_theta=1e4,
                        sep_rate=0.3)),
    ("alibi_sep_capped", dict(B=1, Hq=4, Hkv=1, T=400, d=128, n_start=4, window=64, L_pretrain=64, sep_rate=0.2,
                              alibi=True)),
    ("pos_interp_gqa", dict(B=1, Hq=2, Hkv=1, T=500, d=128, n_start=4, window=64, L_pretrain=64, rope_theta=1e4,
                            rope_pos_scale=0.5)),
    ("window0_all_seps", dict(B=1, Hq=2, Hkv=2, T=257, d=128, n_start=1, window=0, sep_rate=1.0)),
    ("tiny", dict(B=1, Hq=1, Hkv=1, T=5, d=128, n_start=4, window=2, rope_theta=1e4)),
    # sink spans wider than 16: the sink keys staged in several passes
    ("sinks12_capped_gqa", dict(B=1, Hq=4, Hkv=2, T=600, d=128, n_start=12, window=64, L_pretrain=64,
                                rope_theta=1e4, sink_scale=8.0)),
    ("sinks40_sep_capped", dict(B=1, Hq=2, Hkv=2, T=700, d=128, n_start=40, window=64, L_pretrain=64,
                                rope_theta=1e4, sep_rate=0.1, sink_scale=8.0)),
    ("sinks40_d64_uncapped", dict(B=1, Hq=2, Hkv=1, T=500, d=64, n_start=40, window=30, rope_theta=5e5,
                                  sep_rate=0.1)),
    # separators with the window below the cap: the uncapped ones (w < i - j
    # <= L) in the band tiles, the capped ones in the compacted tiles
    ("sep_window_below_cap", dict(B=1, Hq=2, Hkv=2, T=700, d=128, n_start=4, window=50, L_pretrain=130,
                                  rope_theta=1e4, sep_rate=0.15)),
    ("sep_window_below_cap_d64_gqa", dict(B=2, Hq=4, Hkv=2, T=600, d=64, n_start=2, window=30, L_pretrain=200,
                                          rope_theta=5e5, sep_rate=0.2)),
    ("alibi_sep_window_below_cap", dict(B=1, Hq=4, Hkv=1, T=500, d=128, n_start=4, window=40, L_pretrain=150,
                                        sep_rate=0.2, alibi=True)),
    # top-k middle keys (fp32 side keys, the selection a constant): capped
    # (L = w), with separators, uncapped (L = 0), and with the clipped ALiBi bias
    ("topk_capped_sinks_gqa", dict(B=1, Hq=4, Hkv=2, T=700, d=128, n_start=4, window=64, L_pretrain=64,
                                   rope_theta=1e4, topk=4, sink_scale=8.0)),
    ("topk_sep_d64", dict(B=2, Hq=2, Hkv=1, T=600, d=64, n_start=2, window=50, L_pretrain=50, rope_theta=1e4,
                          topk=3, sep_rate=0.1)),
    ("topk_uncapped_k8", dict(B=1, Hq=2, Hkv=2, T=500, d=128, n_start=4, window=40, rope_theta=1e4, topk=8)),
    ("topk_alibi", dict(B=1, Hq=4, Hkv=1, T=400, d=128, n_start=4, window=64, L_pretrain=64, topk=3,
                        alibi=True)),
    ("topk_window_below_cap_sep", dict(B=1, Hq=2, Hkv=2, T=700, d=128, n_start=4, window=50, L_pretrain=130,
                                       rope_theta=1e4, topk=4, sep_rate=0.1)),
    ("topk16_sinks20_sep", dict(B=1, Hq=2, Hkv=2, T=640, d=128, n_start=20, window=48, L_pretrain=48,
                                rope_theta=1e4, topk=16, sep_rate=0.05)),
]


@pytest.mark.parametrize("name,cfg", BF16_CASES, ids=[c[0] for c in BF16_CASES])
def test_bwd_bf16(oracle_mod, name, cfg):
    wl = synth.Workload(name=name, dtype="bf16", **cfg)
    _run(oracle_mod, wl, 31, BF16_GRAD_REL, BF16_GRAD_MEAN_REL)


@pytest.mark.parametrize("topk", [0, 5])
def test_bwd_bf16_deterministic(oracle_mod, topk):
    wl = synth.Workload(name="det16", B=1, Hq=4, Hkv=2, T=600, d=128, dtype="bf16", n_start=4, window=64,
                        L_pretrain=64, rope_theta=1e4, sep_rate=0.1, topk=topk)
    grads, (q, k, v, O, lse, dO, sep, idx) = _run(oracle_mod, wl, 8, BF16_GRAD_REL, BF16_GRAD_MEAN_REL)
    for _ in range(2):
        again = sa.bwd(q, k, v, O, lse, dO, is_sep=sep, topk=wl.topk, topk_idx=idx, **_kw(wl))
        torch.cuda.synchronize()
        assert all(torch.equal(a, b) for a, b in zip(grads, again))


def test_bwd_rejects_missing_topk_selection():
    q = torch.zeros((1, 1, 64, 64), dtype=torch.float32, device="cuda")
    lse = torch.zeros((1, 1, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(_lib.SattnError):
        sa.bwd(q, q, q, q, lse, q, window=4, L_pretrain=4, topk=2)


def _sample_keys(wl, flags, rng):
    """Keys (b, kv head, j) of every kind the layer has: a sink, the first
    non-sink key, tile and window edges, the last key, separators early and
    late, and random keys."""
    keys = []
    js = [0, wl.n_start, 127, 128, wl.window, wl.window + 1, wl.T // 2, wl.T - 129, wl.T - 1]
    js += [int(x) for x in rng.integers(wl.n_start, wl.T, 6)]
    for x, j in enumerate(js):
        keys.append((x % wl.B, x % wl.Hkv, j))
    if flags is not None:
        for b in sorted({0, wl.B - 1}):
            sp = np.flatnonzero(flags[b][wl.n_start:]) + wl.n_start
            for x, j in enumerate((sp[0], sp[len(sp) // 2], sp[-1])):
                keys.append((b, (x + b) % wl.Hkv, int(j)))
    keys.append((wl.B - 1, wl.Hkv - 1, int(rng.integers(wl.n_start, wl.T))))
    return np.array(keys, dtype=np.int64)


@pytest.mark.parametrize("name", ["c2_lminf_16k", "c3_sepllm_gqa_8k"])
def test_bwd_full_size_sampled(oracle_mod, name):
    """The backward at the benchmark's full sizes (the launch the backward
    workloads time), element by element on samples: dQ of sampled rows
    against the oracle's rows entry, dK and dV of sampled keys (sinks,
    separators, window and tile edges) against its keys entry -- each the
    same arithmetic as the full oracle backward, pinned equal to it bit for
    bit.  Bars relative to each group's largest gradient (sink keys, whose
    sums run over every row, separately).  Plus, for every kv head, the sum
    of dV over keys against its group's sum of dO over rows (every row's
    weights sum to one), within 2^-7 of sum |dV|."""
    wl = synth.WORKLOADS[name]
    inp = synth.make_inputs(wl, seed=0)
    q, k, v = (to_dev(inp[x]) for x in ("q", "k", "v"))
    sep = to_dev(inp["is_sep"])
    g = np.random.default_rng(7)
    dO_h = (g.standard_normal(inp["q"].shape).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    dO = to_dev(dO_h)
    O, lse = sa.fwd(q, k, v, is_sep=sep, **_kw(wl))
    dq, dk, dv = sa.bwd(q, k, v, O, lse, dO, is_sep=sep, **_kw(wl))
    torch.cuda.synchronize()
    assert sa.stream_status() == 0
    p = oracle_mod.params_of(wl)
    rng = np.random.default_rng(1)
    n = 48
    rows = np.stack([rng.integers(0, wl.B, n), rng.integers(0, wl.Hq, n), rng.integers(0, wl.T, n)], axis=1)
    rows[:4, 2] = [0, 1, wl.T // 2, wl.T - 1]
    ref = oracle_mod.bwd_dq_rows(p, inp["q"], inp["k"], inp["v"], inp["is_sep"], dO_h, rows)
    ri = torch.as_tensor(rows, device=dq.device)
    got = dq[ri[:, 0], ri[:, 1], ri[:, 2]].float().cpu().numpy().astype(np.float64)
    compare_grad("dQ rows", got, ref, BF16_GRAD_REL, BF16_GRAD_MEAN_REL)
    keys = _sample_keys(wl, inp["is_sep"], np.random.default_rng(2))
    rdk, rdv = oracle_mod.bwd_dkv_keys(p, inp["q"], inp["k"], inp["v"], inp["is_sep"], dO_h, keys)
    ki = torch.as_tensor(keys, device=dk.device)
    gdk = dk[ki[:, 0], ki[:, 1], ki[:, 2]].float().cpu().numpy().astype(np.float64)
    gdv = dv[ki[:, 0], ki[:, 1], ki[:, 2]].float().cpu().numpy().astype(np.float64)
    sink = keys[:, 2] < wl.n_start
    for part, sel in (("sink keys", sink), ("other keys", ~sink)):
        if sel.any():
            compare_grad("dK " + part, gdk[sel], rdk[sel], BF16_GRAD_REL, BF16_GRAD_MEAN_REL)
            compare_grad("dV " + part, gdv[sel], rdv[sel], BF16_GRAD_REL, BF16_GRAD_MEAN_REL)
    rep = wl.Hq // wl.Hkv
    dv64 = dv.double()
    lhs = dv64.sum(dim=2)
    rhs = dO.double().reshape(wl.B, wl.Hkv, rep, wl.T, wl.d).sum(dim=(2, 3))
    bound = dv64.abs().sum(dim=2) * 2.0 ** -7 + 1e-6
    excess = ((lhs - rhs).abs() - bound).max().item()
    print("dV sum: max |lhs - rhs| %.3g, bound %.3g" % ((lhs - rhs).abs().max().item(), bound.min().item()))
    assert excess <= 0.0
