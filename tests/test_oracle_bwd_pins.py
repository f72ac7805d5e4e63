"""Pins of the oracle's backward pass (gradients of sum(dO * O)).

No GPU.  The backward is checked against things other than itself:
central finite differences of the oracle's forward (pinned on its own in
test_oracle_pins.py) on tiny problems whose inputs and steps are exact in
fp32, torch autograd through fp64 scaled-dot-product attention on the cases
that reduce to it, and exact invariants of the softmax.
"""
import math

import numpy as np
import pytest
import torch

EPS = 2.0 ** -12  # x +- EPS is exact in fp32 for the inputs below


def _grid_inputs(B, Hq, Hkv, T, d, seed):
    """fp32 inputs on a 2^-8 grid in [-2, 2): perturbations by EPS stay exact."""
    g = np.random.default_rng(seed)
    mk = lambda *s: (g.integers(-512, 512, s) / 256.0).astype(np.float32)
    return mk(B, Hq, T, d), mk(B, Hkv, T, d), mk(B, Hkv, T, d), mk(B, Hq, T, d)


def _loss(O, p, q, k, v, sep, dO, forced):
    rows = O.all_rows(p.B, p.Hq, p.T)
    out, *_ = O.fwd_rows(p, q, k, v, sep, rows, forced_topk=forced, nthreads=1)
    return float(np.sum(out.reshape(dO.shape) * dO.astype(np.float64)))


def _fd_check(O, p, q, k, v, sep, dO, forced=None, tol=2e-6):
    dQ, dK, dV = O.bwd(p, q, k, v, sep, dO, forced_topk=forced, nthreads=2)
    for name, x, g in (("q", q, dQ), ("k", k, dK), ("v", v, dV)):
        num = np.zeros_like(g)
        for idx in np.ndindex(*x.shape):
            x0 = x[idx]
            x[idx] = x0 + EPS
            lp = _loss(O, p, q, k, v, sep, dO, forced)
            x[idx] = x0 - EPS
            lm = _loss(O, p, q, k, v, sep, dO, forced)
            x[idx] = x0
            num[idx] = (lp - lm) / (2 * EPS)
        scale = max(1.0, np.abs(num).max())
        err = np.abs(num - g).max() / scale
        assert err < tol, "d%s: max rel err %.3g" % (name, err)
        assert np.abs(g).max() > 1e-3, "d%s is trivially zero" % name


def _forced_of(O, p, q, k, v, sep):
    rows = O.all_rows(p.B, p.Hq, p.T)
    _, _, tki, _, _ = O.fwd_rows(p, q, k, v, sep, rows, nthreads=1)
    return tki.reshape(p.B, p.Hq, p.T, p.topk).copy()


def test_fd_lambda_capped_rope_gqa(oracle_mod):
    """Sinks, window, capped rotary logits (i - j > L) and GQA."""
    O = oracle_mod
    B, Hq, Hkv, T, d = 1, 2, 1, 11, 8
    q, k, v, dO = _grid_inputs(B, Hq, Hkv, T, d, 1)
    p = O.params(B, Hq, Hkv, T, d, "f32", 2, 3, 3, 0, 1e2)
    _fd_check(O, p, q, k, v, None, dO)


def test_fd_separators_topk_position_scale(oracle_mod):
    """Separators, forced top-k sets, position interpolation, cap above the window."""
    O = oracle_mod
    B, Hq, Hkv, T, d = 1, 2, 2, 12, 8
    q, k, v, dO = _grid_inputs(B, Hq, Hkv, T, d, 2)
    sep = np.zeros((B, T), dtype=np.uint8)
    sep[0, [3, 6]] = 1
    p = O.params(B, Hq, Hkv, T, d, "f32", 1, 2, 4, 2, 1e2, 0.5)
    forced = _forced_of(O, p, q, k, v, sep)
    assert (forced >= 0).any()
    _fd_check(O, p, q, k, v, sep, dO, forced)


def test_fd_alibi_clipped(oracle_mod):
    O = oracle_mod
    B, H, T, d = 1, 2, 10, 8
    q, k, v, dO = _grid_inputs(B, H, H, T, d, 3)
    p = O.params(B, H, H, T, d, "f32", 2, 3, 3, 0, 0.0, alibi=True)
    _fd_check(O, p, q, k, v, None, dO)


def _sdpa_grads(q, k, v, dO, mask):
    rep = q.shape[1] // k.shape[1]
    qt = torch.tensor(q, dtype=torch.float64, requires_grad=True)
    kt = torch.tensor(k, dtype=torch.float64, requires_grad=True)
    vt = torch.tensor(v, dtype=torch.float64, requires_grad=True)
    out = torch.nn.functional.scaled_dot_product_attention(
        qt, kt.repeat_interleave(rep, dim=1), vt.repeat_interleave(rep, dim=1), attn_mask=torch.from_numpy(mask))
    (out * torch.tensor(dO, dtype=torch.float64)).sum().backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("ns,w", [(0, 100), (0, 5), (3, 4), (20, 3)])
def test_autograd_sdpa_masks(oracle_mod, ns, w):
    """No rotation and no cap: the oracle's gradients equal torch autograd
    through fp64 SDPA with the Lambda mask (full causal, sliding window,
    sinks + window), GQA by head repetition."""
    O = oracle_mod
    B, Hq, Hkv, T, d = 2, 4, 2, 33, 16
    q, k, v, dO = _grid_inputs(B, Hq, Hkv, T, d, 4)
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    mask = (j <= i) & ((j < ns) | (i - j <= w))
    p = O.params(B, Hq, Hkv, T, d, "f32", ns, w, 0, 0, 0.0)
    got = O.bwd(p, q, k, v, None, dO, nthreads=2)
    ref = _sdpa_grads(q, k, v, dO, mask)
    for g, r in zip(got, ref):
        assert np.abs(g - r).max() < 1e-11


def test_autograd_sdpa_separators_bf16(oracle_mod):
    """bf16-encoded inputs and dO, SepLLM mask from the oracle's own mask rows."""
    O = oracle_mod
    B, H, T, d = 1, 2, 40, 16
    g = torch.Generator().manual_seed(5)
    mk = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)
    q, k, v, dO = mk(B, H, T, d), mk(B, H, T, d), mk(B, H, T, d), mk(B, H, T, d)
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    rng = np.random.default_rng(6)
    sep = (rng.random((B, T)) < 0.2).astype(np.uint8)
    ns, w = 2, 4
    p = O.params(B, H, H, T, d, "bf16", ns, w, 0, 0, 0.0)
    got = O.bwd(p, bits(q), bits(k), bits(v), sep, bits(dO), nthreads=2)
    mask = np.stack([O.mask_row(T, i, ns, w, sep[0])[0] for i in range(T)]).astype(bool)
    ref = _sdpa_grads(*(t.double().numpy() for t in (q, k, v, dO)), mask)
    for a, r in zip(got, ref):
        assert np.abs(a - r).max() < 1e-11


def test_invariants(oracle_mod):
    """sum_j dV_j = sum_i dO_i over a kv head's group (each row's weights sum
    to one); without a rotation a common shift of every key leaves every
    row's weights unchanged, so sum_j dK_j = 0; dO = 0 gives zero gradients."""
    O = oracle_mod
    B, Hq, Hkv, T, d = 2, 4, 2, 30, 8
    q, k, v, dO = _grid_inputs(B, Hq, Hkv, T, d, 7)
    rng = np.random.default_rng(8)
    sep = (rng.random((B, T)) < 0.3).astype(np.uint8)
    p = O.params(B, Hq, Hkv, T, d, "f32", 2, 4, 6, 3, 0.0, alibi=True)
    dQ, dK, dV = O.bwd(p, q, k, v, sep, dO, nthreads=2)
    rep = Hq // Hkv
    dO_group = dO.astype(np.float64).reshape(B, Hkv, rep, T, d).sum(axis=(2, 3))
    assert np.abs(dV.sum(axis=2) - dO_group).max() < 1e-10
    assert np.abs(dK.sum(axis=2)).max() < 1e-10
    z = O.bwd(p, q, k, v, sep, np.zeros_like(dO), nthreads=2)
    assert all(np.all(a == 0) for a in z)
    # with a rotation the shift invariance is gone
    p2 = O.params(B, Hq, Hkv, T, d, "f32", 2, 4, 6, 3, 1e2)
    _, dK2, _ = O.bwd(p2, q, k, v, sep, dO, nthreads=2)
    assert np.abs(dK2.sum(axis=2)).max() > 1e-3


@pytest.mark.parametrize("cfg", [
    dict(dtype="f32", n_start=2, window=4, L_pretrain=6, topk=3, rope_theta=1e2),   # capped, separators, top-k
    dict(dtype="f32", n_start=1, window=5, L_pretrain=5, topk=0, alibi=True),       # clipped ALiBi
    dict(dtype="f32", n_start=0, window=100, L_pretrain=0, topk=0, rope_theta=0.0),  # full causal
])
def test_dq_rows_entry_equals_full_backward(oracle_mod, cfg):
    """oracle_bwd_dq_rows (the rows-only entry used at full sizes) runs the
    same row arithmetic as the pinned full backward: equal bits."""
    O = oracle_mod
    B, Hq, Hkv, T, d = 2, 4, 2, 40, 8
    q, k, v, dO = _grid_inputs(B, Hq, Hkv, T, d, 11)
    rng = np.random.default_rng(12)
    sep = (rng.random((B, T)) < 0.3).astype(np.uint8)
    p = O.params(B, Hq, Hkv, T, d, **cfg)
    forced = _forced_of(O, p, q, k, v, sep) if p.topk else None
    dQ, _, _ = O.bwd(p, q, k, v, sep, dO, forced_topk=forced, nthreads=2)
    rows = np.array([(b, h, i) for b in range(B) for h in range(Hq) for i in (0, 1, 7, 20, T - 1)])
    dq = O.bwd_dq_rows(p, q, k, v, sep, dO, rows, forced_topk=forced, nthreads=2)
    assert np.array_equal(dq, dQ[rows[:, 0], rows[:, 1], rows[:, 2]])
    with pytest.raises(RuntimeError):
        O.bwd_dq_rows(p, q, k, v, sep, dO, np.array([(0, 0, T)]))


@pytest.mark.parametrize("cfg", [
    dict(dtype="f32", n_start=2, window=4, L_pretrain=6, topk=3, rope_theta=1e2),   # capped, separators, top-k
    dict(dtype="f32", n_start=1, window=5, L_pretrain=5, topk=0, alibi=True),       # clipped ALiBi
    dict(dtype="f32", n_start=3, window=3, L_pretrain=3, topk=0, rope_theta=1e2, rope_pos_scale=0.5),
])
def test_dkv_keys_entry_equals_full_backward(oracle_mod, cfg):
    """oracle_bwd_dkv_keys (the keys-only entry used at full sizes) takes the
    same key-side sums as the pinned full backward, in the same order: equal
    bits for sinks, separators, window and top-k keys, every kv head."""
    O = oracle_mod
    B, Hq, Hkv, T, d = 2, 4, 2, 40, 8
    q, k, v, dO = _grid_inputs(B, Hq, Hkv, T, d, 13)
    rng = np.random.default_rng(14)
    sep = (rng.random((B, T)) < 0.3).astype(np.uint8)
    p = O.params(B, Hq, Hkv, T, d, **cfg)
    forced = _forced_of(O, p, q, k, v, sep) if p.topk else None
    _, dK, dV = O.bwd(p, q, k, v, sep, dO, forced_topk=forced, nthreads=2)
    keys = np.array([(b, g, j) for b in range(B) for g in range(Hkv) for j in (0, 1, 2, 5, 9, 17, 30, T - 1)])
    dk, dv = O.bwd_dkv_keys(p, q, k, v, sep, dO, keys, forced_topk=forced, nthreads=2)
    assert np.array_equal(dk, dK[keys[:, 0], keys[:, 1], keys[:, 2]])
    assert np.array_equal(dv, dV[keys[:, 0], keys[:, 1], keys[:, 2]])
    assert np.abs(dk).max() > 1e-3 and np.abs(dv).max() > 1e-3
    with pytest.raises(RuntimeError):
        O.bwd_dkv_keys(p, q, k, v, sep, dO, np.array([(0, Hkv, 0)]))
