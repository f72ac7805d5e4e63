"""Pins of the oracle's segmented-execution backward
(`oracle_segment_bwd`), against things other than itself:

* central finite differences of the loss sum(dO * O), with O from the
  pinned segmented forward (`oracle_segment_rows`); the retrieval selection
  is a constant of the backward pass, so elements whose perturbation would
  change the selected blocks are not differenced (with R covering the whole
  history, none does);
* one segment (S = T): segmented execution is plain causal attention, whose
  backward is the pinned structured backward with a full causal mask;
* each row's weights sum to one, so every kv head's sum of dV over keys is
  its group's sum of dO over rows.
"""
import numpy as np
import pytest

EPS = 2.0 ** -10


def _grid(shape, g):
    return (g.integers(-512, 512, shape) / 256.0).astype(np.float32)


def _inputs(B, Hq, Hkv, T, d, seed):
    g = np.random.default_rng(seed)
    return _grid((B, Hq, T, d), g), _grid((B, Hkv, T, d), g), _grid((B, Hkv, T, d), g), _grid((B, Hq, T, d), g)


def _loss(O, p, seg, q, k, v, dO):
    S, M, R, blk, il = seg
    rows = O.all_rows(p.B, p.Hq, p.T)
    out, _, _ = O.segment_rows(p, S, M, R, blk, il, q, k, v, rows, nthreads=1)
    return float(np.sum(out.reshape(dO.shape) * dO.astype(np.float64)))


def _fd(O, p, seg, q, k, v, dO, tol=2e-6):
    S, M, R, blk, il = seg
    grads = O.segment_bwd(p, S, M, R, blk, il, q, k, v, dO, nthreads=2)
    base_blocks = O.segment_blocks(p, S, R, blk, il, q, k)[0]
    checked = 0
    for name, x, gr in (("q", q, grads[0]), ("k", k, grads[1]), ("v", v, grads[2])):
        num = np.full_like(gr, np.nan)
        for idx in np.ndindex(*x.shape):
            x0 = x[idx]
            vals = []
            stable = True
            for sgn in (1.0, -1.0):
                x[idx] = x0 + sgn * EPS
                if name != "v" and not np.array_equal(O.segment_blocks(p, S, R, blk, il, q, k)[0], base_blocks):
                    stable = False
                vals.append(_loss(O, p, seg, q, k, v, dO))
            x[idx] = x0
            if stable:
                num[idx] = (vals[0] - vals[1]) / (2 * EPS)
        ok = ~np.isnan(num)
        checked += int(ok.sum())
        scale = max(1.0, np.abs(num[ok]).max())
        err = np.abs(num[ok] - gr[ok]).max() / scale
        assert err < tol, "d%s: max rel err %.3g" % (name, err)
        assert np.abs(gr).max() > 1e-3, "d%s is trivially zero" % name
    return checked


def test_fd_whole_history_retrieved(oracle_mod):
    """Three segments; head 0 long (R covers every earlier block, so the
    selection cannot change), head 1 local with a tail of M = 2; rotary
    positions re-based on the prefix."""
    O = oracle_mod
    B, Hq, Hkv, T, d = 1, 2, 1, 12, 8
    q, k, v, dO = _inputs(B, Hq, Hkv, T, d, 3)
    p = O.params(B, Hq, Hkv, T, d, "f32", rope_theta=1e2)
    seg = (4, 2, 8, 4, np.array([1, 0], dtype=np.uint8))
    n = _fd(O, p, seg, q, k, v, dO)
    assert n == q.size + k.size + v.size


def test_fd_partial_retrieval(oracle_mod):
    """Four segments, R = one block of two out of up to six: the selection
    is real; elements whose perturbation flips it are left out."""
    O = oracle_mod
    B, Hq, Hkv, T, d = 1, 2, 2, 16, 8
    q, k, v, dO = _inputs(B, Hq, Hkv, T, d, 5)
    p = O.params(B, Hq, Hkv, T, d, "f32", rope_theta=1e2)
    seg = (4, 1, 2, 2, np.array([1, 1], dtype=np.uint8))
    n = _fd(O, p, seg, q, k, v, dO)
    assert n > 0.9 * (q.size + k.size + v.size)


def test_one_segment_is_causal_attention(oracle_mod):
    O = oracle_mod
    B, Hq, Hkv, T, d = 2, 4, 2, 24, 8
    q, k, v, dO = _inputs(B, Hq, Hkv, T, d, 7)
    p = O.params(B, Hq, Hkv, T, d, "f32", rope_theta=1e2)
    got = O.segment_bwd(p, T, 3, 4, 2, np.array([1, 0, 1, 0], dtype=np.uint8), q, k, v, dO, nthreads=2)
    pc = O.params(B, Hq, Hkv, T, d, "f32", n_start=0, window=T, rope_theta=1e2)
    ref = O.bwd(pc, q, k, v, None, dO, nthreads=2)
    for a, r in zip(got, ref):
        assert np.abs(a - r).max() < 1e-11


def test_dv_sums_to_do(oracle_mod):
    O = oracle_mod
    B, Hq, Hkv, T, d = 2, 4, 2, 32, 8
    q, k, v, dO = _inputs(B, Hq, Hkv, T, d, 9)
    p = O.params(B, Hq, Hkv, T, d, "f32", rope_theta=1e3)
    dQ, dK, dV = O.segment_bwd(p, 8, 3, 4, 2, np.array([1, 0, 0, 1], dtype=np.uint8), q, k, v, dO, nthreads=2)
    rep = Hq // Hkv
    dO_group = dO.astype(np.float64).reshape(B, Hkv, rep, T, d).sum(axis=(2, 3))
    assert np.abs(dV.sum(axis=2) - dO_group).max() < 1e-10
    z = O.segment_bwd(p, 8, 3, 4, 2, np.array([1, 0, 0, 1], dtype=np.uint8), q, k, v, np.zeros_like(dO))
    assert all(np.all(a == 0) for a in z)
