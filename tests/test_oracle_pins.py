"""Pins of the fp64 oracle against what the pages and the mathematics fix.

No GPU.  Every check compares the oracle with something other than itself:
hand-written golden masks, closed forms, torch's scaled-dot-product
attention on the degenerate cases the pages name, numpy routines, and brute
force on tiny inputs.
"""
import math
import os

import numpy as np
import pytest
import torch

from long_context_structured_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f64(bits_or_f32):
    a = np.asarray(bits_or_f32)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def _rand_inputs(B, Hq, Hkv, T, d, seed, dtype="bf16"):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, T, d, generator=g)
    k = torch.randn(B, Hkv, T, d, generator=g)
    v = torch.randn(B, Hkv, T, d, generator=g)
    if dtype == "bf16":
        cv = lambda x: x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        return cv(q), cv(k), cv(v)
    return q.numpy(), k.numpy(), v.numpy()


def _sdpa(q64, k64, v64, mask_bool):
    """torch SDPA in fp64; mask_bool [T, T] True = attend.  GQA by repeat."""
    rep = q64.shape[1] // k64.shape[1]
    q = torch.from_numpy(q64)
    k = torch.from_numpy(np.repeat(k64, rep, axis=1))
    v = torch.from_numpy(np.repeat(v64, rep, axis=1))
    m = torch.from_numpy(mask_bool)
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m).numpy()


def _lse_ref(q64, k64, mask_bool):
    rep = q64.shape[1] // k64.shape[1]
    k = np.repeat(k64, rep, axis=1)
    s = np.einsum("bhid,bhjd->bhij", q64, k) / math.sqrt(q64.shape[-1])
    s = np.where(mask_bool[None, None], s, -np.inf)
    mx = s.max(-1, keepdims=True)
    return (mx + np.log(np.exp(s - mx).sum(-1, keepdims=True)))[..., 0]


def _rotate_all(x64, theta, O):
    out = np.empty_like(x64)
    T = x64.shape[2]
    for idx in np.ndindex(*x64.shape[:2]):
        for i in range(T):
            out[idx + (i,)] = O.rope(x64[idx + (i,)], i, theta)
    return out


# ----------------------------------------------------------------------------
# bf16 decoding
# ----------------------------------------------------------------------------

def test_decode_bf16_hand_values(oracle_mod):
    O = oracle_mod
    # values worked out by hand from sign / 8-bit exponent / 7-bit fraction
    cases = {
        0x3F80: 1.0, 0xC000: -2.0, 0x4049: 3.140625, 0x3F00: 0.5,
        0x0001: 2.0 ** -133, 0x0080: 2.0 ** -126, 0x7F7F: (2 - 2 ** -7) * 2.0 ** 127,
        0x8000: -0.0, 0x4180: 16.0, 0xBF40: -0.75,
    }
    for bits, val in cases.items():
        assert O.decode_bf16(bits) == val, hex(bits)
    assert math.isinf(O.decode_bf16(0x7F80)) and O.decode_bf16(0xFF80) < 0
    assert math.isnan(O.decode_bf16(0x7FC0))


def test_decode_bf16_matches_bit_widening(oracle_mod):
    bits = np.arange(0, 65536, 7, dtype=np.uint16)
    ref = _f64(bits)
    got = np.array([oracle_mod.decode_bf16(int(b)) for b in bits])
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])


# ----------------------------------------------------------------------------
# rotary rotation and the capped logit
# ----------------------------------------------------------------------------

def test_rope_quarter_turn_and_frequencies(oracle_mod):
    O = oracle_mod
    # d = 2: one pair, inverse frequency theta^0 = 1; a quarter turn maps
    # (1, 0) to (0, 1) (counter-clockwise, first half gets x cos - y sin)
    r = O.rope(np.array([1.0, 0.0]), math.pi / 2, 10000.0)
    assert abs(r[0]) < 1e-15 and abs(r[1] - 1.0) < 1e-15
    # d = 4: the second pair turns with theta^(-1/2); at pos = pi*sqrt(theta)
    # it has turned by pi, the first pair by pos
    theta = 100.0
    pos = math.pi * math.sqrt(theta)
    r = O.rope(np.array([0.0, 1.0, 0.0, 0.0]), pos, theta)
    assert np.allclose(r, [0.0, -1.0, 0.0, 0.0], atol=1e-12)
    # theta == 0 disables rotation
    x = np.arange(8, dtype=np.float64)
    assert np.array_equal(O.rope(x, 12345, 0.0), x)


def test_rope_group_and_norm(oracle_mod):
    O = oracle_mod
    rng = np.random.default_rng(0)
    for d in (2, 64, 128):
        x = rng.standard_normal(d)
        a, b = 37.0, 1201.0
        assert np.allclose(O.rope(O.rope(x, a, 1e4), b, 1e4), O.rope(x, a + b, 1e4), atol=1e-10)
        assert abs(np.linalg.norm(O.rope(x, 999.0, 5e5)) - np.linalg.norm(x)) < 1e-10


def test_rope_relative_position_identity(oracle_mod):
    O = oracle_mod
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    for (i, j) in [(5, 3), (4096, 17), (32767, 31000)]:
        lhs = np.dot(O.rope(q, i, 1e4), O.rope(k, j, 1e4))
        rhs = np.dot(O.rope(q, i - j, 1e4), k)
        assert abs(lhs - rhs) < 1e-9 * max(1.0, abs(lhs))


def test_capped_logit_equals_shifted_distance(oracle_mod):
    """LM-Infinite states the cap two ways: d' = min(d, L) inside the logit
    function, and, for RoPE, 'key unrotated, query rotated to L'.  The oracle
    implements the second; it must equal the first."""
    O = oracle_mod
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    L = 100
    for (i, j) in [(500, 2), (101, 0), (5000, 3)]:
        z = O.logit(q, k, i, j, L, 1e4)
        d_capped = min(i - j, L)
        ref = np.dot(O.rope(q, j + d_capped, 1e4), O.rope(k, j, 1e4))
        assert abs(z - ref) < 1e-9
    # within the cap the logit is the plain rotary one
    for (i, j) in [(100, 0), (50, 49), (7, 7)]:
        z = O.logit(q, k, i, j, L, 1e4)
        assert abs(z - np.dot(O.rope(q, i, 1e4), O.rope(k, j, 1e4))) < 1e-12
    # L >= distance or L = 0: uncapped
    assert O.logit(q, k, 900, 1, 0, 1e4) == pytest.approx(np.dot(O.rope(q, 899, 1e4), k), abs=1e-9)


# ----------------------------------------------------------------------------
# mask rows: hand-written goldens and closed-form sizes
# ----------------------------------------------------------------------------

def _read_golden(name):
    lines = [l.strip() for l in open(os.path.join(GOLDEN, name)) if l.strip() and not l.startswith("#")]
    return lines


def test_lambda_mask_golden(oracle_mod):
    lines = _read_golden("lambda_mask_T8_ns2_w2.txt")
    T, ns, w = map(int, lines[0].split())
    for i, row in enumerate(lines[1:]):
        m, cnt = oracle_mod.mask_row(T, i, ns, w)
        assert "".join(map(str, m)) == row, i
        assert cnt == row.count("1")


def test_sepllm_mask_golden(oracle_mod):
    lines = _read_golden("sepllm_mask_T10_a1_n2.txt")
    T, a, n = map(int, lines[0].split())
    sep = np.zeros(T, dtype=np.uint8)
    sep[list(map(int, lines[1].split()))] = 1
    for i, row in enumerate(lines[2:]):
        m, _ = oracle_mod.mask_row(T, i, a, n, sep)
        assert "".join(map(str, m)) == row, i


def _closed_form_count(i, ns, w, sep, k):
    base = min(i + 1, ns + w + 1)
    mid_sep = int(sum(1 for j in range(ns, max(ns, i - w)) if sep[j]))
    n_mid = max(0, i - w - ns)
    return base + mid_sep + min(k, max(0, n_mid - mid_sep))


def test_mask_sizes_closed_form_bruteforce(oracle_mod):
    """|A_i| = min(i+1, ns+w+1) + #separators in [ns, i-w) for every flag
    pattern of a length-8 sequence and every (ns, w)."""
    T = 8
    for pat in range(1 << T):
        sep = np.array([(pat >> j) & 1 for j in range(T)], dtype=np.uint8)
        for ns in range(0, T + 1, 3):
            for w in range(0, T + 1, 2):
                for i in range(T):
                    _, cnt = oracle_mod.mask_row(T, i, ns, w, sep)
                    assert cnt == _closed_form_count(i, ns, w, sep, 0), (pat, ns, w, i)


def test_attended_counts_with_topk_closed_form(oracle_mod):
    T, d = 40, 8
    q, k, v = _rand_inputs(1, 1, 1, T, d, 3)
    rng = np.random.default_rng(4)
    sep = (rng.random((1, T)) < 0.3).astype(np.uint8)
    for (ns, w, kk) in [(2, 3, 2), (0, 5, 4), (3, 0, 1), (1, 2, 50)]:
        p = oracle_mod.params(1, 1, 1, T, d, "bf16", ns, w, 0, kk, 1e4)
        rows = oracle_mod.all_rows(1, 1, T)
        _, _, _, _, cnt = oracle_mod.fwd_rows(p, q, k, v, sep, rows)
        for i in range(T):
            assert cnt[i] == _closed_form_count(i, ns, w, sep[0], kk), (ns, w, kk, i)


# ----------------------------------------------------------------------------
# forward: degenerate cases against torch SDPA (fp64)
# ----------------------------------------------------------------------------

def _tri(T):
    return np.tril(np.ones((T, T), dtype=bool))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_full_causal_equals_sdpa(oracle_mod, dtype):
    B, Hq, Hkv, T, d = 2, 4, 2, 37, 16
    q, k, v = _rand_inputs(B, Hq, Hkv, T, d, 5, dtype)
    p = oracle_mod.params(B, Hq, Hkv, T, d, dtype, 0, T + 3, 0, 0, 0.0)
    O, lse, *_ = oracle_mod.fwd_rows(p, q, k, v, None, oracle_mod.all_rows(B, Hq, T))
    ref = _sdpa(_f64(q), _f64(k), _f64(v), _tri(T))
    assert np.abs(O.reshape(ref.shape) - ref).max() < 1e-12
    lref = _lse_ref(_f64(q), _f64(k), _tri(T))
    assert np.abs(lse.reshape(lref.shape) - lref).max() < 1e-12


def test_full_causal_with_rope_equals_sdpa(oracle_mod):
    B, H, T, d = 1, 2, 29, 8
    q, k, v = _rand_inputs(B, H, H, T, d, 6)
    theta = 10000.0
    p = oracle_mod.params(B, H, H, T, d, "bf16", 0, T, 0, 0, theta)
    O, *_ = oracle_mod.fwd_rows(p, q, k, v, None, oracle_mod.all_rows(B, H, T))
    qr = _rotate_all(_f64(q), theta, oracle_mod)
    kr = _rotate_all(_f64(k), theta, oracle_mod)
    ref = _sdpa(qr, kr, _f64(v), _tri(T))
    assert np.abs(O.reshape(ref.shape) - ref).max() < 1e-12


def test_sliding_window_equals_sdpa(oracle_mod):
    """n_start = 0 and no separators: pure recent-window attention (the
    degenerate case LM-Infinite names)."""
    B, H, T, d, w = 1, 3, 50, 8, 6
    q, k, v = _rand_inputs(B, H, H, T, d, 7)
    p = oracle_mod.params(B, H, H, T, d, "bf16", 0, w, 0, 0, 0.0)
    O, *_ = oracle_mod.fwd_rows(p, q, k, v, None, oracle_mod.all_rows(B, H, T))
    band = _tri(T) & ~np.tril(np.ones((T, T), dtype=bool), k=-(w + 1))
    ref = _sdpa(_f64(q), _f64(k), _f64(v), band)
    assert np.abs(O.reshape(ref.shape) - ref).max() < 1e-12


@pytest.mark.parametrize("ns,w", [(3, 4), (40, 5)])
def test_sink_window_separator_equals_sdpa(oracle_mod, ns, w):
    """Sinks + window + separators with no rotation: SDPA with the mask read
    from the hand-checked oracle mask rows (a narrow and a wide sink span)."""
    B, H, T, d = 2, 2, 80, 8
    q, k, v = _rand_inputs(B, H, H, T, d, 8)
    rng = np.random.default_rng(9)
    sep = (rng.random((B, T)) < 0.2).astype(np.uint8)
    p = oracle_mod.params(B, H, H, T, d, "bf16", ns, w, 0, 0, 0.0)
    O, *_ = oracle_mod.fwd_rows(p, q, k, v, sep, oracle_mod.all_rows(B, H, T))
    O = O.reshape(B, H, T, d)
    for b in range(B):
        mask = np.stack([oracle_mod.mask_row(T, i, ns, w, sep[b])[0] for i in range(T)]).astype(bool)
        ref = _sdpa(_f64(q)[b:b + 1], _f64(k)[b:b + 1], _f64(v)[b:b + 1], mask)
        assert np.abs(O[b] - ref[0]).max() < 1e-12


def test_window_covers_all_is_full_attention(oracle_mod):
    """w + n_start >= T: identical to full causal attention."""
    B, H, T, d = 1, 2, 33, 8
    q, k, v = _rand_inputs(B, H, H, T, d, 10)
    p = oracle_mod.params(B, H, H, T, d, "bf16", 4, T - 4, 0, 0, 0.0)
    O, *_ = oracle_mod.fwd_rows(p, q, k, v, None, oracle_mod.all_rows(B, H, T))
    ref = _sdpa(_f64(q), _f64(k), _f64(v), _tri(T))
    assert np.abs(O.reshape(ref.shape) - ref).max() < 1e-12


def test_rows_are_probability_weights(oracle_mod):
    """One-hot values expose the weight matrix: supported exactly on the
    kept set, summing to one, and sum exp(s - LSE) = 1."""
    T = d = 24
    B = H = 1
    q, k, _ = _rand_inputs(B, H, H, T, d, 11, "f32")
    v = np.eye(T, d, dtype=np.float32)[None, None]
    rng = np.random.default_rng(12)
    sep = (rng.random((1, T)) < 0.25).astype(np.uint8)
    ns, w, kk, L = 2, 3, 2, 5
    p = oracle_mod.params(B, H, H, T, d, "f32", ns, w, L, kk, 1e4)
    O, lse, tki, _, _ = oracle_mod.fwd_rows(p, q, k, v, sep, oracle_mod.all_rows(B, H, T))
    for i in range(T):
        m, _ = oracle_mod.mask_row(T, i, ns, w, sep[0])
        for j in tki[i]:
            if j >= 0:
                m[j] = 1
        wts = O[i]
        assert abs(wts.sum() - 1.0) < 1e-12
        assert np.all(wts[m == 0] == 0.0)
        assert np.all(wts[m == 1] > 0.0)


def test_output_invariant_outside_kept_set(oracle_mod):
    B, H, T, d = 1, 1, 60, 16
    q, k, v = _rand_inputs(B, H, H, T, d, 13)
    rng = np.random.default_rng(14)
    sep = (rng.random((1, T)) < 0.15).astype(np.uint8)
    ns, w, kk, L = 2, 5, 3, 5
    p = oracle_mod.params(B, H, H, T, d, "bf16", ns, w, L, kk, 1e4)
    i = 51
    O0, l0, tki, _, _ = oracle_mod.fwd_rows(p, q, k, v, sep, np.array([[0, 0, i]]))
    m, _ = oracle_mod.mask_row(T, i, ns, w, sep[0])
    for j in tki[0]:
        m[j] = 1
    v2 = v.copy()
    # perturb values of keys outside the kept set (keys of later rows too)
    outside = np.where(m == 0)[0]
    v2[0, 0, outside, :] ^= np.uint16(0x0101)
    O1, l1, *_ = oracle_mod.fwd_rows(p, q, k, v2, sep, np.array([[0, 0, i]]), forced_topk=tki)
    assert np.array_equal(O0, O1) and np.array_equal(l0, l1)


def test_cap_beyond_sequence_is_uncapped(oracle_mod):
    B, H, T, d = 1, 2, 40, 8
    q, k, v = _rand_inputs(B, H, H, T, d, 15)
    rows = oracle_mod.all_rows(B, H, T)
    a = oracle_mod.fwd_rows(oracle_mod.params(B, H, H, T, d, "bf16", 2, 5, 0, 0, 1e4), q, k, v, None, rows)
    b = oracle_mod.fwd_rows(oracle_mod.params(B, H, H, T, d, "bf16", 2, 5, T, 0, 1e4), q, k, v, None, rows)
    assert np.array_equal(a[0], b[0])


@pytest.mark.parametrize("ns,w,L,kk", [(4, 6, 6, 0), (4, 6, 6, 2), (3, 4, 10, 2), (2, 5, 9, 0), (40, 3, 3, 1)])
def test_capped_rope_forward_against_distance_capped_logits(oracle_mod, ns, w, L, kk):
    """The capped-RoPE forward as a whole ("LM-Infinite", section 方法: the
    distance d_ij = i - j is capped to d'_ij = min(d_ij, L) and the rotary
    logit is taken at that distance).  The reference builds every kept
    logit in the test as <R(j + d'_ij) q_i, R(j) k_j> -- the query rotated
    to the key's position plus the capped distance, not the oracle's
    <R(L) q_i, k_j> form -- and takes a plain fp64 softmax over the mask
    rows plus forced top-k keys.  Sinks scaled x8, separators, windows equal
    to and below the cap (so separators and top-k keys fall both inside and
    past the cap), a sink span wider than the window."""
    O = oracle_mod
    B, Hq, Hkv, T, d, theta = 1, 2, 1, 48, 16, 1e4
    q, k, v = _rand_inputs(B, Hq, Hkv, T, d, 31, "f32")
    k = k.copy()
    k[:, :, :4] *= 8.0
    rng = np.random.default_rng(32)
    sep = (rng.random((B, T)) < 0.2).astype(np.uint8)
    forced = np.full((B, Hq, T, max(kk, 1)), -1, dtype=np.int32)
    for h in range(Hq):
        for i in range(T):
            cand = [j for j in range(ns, i - w) if not sep[0, j]]
            if kk and cand:
                pick = rng.choice(cand, size=min(kk, len(cand)), replace=False)
                forced[0, h, i, :len(pick)] = pick
    p = O.params(B, Hq, Hkv, T, d, "f32", ns, w, L, kk, theta)
    rows = O.all_rows(B, Hq, T)
    got, lse, *_ = O.fwd_rows(p, q, k, v, sep, rows, forced_topk=forced[..., :kk] if kk else None)
    q64, k64, v64 = _f64(q), _f64(k), _f64(v)
    n_capped = 0
    for r, (b, h, i) in enumerate(rows):
        g = h * Hkv // Hq
        m, _ = O.mask_row(T, i, ns, w, sep[b])
        for j in forced[b, h, i, :kk]:
            if j >= 0:
                m[j] = 1
        js = np.flatnonzero(m)
        z = np.empty(len(js))
        for x, j in enumerate(js):
            dd = min(i - j, L)
            n_capped += (i - j) > L
            z[x] = np.dot(O.rope(q64[b, h, i], j + dd, theta), O.rope(k64[b, g, j], j, theta))
        s = z / math.sqrt(d)
        mx = s.max()
        wts = np.exp(s - mx)
        ref_lse = mx + math.log(wts.sum())
        ref_o = (np.exp(s - ref_lse)[:, None] * v64[b, g, js]).sum(0)
        assert abs(lse[r] - ref_lse) < 1e-12
        assert np.abs(got[r] - ref_o).max() < 1e-12
    assert n_capped > 100  # the cap is exercised


# ----------------------------------------------------------------------------
# top-k middle tokens
# ----------------------------------------------------------------------------

def test_topk_all_middle_is_full_causal(oracle_mod):
    B, H, T, d = 1, 2, 31, 8
    q, k, v = _rand_inputs(B, H, H, T, d, 16)
    p = oracle_mod.params(B, H, H, T, d, "bf16", 1, 2, 0, T, 0.0)
    O, *_ = oracle_mod.fwd_rows(p, q, k, v, None, oracle_mod.all_rows(B, H, T))
    ref = _sdpa(_f64(q), _f64(k), _f64(v), _tri(T))
    assert np.abs(O.reshape(ref.shape) - ref).max() < 1e-12


def test_topk_bruteforce_selection_and_ties(oracle_mod):
    """Brute force: logits of every middle key from the stand-alone capped
    logit, Python's sort by (-z, j).  Duplicated keys create exact ties."""
    T, d = 30, 8
    q, k, v = _rand_inputs(1, 1, 1, T, d, 17, "f32")
    k[0, 0, 10] = k[0, 0, 7]       # exact tie between keys 7 and 10
    k[0, 0, 12] = k[0, 0, 7]
    ns, w, L, kk, theta = 2, 3, 3, 4, 0.0
    p = oracle_mod.params(1, 1, 1, T, d, "f32", ns, w, L, kk, theta)
    _, _, tki, tkz, _ = oracle_mod.fwd_rows(p, q, k, v, None, oracle_mod.all_rows(1, 1, T))
    qd, kd = _f64(q)[0, 0], _f64(k)[0, 0]
    for i in range(T):
        cands = [(oracle_mod.logit(qd[i], kd[j], i, j, L, theta), j) for j in range(ns, max(ns, i - w))]
        best = sorted(cands, key=lambda t: (-t[0], t[1]))[:kk]
        exp_idx = [j for _, j in best] + [-1] * (kk - len(best))
        assert list(tki[i]) == exp_idx, i
        for r, (z, _) in enumerate(best):
            assert tkz[i, r] == z


def test_topk_finds_planted_keys(oracle_mod):
    """Planted keys (cosine 0.9 to the rotated-to-cap query of a later run)
    must be among the top-k of their run's queries."""
    wl = synth.WORKLOADS["c4_lminf_topk_32k"].scaled(Hq=2, Hkv=2, T=2048, window=256, L_pretrain=256, plant=3)
    inp = synth.make_inputs(wl, seed=3)
    p = oracle_mod.params_of(wl)
    planted = inp["meta"]["planted"]
    rows = []
    for (b, h, j, start) in planted:
        rows += [(b, h, start), (b, h, start + wl.plant_run - 1)]
    rows = np.array(rows, dtype=np.int64)
    _, _, tki, _, _ = oracle_mod.fwd_rows(p, inp["q"], inp["k"], inp["v"], None, rows)
    found = 0
    for r, (b, h, j, start) in enumerate(np.repeat(np.array(planted), 2, axis=0)):
        found += int(j in tki[r])
    assert found >= len(rows) - 1  # a later cluster may overwrite a run


# ----------------------------------------------------------------------------
# block map
# ----------------------------------------------------------------------------

def _classes_from_mask(mask, BM, BN):
    T = mask.shape[0]
    nQT, nKT = -(-T // BM), -(-T // BN)
    out = np.zeros((nQT, nKT), dtype=np.uint8)
    for t in range(nQT):
        for u in range(nKT):
            blk = mask[t * BM:(t + 1) * BM, u * BN:(u + 1) * BN]
            out[t, u] = 0 if not blk.any() else (2 if blk.all() else 1)
    return out


def test_blockmap_against_numpy(oracle_mod):
    B, T, ns, w, BM, BN = 3, 300, 4, 37, 32, 16
    rng = np.random.default_rng(18)
    sep = (rng.random((B, T)) < 0.1).astype(np.uint8)
    cls, pos, cnt, rng_ = oracle_mod.blockmap(B, T, ns, w, BM, BN, sep)
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    for b in range(B):
        sp = np.flatnonzero(sep[b, ns:]) + ns
        assert cnt[b] == len(sp)
        assert np.array_equal(pos[b, : len(sp)], sp) and np.all(pos[b, len(sp):] == -1)
        for t in range(-(-T // BM)):
            first, last = t * BM, min(T - 1, t * BM + BM - 1)
            assert rng_[b, t, 0] == np.searchsorted(sp, first - w, "left")
            assert rng_[b, t, 1] == np.searchsorted(sp, last - w, "left")
        mask = (j <= i) & ((j < ns) | (i - j <= w) | ((sep[b][None, :] == 1) & (j < i)))
        assert np.array_equal(cls[b], _classes_from_mask(mask, BM, BN))


def test_blockmap_band_geometry_no_separators(oracle_mod):
    """Without separators the classes follow from interval arithmetic on the
    sink span and the band i-w <= j <= i."""
    T, ns, w, BM, BN = 512, 4, 100, 64, 64
    cls, _, cnt, _ = oracle_mod.blockmap(1, T, ns, w, BM, BN, None)
    assert cnt[0] == 0
    for t in range(T // BM):
        i0, i1 = t * BM, t * BM + BM - 1
        for u in range(T // BN):
            j0, j1 = u * BN, u * BN + BN - 1
            if j0 > i1:
                exp = 0
            elif j1 <= i0 and (j1 < ns or max(j0, ns) >= i1 - w):
                exp = 2
            elif (j0 < ns) or (j1 >= max(i0, j0) - w):
                exp = 1
            else:
                exp = 0
            assert cls[0, t, u] == exp, (t, u)


# ----------------------------------------------------------------------------
# segmented execution
# ----------------------------------------------------------------------------

def test_segment_key_lists_golden(oracle_mod):
    T, S, M, R, blk, d = 12, 4, 2, 4, 2, 4
    q, k, _ = _rand_inputs(1, 2, 2, T, d, 19)
    p = oracle_mod.params(1, 2, 2, T, d, "bf16", rope_theta=1e4)
    is_long = np.array([0, 1], dtype=np.uint8)
    for line in _read_golden("segment_keys_T12_S4_M2_R4.txt"):
        kind, i, P, keys, poss = line.split()
        h = 0 if kind == "local" else 1
        kj, kp, P_ = oracle_mod.segment_keys(p, S, M, R, blk, is_long, q, k, 0, h, int(i))
        assert P_ == int(P)
        assert list(kj) == list(map(int, keys.split(","))), line
        assert list(kp) == list(map(int, poss.split(","))), line


def test_segment_whole_sequence_is_causal(oracle_mod):
    B, H, T, d = 1, 2, 24, 8
    q, k, v = _rand_inputs(B, H, H, T, d, 20)
    p = oracle_mod.params(B, H, H, T, d, "bf16")
    O, *_ = oracle_mod.segment_rows(p, T, 4, 8, 4, np.array([0, 1], np.uint8), q, k, v,
                                    oracle_mod.all_rows(B, H, T))
    ref = _sdpa(_f64(q), _f64(k), _f64(v), _tri(T))
    assert np.abs(O.reshape(ref.shape) - ref).max() < 1e-12


def test_segment_full_retrieval_is_two_segment_causal(oracle_mod):
    """R = S: the long head at segment 1 retrieves the whole previous segment
    at positions 0..S-1 and sits at S+t, i.e. plain causal attention."""
    B, H, T, d, S = 1, 1, 16, 8, 8
    q, k, v = _rand_inputs(B, H, H, T, d, 21)
    theta = 1e4
    p = oracle_mod.params(B, H, H, T, d, "bf16", rope_theta=theta)
    O, *_ = oracle_mod.segment_rows(p, S, 0, S, 2, np.array([1], np.uint8), q, k, v, oracle_mod.all_rows(B, H, T))
    ref = _sdpa(_rotate_all(_f64(q), theta, oracle_mod), _rotate_all(_f64(k), theta, oracle_mod), _f64(v), _tri(T))
    assert np.abs(O.reshape(ref.shape) - ref).max() < 1e-12


def test_segment_local_tail_is_shifted_window(oracle_mod):
    """Local heads: tail + segment with positions re-based is the same as the
    keys [sS-M, i] at their original positions (a pure shift)."""
    B, H, T, d, S, M = 1, 1, 24, 8, 8, 3
    q, k, v = _rand_inputs(B, H, H, T, d, 22)
    theta = 1e4
    p = oracle_mod.params(B, H, H, T, d, "bf16", rope_theta=theta)
    O, *_ = oracle_mod.segment_rows(p, S, M, 0, 1, np.array([0], np.uint8), q, k, v, oracle_mod.all_rows(B, H, T))
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    lo = np.where(i // S == 0, 0, (i // S) * S - M)
    mask = (j <= i) & (j >= lo)
    ref = _sdpa(_rotate_all(_f64(q), theta, oracle_mod), _rotate_all(_f64(k), theta, oracle_mod), _f64(v), mask)
    assert np.abs(O.reshape(ref.shape) - ref).max() < 1e-12


def test_segment_no_state_is_block_diagonal(oracle_mod):
    B, H, T, d, S = 1, 2, 20, 4, 5
    q, k, v = _rand_inputs(B, H, H, T, d, 23)
    p = oracle_mod.params(B, H, H, T, d, "bf16")
    O, *_ = oracle_mod.segment_rows(p, S, 0, 0, 1, np.array([0, 1], np.uint8), q, k, v, oracle_mod.all_rows(B, H, T))
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    ref = _sdpa(_f64(q), _f64(k), _f64(v), (j <= i) & (j // S == i // S))
    assert np.abs(O.reshape(ref.shape) - ref).max() < 1e-12


def test_segment_retrieval_blocks_bruteforce(oracle_mod):
    B, H, T, d, S, R, blk = 1, 3, 64, 8, 16, 8, 4
    q, k, _ = _rand_inputs(B, H, H, T, d, 24)
    is_long = np.array([1, 0, 1], np.uint8)
    p = oracle_mod.params(B, H, H, T, d, "bf16", rope_theta=1e4)
    got, _ = oracle_mod.segment_blocks(p, S, R, blk, is_long, q, k)
    qd, kd = _f64(q), _f64(k)
    for h in range(H):
        for s in range(T // S):
            if not is_long[h] or s == 0:
                assert np.all(got[0, h, s] == -1)
                continue
            z = kd[0, h, : s * S] @ qd[0, h, s * S - 1]
            bs = z.reshape(-1, blk).max(1)
            order = sorted(range(len(bs)), key=lambda u: (-bs[u], u))[: R // blk]
            assert list(got[0, h, s]) == sorted(order)


def test_segment_effective_context_closed_form(oracle_mod):
    """Keys seen by the last query of a segment s >= 1, averaged over heads,
    is S + alpha*M + (1-alpha)*R (one long layer, beta = 1)."""
    B, H, T, d, S, M, R, blk = 1, 4, 48, 4, 16, 5, 8, 4
    q, k, v = _rand_inputs(B, H, H, T, d, 25)
    is_long = np.array([0, 0, 0, 1], np.uint8)
    alpha = 3 / 4
    p = oracle_mod.params(B, H, H, T, d, "bf16", rope_theta=1e4)
    for s in (1, 2):
        i = s * S + S - 1
        rows = np.array([[0, h, i] for h in range(H)], dtype=np.int64)
        _, _, cnt = oracle_mod.segment_rows(p, S, M, R, blk, is_long, q, k, v, rows)
        assert cnt.mean() == pytest.approx(S + alpha * M + (1 - alpha) * R)


def test_segment_retrieval_ties_go_to_lower_block(oracle_mod):
    """Identical keys in every block make every block score equal: the prefix
    must then be the lowest-numbered blocks."""
    B, H, T, d, S, R, blk = 1, 1, 48, 8, 16, 8, 4
    q, k, _ = _rand_inputs(B, H, H, T, d, 26)
    k = k.copy()
    k[0, 0, :, :] = k[0, 0, 5, :]
    p = oracle_mod.params(B, H, H, T, d, "bf16", rope_theta=1e4)
    got, _ = oracle_mod.segment_blocks(p, S, R, blk, np.array([1], np.uint8), q, k)
    assert list(got[0, 0, 1]) == [0, 1]
    assert list(got[0, 0, 2]) == [0, 1]


# ----------------------------------------------------------------------------
# position interpolation (rotary positions squeezed by one constant factor)
# ----------------------------------------------------------------------------

def test_position_interpolation_equals_spread_sequence(oracle_mod):
    """Position interpolation with scale 1/4 on a sequence whose real tokens
    sit at positions 4j equals plain RoPE attention on the dense sequence:
    a row 4i that keeps exactly the keys 4j (j <= i) -- SepLLM mask with
    window 0 and separators at 4j -- sees rotary positions i and j.  Both
    sides come from the oracle with different masks and scales, so a scale
    applied to only one operand, twice, or to the frequency instead of the
    position fails."""
    B, H, T, d, s = 1, 2, 24, 16, 4
    theta = 1e4
    q, k, v = _rand_inputs(B, H, H, T, d, 21)
    # dense sequence: plain causal attention with rotation
    pd = oracle_mod.params(B, H, H, T, d, "bf16", 0, T, 0, 0, theta)
    Od, ld, *_ = oracle_mod.fwd_rows(pd, q, k, v, None, oracle_mod.all_rows(B, H, T))
    # spread sequence: token j at position s*j, filler elsewhere
    g = np.random.default_rng(5)
    Ts = s * T
    qs = g.integers(0, 2 ** 16, (B, H, Ts, d)).astype(np.uint16) & np.uint16(0x3fff)  # finite bf16 fillers
    ks = g.integers(0, 2 ** 16, (B, H, Ts, d)).astype(np.uint16) & np.uint16(0x3fff)
    vs = g.integers(0, 2 ** 16, (B, H, Ts, d)).astype(np.uint16) & np.uint16(0x3fff)
    qs[:, :, ::s], ks[:, :, ::s], vs[:, :, ::s] = q, k, v
    sep = np.zeros((B, Ts), dtype=np.uint8)
    sep[:, ::s] = 1
    ps = oracle_mod.params(B, H, H, Ts, d, "bf16", 0, 0, 0, 0, theta, 1.0 / s)
    rows = np.array([(0, h, s * i) for h in range(H) for i in range(T)], dtype=np.int64)
    Os, ls, *_ = oracle_mod.fwd_rows(ps, qs, ks, vs, sep, rows)
    dense_rows = np.array([(0, h, i) for h in range(H) for i in range(T)], dtype=np.int64)
    Od2, ld2, *_ = oracle_mod.fwd_rows(pd, q, k, v, None, dense_rows)
    assert np.abs(Os - Od2).max() < 1e-12
    assert np.abs(ls - ld2).max() < 1e-12
    # and the interpolated rotation is not the plain one
    p1 = oracle_mod.params(B, H, H, Ts, d, "bf16", 0, 0, 0, 0, theta)
    O1, *_ = oracle_mod.fwd_rows(p1, qs, ks, vs, sep, rows)
    assert np.abs(O1 - Od2).max() > 1e-3


def test_position_scale_one_is_identity(oracle_mod):
    B, H, T, d = 1, 2, 50, 16
    q, k, v = _rand_inputs(B, H, H, T, d, 22)
    rows = oracle_mod.all_rows(B, H, T)
    a = oracle_mod.fwd_rows(oracle_mod.params(B, H, H, T, d, "bf16", 4, 9, 9, 0, 1e4), q, k, v, None, rows)
    b = oracle_mod.fwd_rows(oracle_mod.params(B, H, H, T, d, "bf16", 4, 9, 9, 0, 1e4, 1.0), q, k, v, None, rows)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ----------------------------------------------------------------------------
# clipped ALiBi (LM-Infinite, section 方法: the distance bias clipped at L)
# ----------------------------------------------------------------------------

# ALiBi's published slope sets: 8 heads take 1/2, 1/4, ..., 1/256 and 4 heads
# 1/4, 1/16, 1/64, 1/256 (each the geometric sequence from 2^(-8/H))
ALIBI_SLOPES = {8: [2.0 ** -x for x in range(1, 9)], 4: [2.0 ** -x for x in (2, 4, 6, 8)]}


def _sdpa_bias(q64, k64, v64, bias):
    """torch SDPA in fp64 with an additive float mask bias [H, T, T] (-inf =
    masked); returns O and the natural-log LSE of the biased scaled logits."""
    rep = q64.shape[1] // k64.shape[1]
    k = np.repeat(k64, rep, axis=1)
    v = np.repeat(v64, rep, axis=1)
    bt = torch.from_numpy(bias)[None]
    O = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q64), torch.from_numpy(k),
                                                         torch.from_numpy(v), attn_mask=bt).numpy()
    s = np.einsum("bhid,bhjd->bhij", q64, k) / math.sqrt(q64.shape[-1]) + bias[None]
    mx = s.max(-1, keepdims=True)
    lse = (mx + np.log(np.exp(s - mx).sum(-1, keepdims=True)))[..., 0]
    return O, lse


def _alibi_bias(H, T, mask, L):
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    dist = (i - j).astype(np.float64)
    if L > 0:
        dist = np.minimum(dist, L)
    m = np.array(ALIBI_SLOPES[H])[:, None, None]
    return np.where(mask[None], -m * dist[None], -np.inf)


def test_alibi_unclipped_causal_equals_sdpa_with_bias(oracle_mod):
    """L = 0: plain ALiBi over full causal attention, 8 heads with the
    published slopes."""
    B, H, T, d = 1, 8, 40, 16
    q, k, v = _rand_inputs(B, H, 2, T, d, 31)
    p = oracle_mod.params(B, H, 2, T, d, "bf16", 0, T, 0, 0, 0.0, alibi=True)
    O, lse, *_ = oracle_mod.fwd_rows(p, q, k, v, None, oracle_mod.all_rows(B, H, T))
    ref, lref = _sdpa_bias(_f64(q), _f64(k), _f64(v), _alibi_bias(H, T, _tri(T), 0))
    assert np.abs(O.reshape(ref.shape) - ref).max() < 1e-12
    assert np.abs(lse.reshape(lref.shape) - lref).max() < 1e-12


def test_alibi_clipped_lambda_equals_sdpa_with_bias(oracle_mod):
    """Lambda mask (sinks + window w = L) with the bias clipped at L: the
    starting-span keys beyond the window get -m L, window keys -m (i - j)."""
    B, H, T, d = 2, 4, 48, 16
    ns, L = 3, 6
    q, k, v = _rand_inputs(B, H, H, T, d, 32, "f32")
    p = oracle_mod.params(B, H, H, T, d, "f32", ns, L, L, 0, 0.0, alibi=True)
    O, lse, *_ = oracle_mod.fwd_rows(p, q, k, v, None, oracle_mod.all_rows(B, H, T))
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    lam = (j <= i) & ((j < ns) | (i - j <= L))
    ref, lref = _sdpa_bias(_f64(q), _f64(k), _f64(v), _alibi_bias(H, T, lam, L))
    assert np.abs(O.reshape(ref.shape) - ref).max() < 1e-12
    assert np.abs(lse.reshape(lref.shape) - lref).max() < 1e-12
    # the clip matters: the unclipped bias gives another answer
    ref2, _ = _sdpa_bias(_f64(q), _f64(k), _f64(v), _alibi_bias(H, T, lam, 0))
    assert np.abs(O.reshape(ref.shape) - ref2).max() > 1e-3


def test_alibi_clipped_separators_equals_sdpa_with_bias(oracle_mod):
    """SepLLM mask with the clipped bias: every separator beyond the window
    sits at the cap."""
    B, H, T, d = 1, 4, 45, 8
    ns, w = 2, 5
    q, k, v = _rand_inputs(B, H, 1, T, d, 33)
    rng = np.random.default_rng(34)
    sep = (rng.random((B, T)) < 0.25).astype(np.uint8)
    p = oracle_mod.params(B, H, 1, T, d, "bf16", ns, w, w, 0, 0.0, alibi=True)
    O, lse, *_ = oracle_mod.fwd_rows(p, q, k, v, sep, oracle_mod.all_rows(B, H, T))
    mask = np.stack([oracle_mod.mask_row(T, i, ns, w, sep[0])[0] for i in range(T)]).astype(bool)
    ref, lref = _sdpa_bias(_f64(q), _f64(k), _f64(v), _alibi_bias(H, T, mask, w))
    assert np.abs(O.reshape(ref.shape) - ref).max() < 1e-12
    assert np.abs(lse.reshape(lref.shape) - lref).max() < 1e-12


def test_alibi_topk_ranks_by_biased_logit(oracle_mod):
    """Brute force: with the cap above the window the bias varies among the
    candidates and decides the ranking (key z - sqrt(d) m min(i-j, L));
    reported values stay the unbiased z.  With L = w every candidate is past
    the cap and the set equals the one without the bias."""
    T, d, H = 40, 8, 4
    q, k, v = _rand_inputs(1, H, H, T, d, 35, "f32")
    ns, w, L, kk = 2, 3, 12, 4
    p = oracle_mod.params(1, H, H, T, d, "f32", ns, w, L, kk, 0.0, alibi=True)
    _, _, tki, tkz, _ = oracle_mod.fwd_rows(p, q, k, v, None, oracle_mod.all_rows(1, H, T))
    tki = tki.reshape(H, T, kk)
    tkz = tkz.reshape(H, T, kk)
    qd, kd = _f64(q)[0], _f64(k)[0]
    differs = 0
    for h in range(H):
        m = ALIBI_SLOPES[H][h]
        for i in range(T):
            cands = []
            for j in range(ns, max(ns, i - w)):
                z = float(qd[h, i] @ kd[h, j])
                cands.append((z - math.sqrt(d) * m * min(i - j, L), z, j))
            best = sorted(cands, key=lambda t: (-t[0], t[2]))[:kk]
            plain = sorted(cands, key=lambda t: (-t[1], t[2]))[:kk]
            assert list(tki[h, i]) == [j for *_, j in best] + [-1] * (kk - len(best)), (h, i)
            for r, (_, z, _) in enumerate(best):
                assert abs(tkz[h, i, r] - z) < 1e-12
            differs += int([t[2] for t in best] != [t[2] for t in plain])
    assert differs > 0
    p2 = oracle_mod.params(1, H, H, T, d, "f32", ns, w, w, kk, 0.0, alibi=True)
    p3 = oracle_mod.params(1, H, H, T, d, "f32", ns, w, w, kk, 0.0)
    a = oracle_mod.fwd_rows(p2, q, k, v, None, oracle_mod.all_rows(1, H, T))
    b = oracle_mod.fwd_rows(p3, q, k, v, None, oracle_mod.all_rows(1, H, T))
    assert np.array_equal(a[2], b[2])


# ----------------------------------------------------------------------------
# SharedLLM tree cross-attention (sections 关键设计 2 and 4)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("m,depth,alpha", [(6, 1, 1), (6, 2, 1), (6, 3, 2), (8, 4, 1), (8, 2, 4)])
def test_tree_index_closed_form(oracle_mod, m, depth, alpha):
    """Chunk length l = 2^m: the kept left node of level w spans
    [l - l/2^(w-1), l - l/2^w) at rate alpha 2^(D-w), the kept right node of
    level D the last l/2^D positions at rate alpha; every node keeps
    l / (alpha 2^D) rows, equally spaced from its start."""
    l = 2 ** m
    per = l // (alpha * 2 ** depth)
    exp = []
    for w in range(1, depth + 1):
        start = l - l // 2 ** (w - 1)
        exp += [start + k * alpha * 2 ** (depth - w) for k in range(per)]
    exp += [l - l // 2 ** depth + k * alpha for k in range(per)]
    assert list(oracle_mod.tree_index(l, depth, alpha)) == exp


@pytest.mark.parametrize("l", [1, 2, 3, 7, 100, 1000, 1023])
def test_tree_index_properties(oracle_mod, l):
    """Any length: offsets strictly increasing inside [0, l); depth 0 at rate
    1 keeps everything; the kept count is the sum of max(1, floor(m/alpha))
    over the kept nodes of the halving splits."""
    for depth in range(0, 5):
        for alpha in (1, 2, 3):
            idx = oracle_mod.tree_index(l, depth, alpha)
            assert np.all(np.diff(idx) > 0) and idx[0] >= 0 and idx[-1] < l
            # node lengths of the halving splits, independently of the oracle
            nodes, length = [], l
            if depth == 0:
                nodes = [(l, 0)]
            for w in range(1, depth + 1):
                b = length // 2
                nodes.append((b, w))
                if w == depth:
                    nodes.append((length - b, w))
                length -= b
            want = sum(max(1, m // (alpha * 2 ** (depth - w))) for m, w in nodes if m > 0)
            assert len(idx) == want
    assert list(oracle_mod.tree_index(l, 0, 1)) == list(range(l))


def _rot_np(O, x, pos, theta):
    return O.rope(np.ascontiguousarray(x, dtype=np.float64), pos, theta)


@pytest.mark.parametrize("theta,depth,alpha", [(0.0, 0, 1), (1e4, 2, 1), (1e4, 3, 2), (5e5, 1, 4)])
def test_tree_cross_equals_sdpa_on_kept_rows(oracle_mod, theta, depth, alpha):
    """Unmasked SDPA over the kept rows of every chunk, the query rotated to
    position n and chunk c's keys to position c (depth 0, rate 1, no
    rotation: plain dense attention over the whole context)."""
    O = oracle_mod
    B, Hq, Hkv, T, d = 1, 4, 2, 7, 16
    n, l = 5, 24
    q, _, _ = _rand_inputs(B, Hq, Hkv, T, d, 40)
    _, k, v = _rand_inputs(B, Hq, Hkv, n * l, d, 41)
    p = O.params(B, Hq, Hkv, T, d, "bf16", rope_theta=theta)
    got, lse = O.tree_cross(p, n, l, depth, alpha, q, k, v)
    idx = O.tree_index(l, depth, alpha)
    q64, k64, v64 = _f64(q), _f64(k), _f64(v)
    rows = [c * l + j for c in range(n) for j in idx]
    kk = k64[:, :, rows].copy()
    for x, r in enumerate(rows):
        for g in range(Hkv):
            kk[0, g, x] = _rot_np(O, kk[0, g, x], r // l, theta)
    qq = q64.copy()
    for h in range(Hq):
        for i in range(T):
            qq[0, h, i] = _rot_np(O, qq[0, h, i], n, theta)
    ref = _sdpa(qq, kk, v64[:, :, rows], np.ones((T, len(rows)), dtype=bool))
    assert np.abs(got - ref).max() < 1e-12
    if depth == 0 and alpha == 1 and theta == 0.0:
        full = _sdpa(q64, k64, v64, np.ones((T, n * l), dtype=bool))
        assert np.abs(got - full).max() < 1e-12
    lref = _lse_ref(qq, kk, np.ones((T, len(rows)), dtype=bool))
    assert np.abs(lse - lref).max() < 1e-12


def test_tree_index_hand_worked_ragged(oracle_mod):
    """Uneven splits (chunk lengths not a power of two), worked out by hand
    (tests/golden/tree_kept_ragged.txt)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tree_kept_ragged.txt")
    for ln in open(path):
        if not ln.strip() or ln.startswith("#"):
            continue
        l, depth, alpha, want = ln.split()
        got = list(oracle_mod.tree_index(int(l), int(depth), int(alpha)))
        assert got == [int(x) for x in want.split(",")], ln
