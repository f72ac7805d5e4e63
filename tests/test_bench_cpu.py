"""Host logic of the benchmark (CPU only).

The benchmark's metric counts kept (q, k) pairs with closed forms (window and
sink span, separators by prefix sums, top-k, segmented tail / prefix).  These
tests pin those counts to the oracle, which materialises every row's 0/1
mask and reports how many keys it kept.
"""
import numpy as np
import pytest

import bench
from long_context_structured_b200 import synth


@pytest.fixture(scope="module")
def oracle_mod():
    from oracle import oracle as O
    O.build()
    return O


SMALL = [
    synth.Workload(name="lam", B=1, Hq=2, Hkv=1, T=300, d=16, dtype="bf16", n_start=4, window=37,
                   L_pretrain=37, rope_theta=1e4),
    synth.Workload(name="sep", B=3, Hq=4, Hkv=2, T=257, d=16, dtype="bf16", n_start=3, window=20,
                   rope_theta=5e5, sep_rate=0.2),
    synth.Workload(name="tok", B=2, Hq=2, Hkv=2, T=200, d=16, dtype="bf16", n_start=4, window=30,
                   rope_theta=5e5, sep_vocab=100, sep_ids=9, sep_rate=0.1),
    synth.Workload(name="topk", B=1, Hq=2, Hkv=2, T=260, d=16, dtype="bf16", n_start=4, window=40,
                   L_pretrain=40, rope_theta=1e4, topk=5),
]


@pytest.mark.parametrize("wl", SMALL, ids=[w.name for w in SMALL])
def test_pair_counts_match_oracle_masks(oracle_mod, wl):
    O = oracle_mod
    inp = synth.make_inputs(wl, seed=3)
    rows = O.all_rows(wl.B, wl.Hq, wl.T)
    *_, cnt = O.fwd_rows(O.params_of(wl), inp["q"], inp["k"], inp["v"], inp["is_sep"], rows, nthreads=2)
    assert bench.unmasked_pairs(wl, inp["is_sep"]) == int(cnt.sum())
    sub = rows[::7]
    assert bench._pairs_of_rows(wl, sub, inp["is_sep"]) == int(cnt[::7].sum())


def test_segmented_pair_counts_match_oracle(oracle_mod):
    O = oracle_mod
    wl = synth.Workload(name="seg", B=1, Hq=4, Hkv=4, T=256, d=16, dtype="bf16", rope_theta=1e4, seg_S=64,
                        seg_M=16, seg_R=32, retr_block=8, long_heads=(2, 3))
    inp = synth.make_inputs(wl, seed=5)
    rows = O.all_rows(wl.B, wl.Hq, wl.T)
    _, _, cnt = O.segment_rows(O.params_of(wl), wl.seg_S, wl.seg_M, wl.seg_R, wl.retr_block, inp["is_long"],
                               inp["q"], inp["k"], inp["v"], rows, nthreads=2)
    assert bench.unmasked_pairs(wl) == int(cnt.sum())
    assert bench._pairs_of_rows(wl, rows[::5], None) == int(cnt[::5].sum())


def test_full_workload_counts():
    """The counts the benchmark reports for the full workloads (closed forms:
    the Lambda-mask layer keeps min(i+1, n_start+w+1) keys per row; the
    segmented layer keeps t+1 in-segment keys plus M or R carried keys)."""
    W = synth.WORKLOADS
    assert bench.unmasked_pairs(W["c2_lminf_16k"]) == 58_783_734 * 32
    assert bench.unmasked_pairs(W["c5_segmented_32k"]) == 1_183_186_944 + 520_224_768
    c4 = W["c4_lminf_topk_32k"]
    assert bench.unmasked_pairs(c4) == (125_974_518 + 143_325) * 32
    assert bench.scored_candidates(c4) == int(np.maximum(0, np.arange(c4.T) - c4.window - c4.n_start).sum()) * 32


def test_workload_aliases_resolve():
    for short, full in bench.WORKLOAD_ALIASES.items():
        assert full in synth.WORKLOADS, short


def test_decode_key_counts_match_oracle(oracle_mod):
    """Kept keys of the decoded position per sequence equal the oracle's mask
    counts of row T-1."""
    O = oracle_mod
    for wl in SMALL[:3]:
        inp = synth.make_inputs(wl, seed=4)
        rows = np.array([(b, 0, wl.T - 1) for b in range(wl.B)], dtype=np.int64)
        *_, cnt = O.fwd_rows(O.params_of(wl.scaled(topk=0)), inp["q"], inp["k"], inp["v"], inp["is_sep"], rows,
                             nthreads=2)
        assert list(bench.decode_keys(wl, inp["is_sep"])) == list(cnt)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_head_split_work_adds_up(world):
    """The strong-scaling mode reports the whole layer's FLOPs: the ranks'
    head blocks (whole kv groups) count exactly the layer's kept pairs."""
    from long_context_structured_b200.shard import head_shard
    wl = synth.Workload(name="sep", B=2, Hq=16, Hkv=8, T=300, d=16, dtype="bf16", n_start=3, window=20,
                        rope_theta=5e5, sep_rate=0.2)
    inp = synth.make_inputs(wl, seed=4)
    total = bench.unmasked_pairs(wl, inp["is_sep"])
    parts = 0
    for r in range(world):
        q0, q1, kv0, kv1 = head_shard(wl.Hq, wl.Hkv, world, r)
        if q1 > q0:
            parts += bench.unmasked_pairs(wl.scaled(Hq=q1 - q0, Hkv=kv1 - kv0), inp["is_sep"])
    assert parts == total


def test_decode_topk_pairs():
    """A decoding step with top-k keeps the structured keys plus k middle
    keys per head (fewer when fewer candidates exist)."""
    wl = synth.Workload(name="d", B=1, Hq=4, Hkv=4, T=100, d=16, dtype="bf16", n_start=4, window=30,
                        L_pretrain=30, rope_theta=1e4, topk=5)
    keys = bench.decode_keys(wl, None)
    assert int(keys[0]) == 4 + 31  # sinks + window (i - w .. i)
    ncand = wl.T - 1 - wl.window - wl.n_start
    assert ncand == 65 and min(wl.topk, ncand) == 5
