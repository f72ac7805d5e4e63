"""Pins of the streaming-cache reference (SepLLM, section 6.2) against the
page's occupancy bound, a direct characterisation of the kept sets, and
torch SDPA for one decoding step with rolled positions."""
import numpy as np
import pytest
import torch

from oracle.stream_cache import StreamCache, decode_step


@pytest.mark.parametrize("a,s,w,c,rate", [(4, 64, 256, 1024, 0.1), (4, 8, 32, 64, 0.3), (0, 16, 16, 40, 0.05),
                                          (2, 100, 50, 400, 0.5)])
def test_occupancy_bound_and_kept_sets(a, s, w, c, rate):
    rng = np.random.default_rng(a + s + w + c)
    n = 20000
    flags = rng.random(n) < rate
    cache = StreamCache(a, s, w, c)
    sizes = []
    L0 = None  # local start at the last compaction
    for t in range(n):
        compacted = cache.append(t, flags[t])
        size = cache.size()
        sizes.append(size)
        assert size < c
        pos = [p for p, _ in cache.slots()]
        assert pos == sorted(pos) and len(set(pos)) == len(pos)
        assert [p for p, _ in cache.init] == list(range(min(a, t + 1)))
        local = [p for p, _ in cache.local]
        if t + 1 > a:
            assert local == list(range(max(a, t + 1 - w), t + 1))
        if compacted:
            assert not cache.past
            L0 = local[0]
            # the separator cache: the most recent s separators among [a, L0)
            want = [p for p in range(a, L0) if flags[p]]
            want = want[max(0, len(want) - s):]
            assert [p for p, _ in cache.sep] == want
        past = [p for p, _ in cache.past]
        if L0 is not None and past:
            assert past == list(range(L0, local[0]))
    # SepLLM, section 五 item 3: average occupancy <= (w + c + a + s) / 2
    assert np.mean(sizes[c:]) <= (w + c + a + s) / 2
    # and the bound is nearly reached when separators fill their cache
    if rate >= 0.3:
        assert np.mean(sizes[c:]) > 0.8 * (w + c + a + s) / 2


def test_rejects_capacity_without_room():
    with pytest.raises(ValueError):
        StreamCache(4, 10, 20, 34)


@pytest.mark.parametrize("theta", [0.0, 1e4])
def test_decode_step_equals_sdpa_with_rolled_positions(oracle_mod, theta):
    """The query at slot n-1 and key x at slot x: SDPA over the rotated rows."""
    rng = np.random.default_rng(7)
    Hq, Hkv, n, d = 4, 2, 37, 16
    k = rng.standard_normal((Hkv, n, d))
    v = rng.standard_normal((Hkv, n, d))
    q = rng.standard_normal((Hq, d))
    O, lse = decode_step(k, v, q, theta, oracle_mod.rope)
    qr = np.stack([oracle_mod.rope(q[h], n - 1, theta) for h in range(Hq)])[None, :, None, :]
    kr = np.stack([[oracle_mod.rope(k[g, x], x, theta) for x in range(n)] for g in range(Hkv)])[None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qr), torch.from_numpy(kr).repeat_interleave(Hq // Hkv, 1),
        torch.from_numpy(v[None]).repeat_interleave(Hq // Hkv, 1)).numpy()[0, :, 0]
    assert np.abs(O - ref).max() < 1e-12


def test_hand_worked_trace():
    """The cache's contents after every token of a hand-worked stream
    (tests/golden/stream_cache_a1_s2_w2_c6.txt)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "stream_cache_a1_s2_w2_c6.txt")
    lines = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    a, s, w, c = (int(x) for x in lines[0])
    seps = {int(x) for x in lines[1]}
    cache = StreamCache(a, s, w, c)
    for t_str, want in lines[2:]:
        t = int(t_str)
        cache.append(t, t in seps)
        assert [e[0] for e in cache.slots()] == [int(x) for x in want.split(",")], "after token %d" % t
