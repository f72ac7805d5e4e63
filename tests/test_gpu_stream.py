"""GPU parity of the streaming KV cache (SepLLM, section 6.2) against the
plain reference in oracle/stream_cache.py: region sizes and the stream
position of every slot bit-exact after each checked append, and decoding
steps over the cache (rolled positions) within the bf16 bars."""
import numpy as np
import pytest
import torch

import long_context_structured_b200 as sa
from long_context_structured_b200 import _lib
from oracle.stream_cache import StreamCache, decode_step
from _util import BF16_MAX_ABS, BF16_MEAN_ABS, compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


CASES = [
    # B, Hkv, Hq, d, a, s, w, c, sep rate, tokens, theta
    ("gqa2_d128", (2, 2, 4, 128, 4, 32, 64, 160, 0.2, 1200, 1e4)),
    ("no_initial_d64_gqa8", (1, 1, 8, 64, 0, 8, 16, 40, 0.35, 500, 5e5)),
    ("wide_window_rare_seps", (3, 2, 2, 128, 4, 16, 200, 300, 0.03, 900, 1e4)),
    ("window1_all_seps", (1, 1, 1, 128, 2, 5, 1, 12, 1.0, 200, 0.0)),
]


@pytest.mark.parametrize("name,cfg", CASES, ids=[c[0] for c in CASES])
def test_stream_cache_matches_reference(oracle_mod, name, cfg):
    B, Hkv, Hq, d, a, s, w, c, rate, n_tok, theta = cfg
    rng = np.random.default_rng(abs(hash(name)) % 2 ** 32)
    flags = rng.random((B, n_tok)) < rate
    kall = torch.randn(n_tok, B, Hkv, d, generator=torch.Generator().manual_seed(1)).bfloat16()
    vall = torch.randn(n_tok, B, Hkv, d, generator=torch.Generator().manual_seed(2)).bfloat16()
    cache = sa.StreamKV(B, Hkv, d, a, s, w, c)
    refs = [StreamCache(a, s, w, c) for _ in range(B)]
    kd, vd = kall.cuda(), vall.cuda()
    fd = torch.from_numpy(flags.astype(np.uint8)).cuda()
    n_dec = 0
    for t in range(n_tok):
        cache.append(kd[t], vd[t], fd[:, t])
        for b in range(B):
            refs[b].append(t, flags[b, t])
        if t < 3 * c or t % 7 == 0 or t == n_tok - 1:
            sizes, pos = cache.read()
            for b in range(B):
                r = refs[b]
                want = [len(r.init), len(r.sep), len(r.past), len(r.local)]
                assert list(sizes[b]) == want, (t, b)
                assert list(pos[b, : r.size()]) == [p for p, _ in r.slots()], (t, b)
        if t % 97 == 5 or t == n_tok - 1:
            q = torch.randn(B, Hq, 1, d, generator=torch.Generator().manual_seed(t)).bfloat16()
            O, lse = cache.decode(q.cuda(), rope_theta=theta)
            torch.cuda.synchronize()
            for b in range(B):
                slots = [p for p, _ in refs[b].slots()]
                k64 = kall[slots, b].double().numpy().transpose(1, 0, 2)
                v64 = vall[slots, b].double().numpy().transpose(1, 0, 2)
                Oref, lref = decode_step(k64, v64, q[b, :, 0].double().numpy(), theta, oracle_mod.rope)
                compare("O", O[b, :, 0].double().cpu().numpy(), Oref, BF16_MAX_ABS, BF16_MEAN_ABS)
                compare("LSE", lse[b].double().cpu().numpy(), lref, BF16_MAX_ABS, BF16_MEAN_ABS)
            n_dec += 1
    assert n_dec >= 2


def test_stream_rejects_no_room():
    with pytest.raises(_lib.SattnError):
        sa.StreamKV(1, 1, 128, 4, 10, 20, 34)
