"""The end-to-end host path cuts a problem into pieces that are copied,
computed and copied back on separate streams.  The cut is host logic: every
(sequence, kv head) must land in exactly one piece, pieces must be whole
sequence ranges or one sequence's range of kv heads (so each copy of Q, K, V
and the outputs is one contiguous block), and there should be about the
requested number of them."""
import itertools

import pytest

from long_context_structured_b200 import _host_chunks


@pytest.mark.parametrize("B,Hkv,n", [(1, 32, 8), (4, 8, 8), (3, 2, 8), (16, 8, 8), (1, 1, 8), (2, 32, 8),
                                     (5, 3, 4), (1, 7, 8), (64, 8, 8)])
def test_pieces_tile_the_problem(B, Hkv, n):
    pieces = _host_chunks(B, Hkv, n)
    cells = [(b, g) for b0, b1, g0, g1 in pieces for b in range(b0, b1) for g in range(g0, g1)]
    assert sorted(cells) == list(itertools.product(range(B), range(Hkv)))  # each exactly once
    for b0, b1, g0, g1 in pieces:
        assert 0 <= b0 < b1 <= B and 0 <= g0 < g1 <= Hkv
        # contiguous in [B, H, ...] memory: whole heads, or one sequence
        assert (g0, g1) == (0, Hkv) or b1 - b0 == 1
    assert len(pieces) <= max(n, 1)
    assert len(pieces) >= min(n, B * Hkv) // 2

