"""The comparison rule for top-k selections (``_util.topk_row_verdict``),
checked on hand-made rows: selections that must pass and planted mistakes
that must fail.  No GPU."""
import numpy as np

from _util import TIE_REL, topk_row_verdict

INF = float("inf")


def _row(z):
    """Oracle picks 100, 101, ... with the given logits (already sorted)."""
    return [100 + x for x in range(len(z))], np.array(z, dtype=np.float64)


def test_exact_and_padding():
    o, z = _row([5.0, 4.0, 3.0, 2.0, 1.0, 0.5])
    assert topk_row_verdict(o[:3], o, z, 3) == "exact"
    o2 = [100, 101, -1, -1, -1]
    z2 = np.array([5.0, 4.0, -INF, -INF, -INF])
    assert topk_row_verdict([100, 101, -1], o2, z2, 3) == "exact"
    assert topk_row_verdict([100, -1, -1], o2, z2, 3) != "exempt"
    assert topk_row_verdict([101, 100, -1], o2, z2, 3) != "exempt"  # clear order swap


def test_swap_at_the_kth_position_under_a_near_tie():
    zk = 3.0
    o, z = _row([5.0, 4.0, zk, zk * (1 - TIE_REL / 4), 1.0, 0.5])
    assert topk_row_verdict([100, 101, 103], o, z, 3) == "exempt"
    # without the near tie the same swap fails
    o, z = _row([5.0, 4.0, zk, zk * (1 - 10 * TIE_REL), 1.0, 0.5])
    assert topk_row_verdict([100, 101, 103], o, z, 3) != "exempt"


def test_near_tie_higher_up_does_not_excuse_a_wrong_key():
    # the 1st and 2nd logits are near-tied, but the k-th and (k+1)-th are not:
    # a wrong key at position 3 must fail (the old rule let it pass)
    o, z = _row([5.0, 5.0 * (1 - TIE_REL / 4), 3.0, 2.0, 1.0, 0.5])
    assert topk_row_verdict([100, 101, 104], o, z, 3) != "exempt"
    # their order may flip
    assert topk_row_verdict([101, 100, 102], o, z, 3) == "exempt"


def test_key_above_the_tied_run_must_stay():
    zk = 3.0
    o, z = _row([5.0, 4.0, zk, zk * (1 - TIE_REL / 4), 1.0, 0.5])
    # dropping the clear 2nd pick for the tied (k+1)-th fails
    assert topk_row_verdict([100, 102, 103], o, z, 3) != "exempt"


def test_pick_outside_the_listed_candidates_fails():
    o, z = _row([5.0, 4.0, 3.0, 3.0 * (1 - TIE_REL / 4), 1.0])
    assert topk_row_verdict([100, 101, 999], o, z, 3) != "exempt"
    assert topk_row_verdict([100, 100, 101], o, z, 3) != "exempt"


def test_negative_logits():
    zk = -2.0
    o, z = _row([1.0, -1.0, zk, zk * (1 + TIE_REL / 4), -5.0])
    assert topk_row_verdict([100, 101, 103], o, z, 3) == "exempt"
    o, z = _row([1.0, -1.0, zk, zk * (1 + 10 * TIE_REL), -5.0])
    assert topk_row_verdict([100, 101, 103], o, z, 3) != "exempt"
