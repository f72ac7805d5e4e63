"""Precision of the decoding step's rotation angle, restated on the host.

The decoding kernels do not read a rotary table: for rotary pair c at
position p they form the angle in turns, p * f_c with f_c = s theta^(-2c/d)
/ (2 pi) (the rotation of "LM-Infinite", section 方法, whose capped logit
uses the same rotary angles), from
two fp32 parts f_c = hi + lo prepared on the host, as

    t1 = fl(p * hi);  e1 = fma(p, hi, -t1)            (exact residual)
    whole = fl(fl(t1 + 1.5 * 2^23) - 1.5 * 2^23)       (nearest whole turn)
    r = fl(fl(t1 - whole) + fma(p, lo, e1))            (turns, |r| <= 1/2 + 2^-7)

This test replays exactly those fp32 operations with numpy (a float32 fma
is exact in float64 when the result is representable, which the residual
is) and checks the reduced angle against the exact fractional turn count,
over every position a decoding step may use (below 4096 chunks of 128).
"""
import numpy as np
import pytest

MAGIC = np.float32(12582912.0)  # 1.5 * 2^23
MAX_POS = 4096 * 128  # the longest key set a decoding step merges


def _fma32(a, b, c):
    """fp32 fused multiply-add: exact product and sum in float64, one rounding."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _reduced_turns(p, hi, lo):
    fp = p.astype(np.float32)
    t1 = (fp * hi).astype(np.float32)
    e1 = _fma32(fp, hi, -t1)
    whole = ((t1 + MAGIC).astype(np.float32) - MAGIC).astype(np.float32)
    return ((t1 - whole).astype(np.float32) + _fma32(fp, lo, e1)).astype(np.float32)


@pytest.mark.parametrize("theta,scale,d", [(1e4, 1.0, 128), (5e5, 1.0, 128), (1e4, 0.25, 64), (5e5, 0.5, 64)])
def test_reduced_angle_within_bound(theta, scale, d):
    rng = np.random.default_rng(int(theta) + d)
    p = np.concatenate([np.arange(0, 4096), rng.integers(0, MAX_POS, size=20000), [MAX_POS - 1]]).astype(np.int64)
    worst = 0.0
    for c in range(d // 2):
        f = scale * theta ** (-2.0 * c / d) / (2.0 * np.pi)  # turns per position, as the host computes it
        hi = np.float32(f)
        lo = np.float32(f - np.float64(hi))
        r = _reduced_turns(p, hi, lo).astype(np.float64)
        exact = p.astype(np.float64) * f
        err = np.abs(((r - exact) + 0.5) % 1.0 - 0.5)  # distance modulo whole turns
        # the residuals can push the reduced angle just past half a turn: by
        # at most half an ulp of p * hi plus |p * lo|, 2^-7 turns at the
        # largest p
        assert np.all(np.abs(r) <= 0.5 + 2.0 ** -7)
        worst = max(worst, float(err.max()))
    # about 2^-24 of the reduced angle plus the rounding of the two products
    assert worst < 2e-7, worst


def test_magic_rounding_is_nearest_even():
    t = np.array([0.5, 1.5, 2.5, -0.5, -1.5, 3.25, 83000.49, 83000.5, 83001.5, -7.75], dtype=np.float32)
    got = ((t + MAGIC).astype(np.float32) - MAGIC).astype(np.float32)
    assert np.array_equal(got, np.rint(t).astype(np.float32))


def test_int_to_float_by_magic_bits():
    """(float)p as bits(1.5 * 2^23) + p, minus 1.5 * 2^23, for |p| < 2^22."""
    p = np.array([-3, -1, 0, 1, 2, 4095, 123457, MAX_POS - 1, (1 << 22) - 1], dtype=np.int64)
    bits = (np.int64(0x4B400000) + p).astype(np.uint32)
    got = (bits.view(np.float32) - MAGIC).astype(np.float32)
    assert np.array_equal(got, p.astype(np.float32))
