"""The arithmetic behind KIE_SUM_EXACT, checked in float32 on the CPU.

Each contribution v is split into hi = v rounded to a multiple of 2^-8 and
lo = (v - hi) rounded to a multiple of 2^-25; hi and lo are summed in fp32
into separate accumulators.  With fewer than 256 contributions below 256 in
magnitude, every partial sum fits fp32's 24-bit significand, so each addition
is exact: any order gives the same bits, and hi_sum + lo_sum is within
n * 2^-26 of the exact sum of the v.
"""
import numpy as np
import pytest

HI_Q = np.float32(256.0)
LO_Q = np.float32(2.0 ** 25)


def split(v):
    v = np.asarray(v, dtype=np.float32)
    hi = (np.rint(v * HI_Q) / HI_Q).astype(np.float32)
    lo = (np.rint((v - hi) * LO_Q) / LO_Q).astype(np.float32)
    return hi, lo


def fp32_sum(x, order):
    acc = np.float32(0.0)
    for i in order:
        acc = np.float32(acc + x[i])
    return acc


@pytest.mark.parametrize("scale", [1e-3, 0.05, 1.0, 30.0, 255.0])
def test_split_sums_do_not_depend_on_order(scale):
    rng = np.random.default_rng(int(scale * 1000) + 1)
    n = 148
    for trial in range(20):
        v = (rng.standard_normal(n) * scale).astype(np.float32)
        v = np.clip(v, -255.9, 255.9).astype(np.float32)
        hi, lo = split(v)
        # the split is exact: hi + lo differs from v only by lo's rounding
        assert np.all(np.abs((hi.astype(np.float64) + lo) - v) <= 2.0 ** -26)
        assert np.all(np.abs(lo) <= 2.0 ** -9)
        ref = None
        for _ in range(8):
            order = rng.permutation(n)
            s = np.float32(fp32_sum(hi, order) + fp32_sum(lo, order))
            ref = s if ref is None else ref
            assert s.view(np.uint32) == ref.view(np.uint32)
        exact = float(np.sum(v.astype(np.float64)))
        assert abs(float(ref) - exact) <= n * 2.0 ** -26 + abs(exact) * 2.0 ** -24


def test_plain_fp32_sums_do_depend_on_order():
    """The default mode's fp32 sums are not order-independent (why the split exists)."""
    rng = np.random.default_rng(3)
    v = (rng.standard_normal(148) * 0.05).astype(np.float32)
    bits = {fp32_sum(v, rng.permutation(148)).view(np.uint32) for _ in range(50)}
    assert len(bits) > 1
