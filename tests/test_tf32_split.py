"""The error bound that include/fp.h states for the map's tensor-core logits,
checked on the split itself (numpy, no GPU): with x = hi + lo, hi = x with
its low 13 mantissa bits cleared and lo = x - hi, the products
hi.hi + hi.lo + lo.hi -- lo entering the tensor core as tf32, by truncation
or by rounding -- differ from the exact dot product by at most 2^-19 of
sum_k |x_k y_k| (before the fp32 accumulation, whose own rounding is far
smaller at d <= 128)."""
import numpy as np
import pytest


def tf32_trunc(a):
    return (a.astype(np.float32).view(np.uint32) & np.uint32(0xFFFFE000)).view(np.float32)


def tf32_round(a):
    # round to nearest even on the 10-bit tf32 mantissa
    u = a.astype(np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 13) & 1
    u = (u + 0xFFF + lsb) & 0xFFFFE000
    return u.astype(np.uint32).view(np.float32)


@pytest.mark.parametrize("to_tf32", [tf32_trunc, tf32_round])
@pytest.mark.parametrize("d", [64, 128])
def test_three_product_split_error_bound(to_tf32, d):
    rng = np.random.default_rng(d)
    worst = 0.0
    for trial in range(400):
        scale = 2.0 ** rng.integers(-20, 20)
        x = (rng.standard_normal(d) * scale * np.exp(rng.standard_normal(d))).astype(np.float32)
        y = (rng.standard_normal(d) / scale * np.exp(rng.standard_normal(d))).astype(np.float32)
        xh, yh = tf32_trunc(x), tf32_trunc(y)
        xl = (x - xh).astype(np.float32)  # exact in fp32
        yl = (y - yh).astype(np.float32)
        assert np.array_equal(xh.astype(np.float64) + xl, x.astype(np.float64))
        xlt, ylt = to_tf32(xl).astype(np.float64), to_tf32(yl).astype(np.float64)
        xh64, yh64 = xh.astype(np.float64), yh.astype(np.float64)
        got = np.sum(xh64 * yh64 + xh64 * ylt + xlt * yh64)
        exact = np.dot(x.astype(np.float64), y.astype(np.float64))
        ref = np.sum(np.abs(x.astype(np.float64) * y.astype(np.float64)))
        worst = max(worst, abs(got - exact) / ref)
    assert worst <= 2.0 ** -19, worst
    # and the split is not exact: the bound is not vacuous
    assert worst > 2.0 ** -30
