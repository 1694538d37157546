"""The fp32 identities the 8-bit extend kernel's softmax relies on, checked on the host.

The kernel takes the row maximum of the scaled scores on the int32 dots and converts only
the extreme dot of each page half, and it turns a dot into fp32 by an integer add to the
bits of 1.5 * 2^23 followed by a float subtraction.  Both are exact claims about IEEE fp32
round-to-nearest-even arithmetic; these tests evaluate them in numpy float32 (the same
rounding) over dots of the largest magnitude the kernel sees, 128 * 128 * 128 = 2^21.
"""
import numpy as np
import pytest

DOT_MAX = 128 * 128 * 128          # |Q8 . K8| over D = 128 with int8 codes in [-128, 127]
BIAS_BITS = 0x4B400000             # the bits of 1.5 * 2^23
BIAS = np.float32(12582912.0)


def _dots(rng, n):
    d = rng.integers(-DOT_MAX, DOT_MAX + 1, size=n, dtype=np.int64)
    return np.concatenate([d, [DOT_MAX, -DOT_MAX, 0, 1, -1, DOT_MAX - 1, -(DOT_MAX - 1)]]).astype(np.int32)


def test_bias_add_conversion_is_exact():
    rng = np.random.default_rng(7)
    v = _dots(rng, 200_000)
    bits = (v.astype(np.int64) + BIAS_BITS).astype(np.uint32)
    u = bits.view(np.float32)
    got = u - BIAS                                     # one float32 subtraction
    assert got.dtype == np.float32
    np.testing.assert_array_equal(got, v.astype(np.float32))
    # and the float32 of every dot is the dot itself (|dot| < 2^24)
    np.testing.assert_array_equal(v.astype(np.float32).astype(np.int64), v.astype(np.int64))


@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_row_max_of_scaled_dots_from_the_extreme_dot(sign):
    """max_j fp32(sc * fp32(x_j)) == fp32(sc * fp32(max x)) for sc >= 0 (min x for sc < 0)."""
    rng = np.random.default_rng(11 if sign > 0 else 12)
    for _ in range(2000):
        n = int(rng.integers(1, 65))
        x = _dots(rng, n)[:n]
        sc = np.float32(sign * np.exp(rng.uniform(-30.0, 5.0)))   # products of two quantisation scales
        per_key = np.max(sc * x.astype(np.float32))              # float32 products, then the max
        ext = x.max() if sc >= 0 else x.min()
        assert np.float32(sc * np.float32(ext)) == per_key
    # scale zero: every product is zero
    x = _dots(rng, 64)[:64]
    assert np.max(np.float32(0.0) * x.astype(np.float32)) == np.float32(0.0) * np.float32(x.max())


def test_exponent_with_448_folded_in():
    """2^(t + log2 448) stays within 2^-20 (relative) of 448 * 2^t over the range P8 can hold."""
    t = np.linspace(-16.0, 0.0, 4001, dtype=np.float32)       # 448 * 2^-16 is below E4M3's smallest code
    folded = np.exp2((t + np.float32(np.log2(448.0))).astype(np.float32).astype(np.float64))
    direct = 448.0 * np.exp2(t.astype(np.float64))
    assert np.max(np.abs(folded - direct) / direct) < 2.0 ** -20
