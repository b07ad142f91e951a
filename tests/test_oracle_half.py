"""The reference for the FP16 storage of the SH coefficients is IEEE 754 binary16
rounding to nearest, ties to even (numpy's float16 conversion, used by the GPU
tests as the expected value of gs_to_half and to build the rounded scenes the
oracle projects).  Pinned here against bit patterns that follow from the binary16
format itself: 1 sign, 5 exponent (bias 15) and 10 fraction bits."""
import numpy as np
import pytest


def bits(x):
    with np.errstate(over="ignore"):  # 65520 rounds to infinity, as binary16 defines
        return int(np.float32(x).astype(np.float16).view(np.uint16))


def value(b):
    """binary16 bit pattern -> exact value, from the format's definition."""
    s = -1.0 if b >> 15 else 1.0
    e = (b >> 10) & 0x1f
    f = b & 0x3ff
    if e == 0:
        return s * f * 2.0 ** -24
    if e == 31:
        return s * float("inf") if f == 0 else float("nan")
    return s * (1 + f / 1024.0) * 2.0 ** (e - 15)


@pytest.mark.parametrize("x,want", [
    (1.0, 0x3C00),
    (-2.0, 0xC000),
    (0.0, 0x0000),
    (-0.0, 0x8000),
    (65504.0, 0x7BFF),                     # largest finite half
    (65519.99, 0x7BFF),                    # below the midpoint to the next binade
    (65520.0, 0x7C00),                     # the midpoint rounds to infinity (even)
    (2.0 ** -24, 0x0001),                  # smallest subnormal
    (2.0 ** -25, 0x0000),                  # half of it: a tie, to the even 0
    (3 * 2.0 ** -26, 0x0001),              # 0.75 of it rounds up
    (2.0 ** -14, 0x0400),                  # smallest normal
    (1 + 2.0 ** -11, 0x3C00),              # tie between 0x3C00 and 0x3C01: even
    (1 + 3 * 2.0 ** -11, 0x3C02),          # tie between 0x3C01 and 0x3C02: even
    (1 + 2.0 ** -11 + 2.0 ** -20, 0x3C01),  # just above the tie
])
def test_binary16_rounding_bit_patterns(x, want):
    assert bits(x) == want


def test_rounding_is_to_the_nearest_representable_value():
    """Brute force over every finite positive half: values between two neighbours
    round to the nearer one, and an exact midpoint to the one with an even pattern."""
    pats = np.arange(0, 0x7C00, dtype=np.uint32)
    vals = np.array([value(int(b)) for b in pats])
    assert np.array_equal(np.float16(vals).view(np.uint16), pats.astype(np.uint16))  # exact values map to themselves
    lo, hi = vals[:-1], vals[1:]
    mid = (lo + hi) / 2      # exact in double
    q = (3 * lo + hi) / 4    # strictly below the midpoint
    r = (lo + 3 * hi) / 4    # strictly above
    keep = np.float32(q) == q  # only points float32 holds exactly
    assert np.array_equal(np.float32(q[keep]).astype(np.float16).view(np.uint16), pats[:-1][keep].astype(np.uint16))
    keep = np.float32(r) == r
    assert np.array_equal(np.float32(r[keep]).astype(np.float16).view(np.uint16), pats[1:][keep].astype(np.uint16))
    keep = np.float32(mid) == mid
    got = np.float32(mid[keep]).astype(np.float16).view(np.uint16)
    even = np.where(pats[:-1][keep] % 2 == 0, pats[:-1][keep], pats[1:][keep]).astype(np.uint16)
    assert np.array_equal(got, even)
