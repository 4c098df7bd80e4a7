"""Pin for the FP8 write's division (CPU): the kernel computes x / scale as
y = RN(1 / scale), q = RN(x y), then q = RN(q + RN(x - q scale) y), the last
two steps as FMAs (Markstein, IBM J. Res. Dev. 34(1), 1990).  Here that
sequence runs in exact rational arithmetic, each step rounded to float32 by
hand, for every bf16 mantissa of x against every bf16 mantissa of the row
amax (scale = RN(amax / 448)), at quotients from 2^-3 to 448 (exponents
beyond shift every quantity alike): it must equal RN(x / scale) in every
case, while the uncorrected product RN(x y) must not."""
from fractions import Fraction as F

import numpy as np


def _rn32(v: F) -> F:
    """Nearest float32 (ties to even) of a rational in the normal range."""
    if v == 0:
        return F(0)
    sign = -1 if v < 0 else 1
    v = abs(v)
    e = v.numerator.bit_length() - v.denominator.bit_length()
    while v >= F(2) ** (e + 1):
        e += 1
    while v < F(2) ** e:
        e -= 1
    scaled = v * F(2) ** (23 - e)
    m, rem = divmod(scaled.numerator, scaled.denominator)
    rem = F(rem, scaled.denominator)
    if rem > F(1, 2) or (rem == F(1, 2) and m % 2 == 1):
        m += 1
    return sign * F(m) * F(2) ** (e - 23)


def test_rn32_matches_numpy_float32_rounding():
    rng = np.random.default_rng(5)
    for v in rng.standard_normal(2000) * 10.0 ** rng.integers(-6, 6, 2000):
        assert float(_rn32(F(float(v)))) == float(np.float32(v))


def _cases(step):
    for ma in range(0, 128, step):
        a = F(128 + ma, 128)
        s = _rn32(a / 448)
        y = _rn32(1 / s)
        for ex in (-11, -5, 0):       # x / amax in about 2^-11 .. 1: quotients 2^-3 .. 448
            for mx in range(128):
                x = F(128 + mx, 128) * F(2) ** ex
                if x <= a:
                    yield x, s, y


def test_one_fma_correction_gives_the_correctly_rounded_quotient():
    n = 0
    for x, s, y in _cases(1):
        q = _rn32(x * y)
        q = _rn32(q + _rn32(x - q * s) * y)
        assert q == _rn32(x / s), (float(x), float(s))
        n += 1
    assert n > 40000


def test_the_uncorrected_product_is_not_enough():
    off = sum(_rn32(x * y) != _rn32(x / s) for x, s, y in _cases(1))
    assert off > 0
