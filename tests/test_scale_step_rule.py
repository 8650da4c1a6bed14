"""The write kernels settle the quantization step s with fp32 arithmetic only:
a candidate RU16(RU(RU(max - z) * RU(1/top))) and an exact test of the
step below, top * s >= RU(max - z). This checks that rule against exact
rational arithmetic on random and adversarial ranges (top = 15 for INT4,
3 for INT2): the rule must give the smallest fp16 s with top * s + z >= max,
and the oracle's binary16 search must give the same s."""
from fractions import Fraction

import numpy as np
import pytest

import oracle


def _f32(x):
    return np.float32(x)


def _ru32(exact):
    """Smallest fp32 >= the exact rational (no overflow in these ranges)."""
    f = np.float32(float(exact))
    while Fraction(float(f)) < exact:
        f = np.nextafter(f, np.float32(np.inf))
    while True:
        lower = np.nextafter(f, np.float32(-np.inf))
        if Fraction(float(lower)) >= exact:
            f = lower
        else:
            return f


def _half_ru(x32):
    """Smallest fp16 >= x (x finite, within range)."""
    h = np.float16(x32)
    if float(h) < float(x32):
        h = np.nextafter(h, np.float16(np.inf))
    return h


def _kernel_rule(mn, mx, top):
    z = np.float16(mn)
    if float(z) > float(mn):
        z = np.nextafter(z, np.float16(-np.inf))
    zf = Fraction(float(z))
    d = _ru32(Fraction(float(mx)) - zf)                       # RU(mx - z)
    c = _ru32(Fraction(1, top))                               # RU(1/top)
    need = _ru32(Fraction(float(d)) * Fraction(float(c)))     # RU(d * c)
    s = _half_ru(need)
    bits = int(s.view(np.uint16))
    if 0 < bits < 0x7C00:
        pb = np.uint16(bits - 1).view(np.float16)
        # top * pb is exact in fp32; compare with RU(mx - z)
        if float(np.float32(top) * np.float32(pb)) >= float(d):
            bits -= 1
    return bits, int(z.view(np.uint16))


def _exact_rule(mn, mx, top):
    z = np.float16(mn)
    if float(z) > float(mn):
        z = np.nextafter(z, np.float16(-np.inf))
    zf, m = Fraction(float(z)), Fraction(float(mx))

    def covers(bits):  # non-negative fp16 patterns are ordered like their values
        return top * Fraction(float(np.uint16(bits).view(np.float16))) + zf >= m

    lo, hi = 0, 0x7C00  # the answer is the first pattern in [lo, hi] that covers
    if not covers(0x7BFF):
        return 0x7C00, int(z.view(np.uint16))
    while lo < hi:
        mid = (lo + hi) // 2
        if covers(mid):
            hi = mid
        else:
            lo = mid + 1
    return lo, int(z.view(np.uint16))


def _cases(seed, n):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        a, b = np.sort(rng.standard_normal(2) * 10.0 ** rng.integers(-4, 4))
        out.append((_f32(a), _f32(b)))
    # adversarial: max exactly on a step boundary, a zero range, tiny ranges
    for top in (3, 15):
        for k in range(1, 40):
            z = float(np.float16(-k * 0.37))
            s = float(np.float16(0.01 * k))
            out.append((_f32(z), _f32(top * s + z)))
            out.append((_f32(z), _f32(np.nextafter(np.float32(top * s + z), np.float32(np.inf)))))
    out.append((_f32(1.5), _f32(1.5)))
    out.append((_f32(-2.0 ** -20), _f32(2.0 ** -20)))
    return out


@pytest.mark.parametrize("top", [3, 15])
def test_fp32_step_rule_is_exact(top):
    cases = _cases(11 + top, 150)
    for mn, mx in cases:
        got = _kernel_rule(mn, mx, top)
        assert got == _exact_rule(mn, mx, top), (mn, mx, top)
        assert got == oracle.scale_zero_levels(mn, mx, top), (mn, mx, top)
