"""The rotary kernel's per-head scale amax / 448 by constant reciprocal refinement.

The kernel forms RN(amax / 7) as q = RN(amax * RN(1/7)), r = fma(-q, 7, amax),
q' = RN(r * RN(1/7) + q), then multiplies by 2^-6 (448 = 7 * 64, exact).
Markstein's theorem makes q' correctly rounded when q is faithful; this test
checks it outright for every mantissa of one binade. Powers of two scale every
intermediate exactly while all stay normal, which holds for amax in
[2^-60, 2^100], the range where the kernel takes this path (outside it the
kernel divides with IEEE division).
"""
import numpy as np


def test_divide_by_7_refinement_every_mantissa():
    r7 = np.float32(1) / np.float32(7)
    assert r7 == np.float32(0.142857149)          # the constant in the kernel
    for lo in range(2**23, 2**24, 2**21):
        m = np.arange(lo, lo + 2**21, dtype=np.int64)
        a = m.astype(np.float32).astype(np.float64)           # exact
        q = (a * np.float64(r7)).astype(np.float32).astype(np.float64)
        r = a - q * 7.0                                       # exact in fp64
        assert np.all(r.astype(np.float32).astype(np.float64) == r)   # and in fp32
        s = r * np.float64(r7) + q                            # the fma's exact sum, rounded to fp64
        s32 = s.astype(np.float32)
        # no fp64 sum sits on an fp32 midpoint, so rounding twice equals rounding once
        up = np.nextafter(s32, np.float32(np.inf)).astype(np.float64)
        dn = np.nextafter(s32, np.float32(0)).astype(np.float64)
        s32d = s32.astype(np.float64)
        assert not np.any((s == (s32d + up) / 2) | (s == (s32d + dn) / 2))
        # m / 7 has a period-3 binary expansion, so it is never an fp32 midpoint either
        exact = (m.astype(np.float64) / 7.0).astype(np.float32)
        assert np.array_equal(s32, exact)
