"""The rounding facts the convolution's all-pixel-group path rests on, checked by brute
force with Python integers and Fractions (no GPU, no oracle).

A convolution whose output channel groups span every pixel cannot round a tile before
the group exponent over the whole batch is known.  Its Product pass therefore stores
each exact sum x (at exponent r) rounded to odd at a finer exponent e1 = n_tile - 7,
where n_tile is the tile's largest need(), and a streaming pass rounds that to nearest
even at the group exponent e >= n_tile.  Two facts make this exact:

1. Rounding to odd at a grid 2^-k finer than the target (k >= 2), then to nearest even,
   equals rounding the exact value to nearest even (Boldo and Melquiond, "Emulation of
   FMA and correctly rounded sums: proved algorithms using rounding to odd", IEEE
   Trans. Computers 57(4), 2008).  With k = 1 it does not hold.
2. The intermediate fits int16: |RO(x * 2^(r - e1))| <= 127.5 * 2^7 < 2^15 whenever
   need(x, r) <= n_tile.
"""
from fractions import Fraction

import numpy as np


def rne(q: Fraction) -> int:
    return round(q)  # Python rounds halves to even


def ro_shift(x: int, s: int) -> int:
    """Round x * 2^-s to odd the way the kernel does: floor, then the sticky bit ORed in."""
    if s <= 0:
        return x << -s
    return (x >> s) | (1 if x & ((1 << s) - 1) else 0)


def ro_exact(q: Fraction) -> int:
    """Round to odd by its definition: q itself if integral, else the odd neighbour."""
    f = q.numerator // q.denominator
    if f == q:
        return f
    return f if f % 2 else f + 1


def need(x: int, r: int) -> int:
    """Smallest exponent e with |RNE(x * 2^(r - e))| <= 127 (x != 0)."""
    e = r - 10
    while abs(rne(Fraction(x) * Fraction(2) ** (r - e))) > 127:
        e += 1
    return e


def test_round_to_odd_by_floor_and_sticky():
    for x in range(-600, 601):
        for s in range(0, 12):
            assert ro_shift(x, s) == ro_exact(Fraction(x, 2 ** s)), (x, s)


def test_round_to_odd_then_nearest_is_nearest():
    rng = np.random.default_rng(0)
    xs = list(range(-5000, 5001)) + [int(v) for v in rng.integers(-(2 ** 30), 2 ** 30, size=3000)]
    for x in xs:
        for s1 in range(0, 14, 3):
            for s2 in range(2, 10):
                assert rne(Fraction(ro_shift(x, s1), 2 ** s2)) == rne(Fraction(x, 2 ** (s1 + s2))), (x, s1, s2)


def test_one_extra_bit_is_not_enough():
    bad = [x for x in range(-64, 65) if rne(Fraction(ro_shift(x, 1), 2)) != rne(Fraction(x, 4))]
    assert bad, "with k = 1 the double rounding differs for some x"


def test_intermediate_fits_int16():
    rng = np.random.default_rng(1)
    for _ in range(4000):
        r = int(rng.integers(-30, 10))
        xs = rng.integers(-(2 ** int(rng.integers(1, 31))), 2 ** int(rng.integers(1, 31)), size=6)
        xs = [int(v) for v in xs if v]
        if not xs:
            continue
        n_tile = max(need(x, r) for x in xs) + int(rng.integers(0, 3))  # any exponent at or above
        e1 = n_tile - 7
        for x in xs:
            t = ro_shift(x, e1 - r)
            assert abs(t) < 2 ** 15 and abs(t) <= 16321, (x, r, n_tile, t)
            # and the final rounding at any group exponent e >= n_tile is exact
            for e in (n_tile, n_tile + 1, n_tile + 5):
                assert rne(Fraction(t) * Fraction(2) ** (e1 - e)) == rne(Fraction(x) * Fraction(2) ** (r - e))
