"""Brute-force references written with Python's unbounded integers and Fractions.

These are independent of the oracle's C code: rounding is Python's built-in
``round`` on a Fraction (round half to even), and the group exponent is found by
scanning exponents upward from one at which nothing fits.  Only tiny inputs are
fed to them.
"""
from fractions import Fraction

E_ZERO = -128


def pow2(e: int) -> Fraction:
    return Fraction(2) ** e


def value(c: int, e: int) -> Fraction:
    return Fraction(c) * pow2(e)


def fits(v: Fraction, e: int, qmax: int = 127) -> bool:
    return abs(round(v / pow2(e))) <= qmax


def fit_brute(values, qmax: int = 127):
    """Group exponent and mantissas for exact rational values (scan from below)."""
    nz = [v for v in values if v != 0]
    if not nz:
        return [0] * len(values), E_ZERO
    m = max(abs(v) for v in nz)
    e = m.numerator.bit_length() - m.denominator.bit_length() - 12  # m / 2^e >= 2^10
    while not all(fits(v, e, qmax) for v in nz):
        e += 1
    e = max(e, -127)
    return [round(v / pow2(e)) for v in values], e


def groups_of(rows, cols, g_rows, g_cols):
    """Yield (gi, gj, [(i, j), ...]) for every group of a rows x cols grid."""
    for gi in range(-(-rows // g_rows)):
        for gj in range(-(-cols // g_cols)):
            cells = [(i, j)
                     for i in range(gi * g_rows, min(rows, (gi + 1) * g_rows))
                     for j in range(gj * g_cols, min(cols, (gj + 1) * g_cols))]
            yield gi, gj, cells


def fit_matrix_brute(vals, g_rows, g_cols, qmax: int = 127):
    """vals: 2-D list of Fractions -> (mant 2-D list, exp grid 2-D list)."""
    rows, cols = len(vals), len(vals[0]) if vals else 0
    mant = [[0] * cols for _ in range(rows)]
    ng_r, ng_c = -(-rows // g_rows), -(-cols // g_cols)
    exps = [[E_ZERO] * ng_c for _ in range(ng_r)]
    for gi, gj, cells in groups_of(rows, cols, g_rows, g_cols):
        c, e = fit_brute([vals[i][j] for i, j in cells], qmax)
        exps[gi][gj] = e
        for (i, j), cc in zip(cells, c):
            mant[i][j] = cc
    return mant, exps
