"""Property-based pins of the oracle's core routines (hypothesis): random small shapes,
group geometries, values and exponents, each checked against the brute-force references
of tests/brute.py (unbounded Python integers and Fractions, half-to-even `round`)."""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from integer_only_nn_02_b200.workloads import CE, E_ZERO
from tests.brute import fit_matrix_brute, pow2, value

SETTINGS = settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])


@st.composite
def ce_tensors(draw, rows=None, cols=None):
    rows = rows or draw(st.integers(1, 6))
    cols = cols or draw(st.integers(1, 9))
    g_rows = draw(st.integers(1, rows))
    g_cols = draw(st.integers(1, cols))
    ngr, ngc = -(-rows // g_rows), -(-cols // g_cols)
    m = np.array(draw(st.lists(st.integers(-127, 127), min_size=rows * cols, max_size=rows * cols)),
                 np.int8).reshape(rows, cols)
    e = np.array(draw(st.lists(st.integers(-40, 30), min_size=ngr * ngc, max_size=ngr * ngc)),
                 np.int8).reshape(ngr, ngc)
    for gi in range(ngr):  # some all-zero groups
        for gj in range(ngc):
            if draw(st.integers(0, 9)) == 0:
                e[gi, gj] = E_ZERO
                m[gi * g_rows:(gi + 1) * g_rows, gj * g_cols:(gj + 1) * g_cols] = 0
    return CE(m, e, g_rows, g_cols)


def values(t: CE):
    return [[value(int(t.mant[i, j]), int(t.exp[i // t.g_rows, j // t.g_cols]))
             if t.exp[i // t.g_rows, j // t.g_cols] != E_ZERO else 0 for j in range(t.cols)]
            for i in range(t.rows)]


@SETTINGS
@given(st.data())
def test_requant_is_fit_of_exact_values(data):
    rows, cols = data.draw(st.integers(1, 6)), data.draw(st.integers(1, 9))
    bits = data.draw(st.integers(1, 44))
    x = np.array(data.draw(st.lists(st.integers(-(2 ** bits), 2 ** bits), min_size=rows * cols,
                                    max_size=rows * cols)), np.int64).reshape(rows, cols)
    g = (data.draw(st.integers(1, rows)), data.draw(st.integers(1, cols)))
    base = data.draw(st.integers(-60, 20))
    re = np.array(data.draw(st.lists(st.integers(-20, 20), min_size=rows, max_size=rows)), np.int8)
    out = oracle.requant(x, *g, base_exp=base, row_exp=re)
    mant, exps = fit_matrix_brute([[value(int(x[i, j]), base + int(re[i])) for j in range(cols)]
                                   for i in range(rows)], *g)
    assert out.mant.tolist() == mant and out.exp.tolist() == exps


@SETTINGS
@given(st.data())
def test_sum_is_fit_of_exact_sums(data):
    X = data.draw(ce_tensors())
    Y = data.draw(ce_tensors(X.rows, X.cols))
    g = (data.draw(st.integers(1, X.rows)), data.draw(st.integers(1, X.cols)))
    Z = oracle.sum_(X, Y, *g)
    vx, vy = values(X), values(Y)
    mant, exps = fit_matrix_brute([[vx[i][j] + vy[i][j] for j in range(X.cols)] for i in range(X.rows)], *g)
    assert Z.mant.tolist() == mant and Z.exp.tolist() == exps


@SETTINGS
@given(ce_tensors(), st.sampled_from([0, 1]))
def test_align_max_rounds_to_the_largest_group_exponent(t, axis):
    m, e = oracle.align(t, axis=axis)
    vals = values(t)
    n_keep, n_red = (t.rows, t.cols) if axis == 1 else (t.cols, t.rows)
    for a in range(n_keep):
        idx = [(a, b) if axis == 1 else (b, a) for b in range(n_red)]
        live = [int(t.exp[i // t.g_rows, j // t.g_cols]) for i, j in idx
                if t.exp[i // t.g_rows, j // t.g_cols] != E_ZERO]
        assert int(e[a]) == (max(live) if live else E_ZERO)
        for i, j in idx:
            assert int(m[i, j]) == (round(vals[i][j] / pow2(int(e[a]))) if live else 0)


@SETTINGS
@given(ce_tensors(), st.booleans())
def test_relu_keeps_exponents_and_sign(t, six):
    z = oracle.relu_fwd(t, six)
    assert (z.exp == t.exp).all()
    assert (z.mant >= 0).all() and (z.mant <= np.maximum(t.mant, 0)).all()
    if not six:
        assert (z.mant == np.maximum(t.mant, 0)).all()


@SETTINGS
@given(st.data())
def test_sum_scaled_is_fit_of_weighted_exact_sums(data):
    from fractions import Fraction

    X = data.draw(ce_tensors())
    Y = data.draw(ce_tensors(X.rows, X.cols))
    xw = (data.draw(st.integers(-512, 512)), data.draw(st.integers(0, 24)))
    yw = (data.draw(st.integers(-512, 512)), data.draw(st.integers(0, 24)))
    g = (data.draw(st.integers(1, X.rows)), data.draw(st.integers(1, X.cols)))
    Z = oracle.sum_scaled(X, xw, Y, yw, *g)
    vx, vy = values(X), values(Y)
    wx, wy = Fraction(xw[0]) * pow2(-xw[1]), Fraction(yw[0]) * pow2(-yw[1])
    mant, exps = fit_matrix_brute([[wx * vx[i][j] + wy * vy[i][j] for j in range(X.cols)]
                                   for i in range(X.rows)], *g)
    assert Z.mant.tolist() == mant and Z.exp.tolist() == exps


@SETTINGS
@given(st.data())
def test_avgpool_is_fit_of_exact_window_means(data):
    from fractions import Fraction

    K = data.draw(st.integers(1, 4))
    n, hp, wp, c = data.draw(st.integers(1, 2)), data.draw(st.integers(1, 3)), data.draw(st.integers(1, 3)), 4
    h, w = hp * K, wp * K
    npix = n * h * w
    g_in = data.draw(st.sampled_from([1, 2, 4]))  # channel groups spanning all pixels
    m = np.array(data.draw(st.lists(st.integers(-127, 127), min_size=npix * c, max_size=npix * c)),
                 np.int8).reshape(npix, c)
    e = np.array([data.draw(st.sampled_from([E_ZERO] + list(range(-30, 20)))) for _ in range(c // g_in)],
                 np.int8).reshape(1, -1)
    for gj in range(e.shape[1]):  # E_ZERO groups hold zeros only
        if e[0, gj] == E_ZERO:
            m[:, gj * g_in:(gj + 1) * g_in] = 0
    X = CE(m, e, npix, g_in)
    og = (data.draw(st.integers(1, n * hp * wp)), data.draw(st.sampled_from([1, 2, 4])))
    Y = oracle.avgpool_fwd(X, n, h, w, K, *og)
    vx = values(X)
    vals = [[sum((vx[(img * h + p * K + dy) * w + q * K + dx][ch] for dy in range(K) for dx in range(K)),
                 Fraction(0)) / (K * K) for ch in range(c)]
            for img in range(n) for p in range(hp) for q in range(wp)]
    mant, exps = fit_matrix_brute(vals, *og)
    assert Y.mant.tolist() == mant and Y.exp.tolist() == exps
