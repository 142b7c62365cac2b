"""Pins of the oracle's lookup-table nonlinearities ("Memory-Efficient Integer-Only
Training of Deep Neural Networks", Table 7: GELU through LUT_fwd / LUT_bwd; Table 8:
the output head's LUT_exp and LUT_log), each against something other than the oracle:

* every table entry against the same formula evaluated with the C library's double-
  precision exp / log / erf (an independent implementation of the functions), with a
  check that no entry lies close enough to a rounding tie for double precision to be in
  doubt;
* closed forms: exp(0) = 1, log 2, the rows where GELU is ReLU or x / 2, GELU'(0) = 1/2;
* the head: a uniform row (p = 256 / K exactly rounded), a confident row (p clamps to
  254, zero loss, zero gradient), and random rows whose loss lies within the error the
  three roundings (LUT_exp, the quotient, LUT_log) allow around the float64 cross-
  entropy;
* GELU: forward within half a unit of the float64 GELU, backward within the rounding
  of LUT_bwd plus the FIT of the product.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import luts
from integer_only_nn_02_b200.workloads import CE, with_groups
from tests.test_oracle_pins import rand_ce

E_LO, E_HI = luts.E_LO, luts.E_HI


@pytest.fixture(scope="module")
def T():
    return luts.tables()


def _rne_checked(v: float):
    """Round half to even of a double, and whether it is safely away from a tie."""
    f = math.floor(v)
    frac = v - f
    return round(v), abs(frac - 0.5) > 1e-9


def phi(x):
    return 0.5 * (1.0 + math.erf(x / math.sqrt(2.0)))


def dphi(x):
    return math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def test_lut_exp_matches_double_precision(T):
    for e in range(E_LO, E_HI + 1):
        for k in range(-255, 1):
            want, safe = _rne_checked(math.exp(k * 2.0 ** e) * 128.0)
            assert safe, (e, k)
            assert T["exp"][e - E_LO, k + 255] == want, (e, k)


def test_lut_log_matches_double_precision(T):
    for p in range(1, 255):
        want, safe = _rne_checked(-math.log(p / 256.0) * 32.0)
        assert safe, p
        assert T["log"][p] == want, p


def test_lut_gelu_matches_double_precision(T):
    for e in range(E_LO, E_HI + 1):
        for c in range(-127, 128):
            x = c * 2.0 ** e
            f, sf = _rne_checked(c * phi(x))
            b, sb = _rne_checked((phi(x) + x * dphi(x)) * 64.0)
            assert (sf or c == 0) and sb, (e, c)
            assert T["gelu_fwd"][e - E_LO, c + 128] == f, (e, c)
            assert T["gelu_bwd"][e - E_LO, c + 128] == b, (e, c)


def test_lut_closed_forms(T):
    ex, lg, gf, gb = T["exp"], T["log"], T["gelu_fwd"], T["gelu_bwd"]
    assert (ex[:, 255] == 128).all()                      # exp(0) 2^7
    assert (ex[E_HI - E_LO, :255] == 0).all()             # exp(-8 |k|) 2^7 < 1/2
    assert (ex[0] == 128).all()                           # exp(-255 2^-26) 2^7 > 127.5
    assert (np.diff(ex.astype(int), axis=1) >= 0).all()   # non-decreasing in k
    assert lg[128] == 22 and lg[64] == 44 and lg[1] == 177  # 32 ln 2 = 22.18, 64 ln 2, 256 ln 2
    assert (np.diff(lg[1:255].astype(int)) <= 0).all()
    cs = np.arange(-127, 128)
    for e in range(-1, E_HI + 1):                         # GELU rounds to ReLU
        assert (gf[e - E_LO, cs + 128] == np.maximum(cs, 0)).all(), e
    for e in range(E_LO, -13):                            # GELU rounds to ceil(C / 2)
        assert (gf[e - E_LO, cs + 128] == -((-cs) // 2)).all(), e
        assert (gb[e - E_LO, cs + 128] == 32).all(), e
    assert (gb[:, 128] == 32).all()                       # GELU'(0) = 1/2
    for e in range(2, E_HI + 1):
        assert (gb[e - E_LO, cs + 128] == np.where(cs > 0, 64, np.where(cs == 0, 32, 0))).all()
    assert gb.min() == -8 and gb.max() == 72


def test_head_uniform_and_confident_rows(T):
    for K in (2, 3, 10, 100, 1000):
        Z = CE(np.full((2, K), 5, np.int8), np.array([[-3], [4]], np.int8), 1, K)
        loss, dZ = oracle.softmax_ce(Z, np.array([0, K - 1]))
        p = round(Fraction(256, K))                       # every E is 128
        assert (loss == T["log"][min(max(p, 1), 254)]).all(), K
        g = np.full(K, p) - 256 * (np.arange(K) == 0)
        got = dZ.mant[0].astype(int) * 2.0 ** int(dZ.exp[0, 0])
        assert np.allclose(got, g * 2.0 ** -8, atol=2.0 ** (int(dZ.exp[0, 0]) - 1)), K
    # confident: target at +127, the rest at -127, exponent 0 -> every other E is 0
    Z = CE(np.full((1, 10), -127, np.int8), np.zeros((1, 1), np.int8), 1, 10)
    Z.mant[0, 4] = 127
    loss, dZ = oracle.softmax_ce(Z, np.array([4]))
    assert loss[0] == T["log"][254] == 0
    assert (dZ.mant == 0).all() and dZ.exp[0, 0] == -128


def test_head_within_rounding_of_float_cross_entropy(T):
    rng = np.random.default_rng(3)
    for K, e in ((10, -4), (100, -5), (1000, -6), (37, -3)):
        Z = rand_ce(rng, 64, K, 1, K, elo=e, ehi=e)
        tgt = rng.integers(0, K, size=64)
        loss, _ = oracle.softmax_ce(Z, tgt)
        for i in range(64):
            z = Z.mant[i].astype(float) * 2.0 ** e
            zmax = z.max()
            E = np.exp(z - zmax) * 128.0
            S = E.sum()
            # E_t within 1/2, S within K/2, the quotient within 1/2, the log within 1/2
            p_lo = max(256.0 * (E[tgt[i]] - 0.5) / (S + 0.5 * K) - 0.5, 1.0)
            p_hi = min(256.0 * (E[tgt[i]] + 0.5) / max(S - 0.5 * K, 1e-9) + 0.5, 254.0)
            p_lo, p_hi = min(p_lo, 254.0), max(p_hi, 1.0)
            lo = -math.log(p_hi / 256.0) * 32.0 - 0.5
            hi = -math.log(p_lo / 256.0) * 32.0 + 0.5
            assert lo - 1e-9 <= loss[i] <= hi + 1e-9, (K, i, loss[i], lo, hi)


def test_head_gradient_is_p_minus_onehot(T):
    """The gradient's values equal (p - 256 [j = t]) 2^-8 to within the FIT of its row,
    with p the head's own rounded probabilities; its sum over the row is about 0."""
    rng = np.random.default_rng(4)
    Z = rand_ce(rng, 32, 50, 1, 25, elo=-6, ehi=-4)    # two exponent groups per row: aligned first
    tgt = rng.integers(0, 50, size=32)
    loss, dZ = oracle.softmax_ce(Z, tgt, 1, 50)
    ex = T["exp"]
    for i in range(32):
        es = int(Z.exp[i].max())
        c = np.array([round(Fraction(int(Z.mant[i, j])) * Fraction(2) ** (int(Z.exp[i, j // 25]) - es))
                      for j in range(50)])
        E = ex[min(max(es, E_LO), E_HI) - E_LO, c - c.max() + 255].astype(int)
        p = np.array([round(Fraction(256 * int(v), int(E.sum()))) for v in E])
        g = p - 256 * (np.arange(50) == tgt[i])
        got = dZ.mant[i].astype(int) * 2.0 ** int(dZ.exp[i, 0])
        assert np.abs(got - g * 2.0 ** -8).max() <= 2.0 ** (int(dZ.exp[i, 0]) - 1)
        assert abs(int(p.sum()) - 256) <= 25
        assert loss[i] == T["log"][min(max(int(p[tgt[i]]), 1), 254)]


def test_gelu_lut_forward_within_half_unit_of_gelu():
    rng = np.random.default_rng(5)
    H = rand_ce(rng, 40, 64, 1, 32, elo=-30, ehi=6, zero_groups=0.1)
    out = oracle.gelu_lut_fwd(H)
    assert (out.exp == H.exp).all()
    for i in range(40):
        for j in range(64):
            e = int(H.exp[i, j // 32])
            if e == -128:
                assert out.mant[i, j] == 0
                continue
            x = int(H.mant[i, j]) * 2.0 ** e
            assert abs(int(out.mant[i, j]) * 2.0 ** e - x * phi(x)) <= 2.0 ** (e - 1) * (1 + 1e-9), (i, j)


def test_gelu_lut_backward_within_rounding():
    rng = np.random.default_rng(6)
    H = rand_ce(rng, 24, 64, 1, 32, elo=-8, ehi=-3, zero_groups=0.1)
    dY = rand_ce(rng, 24, 64, 1, 32, elo=-14, ehi=-10, zero_groups=0.1)
    dH = oracle.gelu_lut_bwd(H, dY, 1, 32)
    for i in range(24):
        for j in range(64):
            eh, ed, eo = int(H.exp[i, j // 32]), int(dY.exp[i, j // 32]), int(dH.exp[i, j // 32])
            x = 0.0 if eh == -128 else int(H.mant[i, j]) * 2.0 ** eh
            dy = 0.0 if ed == -128 else int(dY.mant[i, j]) * 2.0 ** ed
            want = dy * (phi(x) + x * dphi(x))
            got = 0.0 if eo == -128 else int(dH.mant[i, j]) * 2.0 ** eo
            # LUT_bwd rounds the slope to 2^-7, FIT rounds the product to half its unit
            tol = abs(dy) * 2.0 ** -7 + (0.0 if eo == -128 else 2.0 ** (eo - 1)) + 1e-30
            assert abs(got - want) <= tol * (1 + 1e-9), (i, j, got, want)
