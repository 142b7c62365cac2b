"""Lookup tables of the nonlinear-function primitive, built from their definitions in
high-precision decimal arithmetic (test infrastructure only: the oracle's own tables).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` use
this module.  The CUDA library builds its own tables and shares nothing with it.

Source: "Memory-Efficient Integer-Only Training of Deep Neural Networks".
  Table 8 (output head, "built once at initialization"):
    LUT_exp[e_x][k] = round(exp(k * 2^e_x) * 2^L),   k in [-255, 0], about 30 exponents, L = 7
    LUT_log[p]      = round(-log(p / 2^B) * 2^Ll),   p in [1, 2^B - 2], Ll = 5 (B = 8: 256 entries)
  Table 7 (GELU): forward LUT_fwd[e, C] (Eq. 19, not printed on the page), backward
    (dY * LUT_bwd[e, C]) >> B_G, both INT8 [30, 256]; the exponent e is carried unchanged.

Readings (the page prints the entry formulas but not the exponent range nor Eq. 19):
  * The 30 exponents are e = -26 .. 3.  Outside that range every table row equals its
    nearest end row (an exponent below -26 gives the -26 row, above 3 the 3 row), so a
    lookup clamps e and is exact for every exponent:
      - LUT_exp: exp(-255 * 2^-26) * 128 > 127.5, so every k rounds to 128 at e <= -26;
        exp(-2^3) * 128 < 0.5, so every k < 0 rounds to 0 at e >= 3.
      - GELU: x * Phi(x) at x = C * 2^e rounds to ceil(C / 2) for e <= -14 and to max(C, 0)
        for e >= -1; the derivative times 2^B_G rounds to 32 for e <= -14 and to
        64 * [C > 0] + 32 * [C = 0] for e >= 2.
  * "round" is round half to even of the exact real value.
  * Eq. 19 is taken as the exact GELU, x * Phi(x) with Phi the standard normal CDF, so
    LUT_fwd[e][C] = round(C * Phi(C * 2^e)); its derivative Phi(x) + x * phi(x) has its
    extremes at x = -/+ sqrt(2) (about -0.129 and 1.129), so B_G = 6 keeps
    LUT_bwd[e][C] = round(GELU'(C * 2^e) * 2^6) within int8 ([-8, 72]; 2^7 would not).
  * Tables are indexed [e - E_LO][k + 255] (LUT_exp), [p] (LUT_log), [e - E_LO][C + 128]
    (GELU; the C = -128 column is defined by the same formula and never read).
"""
from __future__ import annotations

from decimal import ROUND_HALF_EVEN, Decimal, localcontext

import numpy as np

E_LO, E_HI = -26, 3          # the 30 table exponents
N_EXP = E_HI - E_LO + 1
L_EXP, L_LOG, B_PROB, B_G = 7, 5, 8, 6
PREC = 90                    # decimal digits carried through every evaluation


def _rne(q: Decimal) -> int:
    return int(q.to_integral_value(rounding=ROUND_HALF_EVEN))


def _pi() -> Decimal:
    """pi by Machin's formula, 16 arctan(1/5) - 4 arctan(1/239)."""
    def arctan_inv(n: int) -> Decimal:
        x, n2, total, term, k, sign = Decimal(1) / n, n * n, Decimal(0), Decimal(1) / n, 1, 1
        while term != 0:
            total += sign * term / k
            term /= n2
            k += 2
            sign = -sign
        return total

    return 16 * arctan_inv(5) - 4 * arctan_inv(239)


def _erf(z: Decimal, pi: Decimal) -> Decimal:
    """erf by its Maclaurin series, 2/sqrt(pi) sum (-1)^n z^(2n+1) / (n! (2n+1)); |z| <= 8."""
    total, term, n = Decimal(0), z, 0  # term = (-1)^n z^(2n+1) / n!
    while True:
        add = term / (2 * n + 1)
        total += add
        if abs(add) < Decimal(10) ** (-(PREC - 5)):
            break
        n += 1
        term = -term * z * z / n
    return 2 * total / pi.sqrt()


def _phi_cdf(x: Decimal, pi: Decimal) -> Decimal:
    """Standard normal CDF.  For |x| >= 11 it is within 1e-27 of 0 or 1, far inside
    every rounding margin the tables meet, so it is taken as 0 or 1 there."""
    if x >= 11:
        return Decimal(1)
    if x <= -11:
        return Decimal(0)
    return (1 + _erf(x / Decimal(2).sqrt(), pi)) / 2


def lut_exp() -> np.ndarray:
    """uint8 [30][256]: LUT_exp[e - E_LO][k + 255] = round(exp(k 2^e) 2^7)."""
    out = np.zeros((N_EXP, 256), np.uint8)
    with localcontext() as ctx:
        ctx.prec = PREC
        for e in range(E_LO, E_HI + 1):
            s = Decimal(2) ** e
            for k in range(-255, 1):
                out[e - E_LO, k + 255] = _rne((k * s).exp() * (2 ** L_EXP))
    return out


def lut_log() -> np.ndarray:
    """uint8 [256]: LUT_log[p] = round(-log(p / 2^8) 2^5) for p in [1, 254]; the unused
    entries 0 and 255 repeat those of 1 and 254 (a lookup clamps p to [1, 254])."""
    out = np.zeros(256, np.uint8)
    with localcontext() as ctx:
        ctx.prec = PREC
        for p in range(1, 255):
            out[p] = _rne(-(Decimal(p) / (2 ** B_PROB)).ln() * (2 ** L_LOG))
    out[0], out[255] = out[1], out[254]
    return out


def lut_gelu() -> tuple[np.ndarray, np.ndarray]:
    """int8 [30][256] each: forward round(C Phi(C 2^e)) and backward
    round((Phi(x) + x phi(x)) 2^6) at x = C 2^e, indexed [e - E_LO][C + 128]."""
    fwd = np.zeros((N_EXP, 256), np.int8)
    bwd = np.zeros((N_EXP, 256), np.int8)
    with localcontext() as ctx:
        ctx.prec = PREC
        pi = _pi()
        inv_sqrt_2pi = 1 / (2 * pi).sqrt()
        for e in range(E_LO, E_HI + 1):
            s = Decimal(2) ** e
            for c in range(-128, 128):
                x = c * s
                cdf = _phi_cdf(x, pi)
                pdf = (-(x * x) / 2).exp() * inv_sqrt_2pi
                fwd[e - E_LO, c + 128] = _rne(c * cdf)
                bwd[e - E_LO, c + 128] = _rne((cdf + x * pdf) * (2 ** B_G))
    return fwd, bwd


_cache: dict = {}


def tables() -> dict:
    """All four tables, built once per process."""
    if not _cache:
        f, b = lut_gelu()
        _cache.update(exp=lut_exp(), log=lut_log(), gelu_fwd=f, gelu_bwd=b)
    return _cache
