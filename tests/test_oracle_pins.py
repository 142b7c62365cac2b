"""Pins for the CPU oracle against things other than itself.

Each test checks the oracle (oracle/ict_oracle.c) against one of: hand-derived
fixtures (tests/golden), brute force with unbounded Python integers and Python's own
half-to-even ``round`` (tests/brute.py), a library primitive (numpy matmul, torch
float64 convolution on exact small integers), or a closed form.  Sized so that the
whole file runs in well under a minute on CPU.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from integer_only_nn_02_b200.workloads import CE, E_ZERO, cdiv, with_groups
from tests.brute import fit_brute, fit_matrix_brute, groups_of, pow2, value

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def ce_from(d, g):
    return CE(np.array(d["mant"], np.int8), np.array(d["exp"], np.int8), g[0], g[1])


def rand_ce(rng, rows, cols, g_rows, g_cols, elo=-12, ehi=-2, zero_groups=0.0, mag=127):
    m = rng.integers(-mag, mag + 1, size=(rows, cols)).astype(np.int8)
    t = with_groups(m, g_rows, g_cols, lambda g: rng.integers(elo, ehi + 1, size=g))
    if zero_groups:
        for gi, gj, cells in groups_of(rows, cols, t.g_rows, t.g_cols):
            if rng.random() < zero_groups:
                t.exp[gi, gj] = E_ZERO
                for i, j in cells:
                    t.mant[i, j] = 0
    return t


def ce_values(t: CE):
    return [[value(int(t.mant[i, j]), int(t.exp[i // t.g_rows, j // t.g_cols]))
             if t.exp[i // t.g_rows, j // t.g_cols] != E_ZERO else Fraction(0)
             for j in range(t.cols)] for i in range(t.rows)]


# --------------------------------------------------------------------- rounding


def test_rne_shift_matches_python_round():
    rng = np.random.default_rng(1)
    for x in range(-300, 301):
        for s in range(0, 9):
            assert oracle.rne_shift(x, -s) == round(Fraction(x, 2 ** s)), (x, s)
    for _ in range(3000):
        x = int(rng.integers(-(2 ** 50), 2 ** 50))
        s = int(rng.integers(1, 62))
        assert oracle.rne_shift(x, -s) == round(Fraction(x, 2 ** s))
    # exact left shifts
    assert oracle.rne_shift(-5, 3) == -40


def test_need_is_smallest_fitting_exponent():
    rng = np.random.default_rng(2)
    xs = list(range(-2000, 2001)) + [int(v) for v in rng.integers(-(2 ** 40), 2 ** 40, 2000)]
    for r in (-20, 0, 9):
        for x in xs:
            if x == 0:
                assert oracle.need(x, r) == E_ZERO
                continue
            e = oracle.need(x, r)
            v = value(x, r)
            assert abs(round(v / pow2(e))) <= 127
            assert abs(round(v / pow2(e - 1))) > 127


def test_requant_golden():
    for case in golden("requant_ties.json")["cases"]:
        x = np.array([case["x"]], np.int64)
        out = oracle.requant(x, 1, x.shape[1], base_exp=case["r"])
        assert out.mant[0].tolist() == case["c"], case
        assert int(out.exp[0, 0]) == case["e"], case


@pytest.mark.parametrize("rows,cols,g_rows,g_cols", [
    (1, 1, 1, 1), (3, 7, 1, 7), (5, 33, 1, 32), (8, 64, 2, 16), (17, 5, 17, 5), (6, 10, 4, 3),
])
def test_requant_matches_bruteforce(rows, cols, g_rows, g_cols):
    rng = np.random.default_rng(rows * 100 + cols)
    for trial in range(4):
        bits = [8, 20, 31, 45][trial]
        x = rng.integers(-(2 ** bits), 2 ** bits, size=(rows, cols)).astype(np.int64)
        x[rng.random((rows, cols)) < 0.2] = 0
        re = rng.integers(-20, 20, size=rows).astype(np.int8)
        ce = rng.integers(-20, 20, size=cols).astype(np.int8)
        out = oracle.requant(x, g_rows, g_cols, base_exp=-3, row_exp=re, col_exp=ce)
        vals = [[value(int(x[i, j]), -3 + int(re[i]) + int(ce[j])) for j in range(cols)]
                for i in range(rows)]
        mant, exps = fit_matrix_brute(vals, g_rows, g_cols)
        assert out.mant.tolist() == mant
        assert out.exp.tolist() == exps


def test_requant_exponent_range_error():
    with pytest.raises(oracle.OracleError) as ei:
        oracle.requant(np.array([[2 ** 40]], np.int64), 1, 1, base_exp=120)
    assert ei.value.code == oracle.ORC_ERR_EXP_RANGE
    # the lower clamp: tiny values saturate at exponent -127 instead of failing
    out = oracle.requant(np.array([[1, 3]], np.int64), 1, 2, base_exp=-200)
    assert int(out.exp[0, 0]) == -127 and out.mant.tolist() == [[0, 0]]


def test_two_term_sticky_matches_unbounded_integers():
    """Exponent gaps far beyond 64 bits, checked with Python's unbounded integers."""
    rng = np.random.default_rng(3)
    for trial in range(400):
        n = int(rng.integers(1, 6))
        a = rng.integers(-30000, 30001, size=n)
        b = rng.integers(-30000, 30001, size=n)
        a[rng.random(n) < 0.2] = 0
        b[rng.random(n) < 0.2] = 0
        base = int(rng.integers(-60, 60))
        spread = [4, 30, 90, 160, 260][trial % 5]
        pa = base + rng.integers(-spread, spread + 1, size=n)
        pb = base + rng.integers(-spread, spread + 1, size=n)
        if trial % 3 == 0:  # group-uniform exponents, as in the SGD update
            pa[:] = pa[0]
            pb[:] = pb[0]
        vals = [value(int(a[i]), int(pa[i])) + value(int(b[i]), int(pb[i])) for i in range(n)]
        cref, eref = fit_brute(vals)
        if eref > 127:
            continue
        c, e = oracle.fit_two_term(a, pa, b, pb)
        assert e == eref and c.tolist() == cref, (a, pa, b, pb)


# --------------------------------------------------------------------- alignment


def test_align_uniform_operand_is_identity():
    rng = np.random.default_rng(4)
    t = rand_ce(rng, 9, 40, 1, 40)
    m, e = oracle.align(t, axis=1)
    assert (m == t.mant).all() and (e == t.exp[:, 0]).all()


@pytest.mark.parametrize("axis", [0, 1])
@pytest.mark.parametrize("g", [(1, 4), (3, 5), (2, 40), (9, 1)])
def test_align_rounds_to_max_group_exponent(axis, g):
    rng = np.random.default_rng(5 + axis)
    t = rand_ce(rng, 9, 13, g[0], g[1], zero_groups=0.15)
    m, e = oracle.align(t, axis=axis)
    mt, et = oracle.align(t, axis=axis, transpose=True)
    assert (mt == m.T).all() and (et == e).all()
    vals = ce_values(t)
    n_keep = t.rows if axis == 1 else t.cols
    n_red = t.cols if axis == 1 else t.rows
    for a in range(n_keep):
        idx = [(a, b) if axis == 1 else (b, a) for b in range(n_red)]
        gexp = [int(t.exp[i // t.g_rows, j // t.g_cols]) for i, j in idx]
        live = [x for x in gexp if x != E_ZERO]
        assert int(e[a]) == (max(live) if live else E_ZERO)
        for (i, j) in idx:
            want = 0 if not live else round(vals[i][j] / pow2(int(e[a])))
            assert int(m[i, j]) == want


@pytest.mark.parametrize("axis", [0, 1])
@pytest.mark.parametrize("g", [(1, 4), (3, 5), (9, 1)])
def test_align_to_raised_targets_matches_python_round(axis, g):
    """ALIGN_MAX to targets above the tensor's own maxima (the maxima of a larger batch):
    every mantissa is Python's half-to-even round of its exact value at the target."""
    rng = np.random.default_rng(40 + axis)
    t = rand_ce(rng, 9, 13, g[0], g[1], zero_groups=0.2)
    _, e = oracle.align(t, axis=axis)
    raise_by = rng.integers(0, 10, size=e.shape)
    target = np.where(e == E_ZERO, rng.integers(-20, 0, size=e.shape), e.astype(np.int64) + raise_by).astype(np.int8)
    target[0] = E_ZERO if e[0] == E_ZERO else target[0]  # an all-zero index may keep E_ZERO
    m = oracle.align_to(t, axis, target)
    assert (oracle.align_to(t, axis, target, transpose=True) == m.T).all()
    vals = ce_values(t)
    for i in range(t.rows):
        for j in range(t.cols):
            tg = int(target[i if axis == 1 else j])
            want = 0 if vals[i][j] == 0 else round(vals[i][j] / pow2(tg))
            assert int(m[i, j]) == want, (i, j)


def test_align_to_own_maxima_equals_align():
    rng = np.random.default_rng(43)
    t = rand_ce(rng, 17, 24, 1, 8, zero_groups=0.1)
    for axis in (0, 1):
        m, e = oracle.align(t, axis=axis)
        assert (oracle.align_to(t, axis, e) == m).all()


def test_align_to_rejects_target_below_a_group():
    t = CE(np.array([[3, 0], [5, 1]], np.int8), np.array([[-4], [-2]], np.int8), 1, 2)
    with pytest.raises(oracle.OracleError):
        oracle.align_to(t, 0, np.array([-3, -3], np.int8))  # row 1's group sits at -2


def test_split_batch_sums_reproduce_whole_batch():
    """Backward weight of a batch split in three (one shard empty): shard-wise alignment to
    the MAX of the shards' targets, exact int64 sums added over the shards, one FIT.  This
    is the whole-batch result, bit for bit (integer addition is exact in any order)."""
    rng = np.random.default_rng(44)
    K, M, N = 50, 24, 40
    dY = rand_ce(rng, K, M, 1, 8, elo=-14, ehi=-3, zero_groups=0.1)
    X = rand_ce(rng, K, N, 1, 8, elo=-9, ehi=-1, zero_groups=0.1)
    cuts = [(0, 21), (21, 21), (21, K)]
    shard = lambda t, a, b: CE(t.mant[a:b].copy(), t.exp[a:b].copy(), 1, t.g_cols)
    parts = [(shard(dY, a, b), shard(X, a, b)) for a, b in cuts]
    e_dy = np.max([oracle.align(p[0], 0)[1] for p in parts], axis=0).astype(np.int8)
    e_x = np.max([oracle.align(p[1], 0)[1] for p in parts], axis=0).astype(np.int8)
    acc = np.zeros((M, N), np.int64)
    for pdy, px in parts:
        acc += oracle.align_to(pdy, 0, e_dy).astype(np.int64).T @ oracle.align_to(px, 0, e_x).astype(np.int64)
    got = oracle.requant(acc, 1, N, 0, row_exp=e_dy, col_exp=e_x)
    ref = oracle.linear_bwd_weight(dY, X)
    assert (got.mant == ref.mant).all() and (got.exp == ref.exp).all()


# --------------------------------------------------------------------- linear


def test_linear_golden():
    g = golden("linear_2x2.json")
    X, W, dY = ce_from(g["X"], g["X"]["g"]), ce_from(g["W"], g["W"]["g"]), ce_from(g["dY"], g["dY"]["g"])
    for name, fn, args in (("fwd", oracle.linear_fwd, (X, W)),
                           ("bwd_data", oracle.linear_bwd_data, (dY, W)),
                           ("bwd_weight", oracle.linear_bwd_weight, (dY, X))):
        ref = g[name]
        out = fn(*args, *ref["g"])
        assert out.mant.tolist() == ref["mant"], name
        assert out.exp.tolist() == ref["exp"], name
    wa, we = oracle.align(W, axis=0)
    assert wa.tolist() == [[5, 1], [0, 2]] and we.tolist() == [-2, -2]


SHAPES = [(1, 1, 1), (2, 3, 5), (5, 8, 17), (17, 33, 8), (33, 5, 3), (8, 17, 33)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_linear_acc_matches_numpy_matmul(M, N, K):
    """Pre-requant accumulators equal the int64 matmul of the aligned mantissas."""
    rng = np.random.default_rng(M * 1000 + N * 10 + K)
    X = rand_ce(rng, M, K, 1, max(1, K // 2), zero_groups=0.1)
    W = rand_ce(rng, N, K, 2, 3, zero_groups=0.1)
    dY = rand_ce(rng, M, N, 1, 2, zero_groups=0.1)

    def ez(a, b):
        return np.where((a[:, None] == E_ZERO) | (b[None, :] == E_ZERO), 0,
                        a[:, None].astype(np.int32) + b[None, :])

    acc, r = oracle.linear_fwd_acc(X, W)
    xa, xe = oracle.align(X, 1)
    wa, we = oracle.align(W, 1)
    assert (acc == xa.astype(np.int64) @ wa.astype(np.int64).T).all()
    assert (r == ez(xe, we)).all()

    acc, r = oracle.linear_bwd_data_acc(dY, W)
    ya, ye = oracle.align(dY, 1)
    wa0, we0 = oracle.align(W, 0)
    assert (acc == ya.astype(np.int64) @ wa0.astype(np.int64)).all()
    assert (r == ez(ye, we0)).all()

    acc, r = oracle.linear_bwd_weight_acc(dY, X)
    ya0, ye0 = oracle.align(dY, 0)
    xa0, xe0 = oracle.align(X, 0)
    assert (acc == ya0.astype(np.int64).T @ xa0.astype(np.int64)).all()
    assert (r == ez(ye0, xe0)).all()


@pytest.mark.parametrize("M,N,K", SHAPES[:4])
def test_linear_outputs_match_bruteforce_fit(M, N, K):
    rng = np.random.default_rng(7 + M + N + K)
    X = rand_ce(rng, M, K, 1, 2)
    W = rand_ce(rng, N, K, 1, K)
    dY = rand_ce(rng, M, N, 1, 3)
    for fn, accfn, args, shape in (
        (oracle.linear_fwd, oracle.linear_fwd_acc, (X, W), (M, N)),
        (oracle.linear_bwd_data, oracle.linear_bwd_data_acc, (dY, W), (M, K)),
        (oracle.linear_bwd_weight, oracle.linear_bwd_weight_acc, (dY, X), (N, K)),
    ):
        g = (1, max(1, shape[1] // 2))
        out = fn(*args, *g)
        acc, r = accfn(*args)
        vals = [[value(int(acc[i, j]), int(r[i, j])) for j in range(shape[1])] for i in range(shape[0])]
        mant, exps = fit_matrix_brute(vals, *g)
        assert out.mant.tolist() == mant and out.exp.tolist() == exps


def test_linear_exact_when_nothing_rounds():
    """All exponents 0 and |acc| <= 127: the (C,e) result is the plain integer matmul."""
    rng = np.random.default_rng(8)
    X = CE(rng.integers(-3, 4, size=(6, 4)).astype(np.int8), np.zeros((1, 1), np.int8), 6, 4)
    W = CE(rng.integers(-3, 4, size=(5, 4)).astype(np.int8), np.zeros((1, 1), np.int8), 5, 4)
    Y = oracle.linear_fwd(X, W, 1, 5)
    ref = X.mant.astype(np.int64) @ W.mant.astype(np.int64).T
    got = [[value(int(Y.mant[i, j]), int(Y.exp[i, 0])) if Y.exp[i, 0] != E_ZERO else 0
            for j in range(5)] for i in range(6)]
    assert got == ref.tolist()


# --------------------------------------------------------------------- conv


def _conv_case(rng, n=2, h=5, w=6, c=8, k=12, g=4, r=3, s=3, pad=1, stride=1):
    P = (h + 2 * pad - r) // stride + 1
    Q = (w + 2 * pad - s) // stride + 1
    X = rand_ce(rng, n * h * w, c, n * h * w, g)
    W = rand_ce(rng, k, r * s * c, 1, r * s * c)
    dY = rand_ce(rng, n * P * Q, k, n * P * Q, g)
    d = dict(n=n, h=h, w=w, c=c, k=k, r=r, s=s, stride=stride, pad=pad)
    return X, W, dY, d, P, Q


@pytest.mark.parametrize("geom", [dict(), dict(stride=2), dict(r=1, s=1, pad=0), dict(h=3, w=3, pad=2),
                                  dict(h=4, w=6, r=2, s=2, pad=0, stride=2)])  # non-overlapping patches
def test_conv_acc_matches_torch_conv(geom):
    torch = pytest.importorskip("torch")
    F = torch.nn.functional
    rng = np.random.default_rng(9)
    X, W, dY, d, P, Q = _conv_case(rng, **geom)
    n, h, w, c, k, r, s = (d[x] for x in ("n", "h", "w", "c", "k", "r", "s"))
    xa, xe = oracle.align(X, 1)
    wa, we = oracle.align(W, 1)
    xt = torch.tensor(xa, dtype=torch.float64).reshape(n, h, w, c).permute(0, 3, 1, 2)
    wt = torch.tensor(wa, dtype=torch.float64).reshape(k, r, s, c).permute(0, 3, 1, 2)
    ref = F.conv2d(xt, wt, stride=d["stride"], padding=d["pad"]).permute(0, 2, 3, 1).reshape(-1, k)
    acc, rx = oracle.conv_acc(oracle.CONV_FWD, d, X, W)
    assert (acc == ref.numpy().astype(np.int64)).all()
    assert (rx == int(xe[0]) + we[None, :].astype(np.int32)).all()

    # bwd-data: W aligned per input channel over (k, r, s)
    W4 = CE(W.mant.reshape(k * r * s, c).copy(), W.exp.copy(), r * s, c)
    wa_c, we_c = oracle.align(W4, 0)
    ya, ye = oracle.align(dY, 1)
    yt = torch.tensor(ya, dtype=torch.float64).reshape(n, P, Q, k).permute(0, 3, 1, 2)
    wct = torch.tensor(wa_c, dtype=torch.float64).reshape(k, r, s, c).permute(0, 3, 1, 2)
    out_pad = (h + 2 * d["pad"] - r) % d["stride"], (w + 2 * d["pad"] - s) % d["stride"]
    ref = F.conv_transpose2d(yt, wct, stride=d["stride"], padding=d["pad"], output_padding=out_pad)
    ref = ref.permute(0, 2, 3, 1).reshape(-1, c)
    acc, rx = oracle.conv_acc(oracle.CONV_BWD_DATA, d, dY, W)
    assert (acc == ref.numpy().astype(np.int64)).all()
    assert (rx == int(ye[0]) + we_c[None, :].astype(np.int32)).all()

    # bwd-weight: both aligned per channel over all pixels
    ya0, ye0 = oracle.align(dY, 0)
    xa0, xe0 = oracle.align(X, 0)
    yt0 = torch.tensor(ya0, dtype=torch.float64).reshape(n, P, Q, k).permute(0, 3, 1, 2)
    xt0 = torch.tensor(xa0, dtype=torch.float64).reshape(n, h, w, c).permute(0, 3, 1, 2)
    ref = torch.nn.grad.conv2d_weight(xt0, (k, c, r, s), yt0, stride=d["stride"], padding=d["pad"])
    ref = ref.permute(0, 2, 3, 1).reshape(k, -1)
    acc, rx = oracle.conv_acc(oracle.CONV_BWD_WEIGHT, d, dY, X)
    assert (acc == ref.numpy().astype(np.int64)).all()
    assert (rx == ye0[:, None].astype(np.int32) + np.tile(xe0, r * s)[None, :]).all()


def test_conv_outputs_match_bruteforce_fit():
    rng = np.random.default_rng(10)
    X, W, dY, d, P, Q = _conv_case(rng, n=1, h=4, w=4, c=4, k=4, g=2)
    for direction, a, b, g in ((oracle.CONV_FWD, X, W, (16, 2)),
                               (oracle.CONV_BWD_DATA, dY, W, (16, 2)),
                               (oracle.CONV_BWD_WEIGHT, dY, X, (1, 36))):
        out = oracle.conv(direction, d, a, b, *g)
        acc, r = oracle.conv_acc(direction, d, a, b)
        vals = [[value(int(acc[i, j]), int(r[i, j])) for j in range(acc.shape[1])]
                for i in range(acc.shape[0])]
        mant, exps = fit_matrix_brute(vals, *g)
        assert out.mant.tolist() == mant and out.exp.tolist() == exps


def test_conv_rejects_pixel_varying_activation_exponents():
    rng = np.random.default_rng(11)
    X, W, dY, d, P, Q = _conv_case(rng)
    Xbad = rand_ce(rng, X.rows, X.cols, 1, 4)
    with pytest.raises(oracle.OracleError) as ei:
        oracle.conv(oracle.CONV_FWD, d, Xbad, W, X.rows, 4)
    assert ei.value.code == oracle.ORC_ERR_LAYOUT


# --------------------------------------------------------------------- SGD


def test_sgd_golden():
    g = golden("sgd_2x2.json")
    W, V, G = (ce_from(g[n], g["g"]) for n in ("W", "V", "G"))
    W2, V2 = oracle.sgd_step(W, V, G, tuple(g["mom"]), tuple(g["lr"]))
    assert V2.mant.tolist() == g["V_new"]["mant"] and V2.exp.tolist() == g["V_new"]["exp"]
    assert W2.mant.tolist() == g["W_new"]["mant"] and W2.exp.tolist() == g["W_new"]["exp"]


def _sgd_brute(W, V, G, mom, lr, qmax=127):
    wv, vv, gv = ce_values(W), ce_values(V), ce_values(G)
    rows, cols = W.rows, W.cols
    vnew = [[Fraction(mom[0]) * vv[i][j] / 2 ** mom[1] + gv[i][j] for j in range(cols)] for i in range(rows)]
    vm, ve = fit_matrix_brute(vnew, W.g_rows, W.g_cols, qmax)
    vq = [[value(vm[i][j], ve[i // W.g_rows][j // W.g_cols]) if ve[i // W.g_rows][j // W.g_cols] != E_ZERO
           else Fraction(0) for j in range(cols)] for i in range(rows)]
    wnew = [[wv[i][j] - Fraction(lr[0]) * vq[i][j] / 2 ** lr[1] for j in range(cols)] for i in range(rows)]
    wm, we = fit_matrix_brute(wnew, W.g_rows, W.g_cols, qmax)
    return wm, we, vm, ve


@pytest.mark.parametrize("g", [(1, 8), (2, 3), (1, 1), (3, 8)])
@pytest.mark.parametrize("erange", [(-16, -4), (-120, 0), (-127, 40)])
def test_sgd_matches_bruteforce(g, erange):
    rng = np.random.default_rng(1000 + g[0] * 7 + g[1] + erange[0])
    for trial in range(3):
        W = rand_ce(rng, 5, 8, *g, elo=erange[0], ehi=erange[1], zero_groups=0.1)
        V = rand_ce(rng, 5, 8, *g, elo=erange[0], ehi=erange[1], zero_groups=0.3)
        G = rand_ce(rng, 5, 8, *g, elo=erange[0], ehi=erange[1], zero_groups=0.1)
        mom, lr = (230, 8), [(1, 4), (205, 11), (3, 0)][trial]
        wm, we, vm, ve = _sgd_brute(W, V, G, mom, lr)
        if max(max(r) for r in we + ve) > 127:
            continue
        W2, V2 = oracle.sgd_step(W, V, G, mom, lr)
        assert V2.mant.tolist() == vm and V2.exp.tolist() == ve
        assert W2.mant.tolist() == wm and W2.exp.tolist() == we


# --------------------------------------------------------------------- GELU


def _h(x: Fraction) -> Fraction:
    return x * min(max((x + 2) / 4, Fraction(0)), Fraction(1))


def _hprime(x: Fraction) -> Fraction:
    if x <= -2:
        return Fraction(0)
    if x >= 2:
        return Fraction(1)
    return (x + 1) / 2


def test_gelu_golden():
    g = golden("gelu_e_minus5.json")
    H = CE(np.array([g["c"]], np.int8), np.array([[g["e"]]], np.int8), 1, len(g["c"]))
    assert oracle.gelu_fwd(H).mant[0].tolist() == g["out"]


def test_gelu_fwd_closed_form_all_mantissas():
    cs = np.arange(-127, 128, dtype=np.int8)
    for e in list(range(-40, 8)) + [-127, -100, 127]:
        H = CE(cs[None, :].copy(), np.array([[e]], np.int8), 1, cs.size)
        out = oracle.gelu_fwd(H)
        assert int(out.exp[0, 0]) == e
        want = [round(_h(value(int(c), e)) / pow2(e)) for c in cs]
        assert out.mant[0].tolist() == want, e


def test_gelu_fwd_close_to_erf_gelu():
    import math
    cs = np.arange(-127, 128, dtype=np.int8)
    e = -5
    out = oracle.gelu_fwd(CE(cs[None, :].copy(), np.array([[e]], np.int8), 1, cs.size))
    for c, o in zip(cs.tolist(), out.mant[0].tolist()):
        x = c * 2.0 ** e
        gelu = 0.5 * x * (1 + math.erf(x / math.sqrt(2)))
        assert abs(o * 2.0 ** e - gelu) <= 0.105 + 2.0 ** (e - 1)  # curve error peaks at 0.1023 near |x| = 1.25


@pytest.mark.parametrize("eh_range", [(-8, 2), (-127, -90), (-30, 10)])
def test_gelu_bwd_matches_bruteforce(eh_range):
    rng = np.random.default_rng(1000 + eh_range[0])
    H = rand_ce(rng, 4, 16, 1, 8, elo=eh_range[0], ehi=eh_range[1], zero_groups=0.1)
    dG = rand_ce(rng, 4, 16, 1, 8, elo=-20, ehi=-5, zero_groups=0.1)
    hv, dv = ce_values(H), ce_values(dG)
    vals = [[dv[i][j] * _hprime(hv[i][j]) for j in range(16)] for i in range(4)]
    mant, exps = fit_matrix_brute(vals, 1, 8)
    out = oracle.gelu_bwd(H, dG, 1, 8)
    assert out.mant.tolist() == mant and out.exp.tolist() == exps


# --------------------------------------------------------------------- errors


def test_input_invariants_are_enforced():
    bad = CE(np.array([[-128, 1]], np.int8), np.array([[0]], np.int8), 1, 2)
    ok = CE(np.array([[1, 1]], np.int8), np.array([[0]], np.int8), 1, 2)
    with pytest.raises(oracle.OracleError):
        oracle.linear_fwd(bad, ok, 1, 1)
    zero_bad = CE(np.array([[0, 3]], np.int8), np.array([[E_ZERO]], np.int8), 1, 2)
    with pytest.raises(oracle.OracleError):
        oracle.linear_fwd(zero_bad, ok, 1, 1)


# --------------------------------------------------------------------- Sum (residual add)


@pytest.mark.parametrize("gx,gy,gz", [((1, 4), (1, 4), (1, 4)), ((9, 5), (1, 13), (3, 4)), ((1, 13), (9, 1), (9, 13))])
@pytest.mark.parametrize("erange", [((-12, -2), (-12, -2)), ((-30, -20), (-3, 5)), ((-127, -90), (10, 40))])
def test_sum_matches_bruteforce(gx, gy, gz, erange):
    """FIT(X + Y) against exact rational sums and the brute-force FIT, with exponent gaps
    from 0 up to beyond the oracle's exact span (its sticky reduction)."""
    rng = np.random.default_rng(60 + gx[0] + gy[1] + abs(erange[0][0]))
    X = rand_ce(rng, 9, 13, *gx, *erange[0], zero_groups=0.15)
    Y = rand_ce(rng, 9, 13, *gy, *erange[1], zero_groups=0.15)
    Z = oracle.sum_(X, Y, *gz)
    vx, vy = ce_values(X), ce_values(Y)
    mant, exps = fit_matrix_brute([[vx[i][j] + vy[i][j] for j in range(13)] for i in range(9)], *gz)
    assert Z.mant.tolist() == mant and Z.exp.tolist() == exps


def test_sum_with_zero_is_requant_of_the_other_term():
    rng = np.random.default_rng(61)
    X = rand_ce(rng, 6, 32, 1, 16)
    Zr = CE(np.zeros((6, 32), np.int8), np.full((6, 2), E_ZERO, np.int8), 1, 16)
    # every group holds a mantissa of magnitude >= 64, so X is its own FIT
    assert (np.abs(X.mant.astype(int)).reshape(6, 2, 16).max(axis=2) >= 64).all()
    Z = oracle.sum_(X, Zr, 1, 16)
    assert (Z.mant == X.mant).all() and (Z.exp == X.exp).all()
    assert (oracle.sum_(Zr, Zr, 1, 16).exp == E_ZERO).all()


def test_sum_of_equal_terms_doubles():
    """x + x = 2x: the exponent rises by one exactly where the mantissa cannot double."""
    rng = np.random.default_rng(62)
    X = rand_ce(rng, 5, 48, 1, 16)
    Z = oracle.sum_(X, X, 1, 16)
    vx, vz = ce_values(X), ce_values(Z)
    for i in range(5):
        for j in range(48):
            assert vz[i][j] == 2 * vx[i][j]  # doubling is exact in (C, e+1)


# --------------------------------------------------------------------- ReLU / ReLU6


def _all_mantissas_ce(e_list):
    """One row per exponent, every mantissa -127..127 once: rows x 255, one group per row."""
    m = np.tile(np.arange(-127, 128, dtype=np.int8), (len(e_list), 1))
    return CE(m, np.array(e_list, np.int8).reshape(-1, 1), 1, 255)


def test_relu_fwd_matches_torch():
    import torch

    X = _all_mantissas_ce(list(range(-127, 128, 3)))
    vals = torch.tensor([[float(v) for v in row] for row in ce_values(X)], dtype=torch.float64)
    for six in (False, True):
        Z = oracle.relu_fwd(X, six)
        assert (Z.exp == X.exp).all()
        got = torch.tensor([[float(v) for v in row] for row in ce_values(Z)], dtype=torch.float64)
        if not six:
            assert torch.equal(got, torch.relu(vals))
            continue
        for r, e in enumerate(X.exp[:, 0].tolist()):
            if e <= 1:  # the bound 6 >> e times 2^e is 6, or q_max * 2^e < 6: exactly relu6
                assert torch.equal(got[r], torch.nn.functional.relu6(vals[r])), e
            else:  # 6 >> e truncates: the largest multiple of 2^e not above 6 (0 for e >= 3)
                cap = (6 >> e) * 2.0 ** e
                assert torch.equal(got[r], torch.clamp(vals[r], 0.0, cap)), e


def test_relu_bwd_matches_torch_autograd():
    import torch

    rng = np.random.default_rng(63)
    X = _all_mantissas_ce(list(range(-12, 3)))
    dY = CE(rng.integers(-127, 128, size=X.mant.shape).astype(np.int8),
            rng.integers(-20, -5, size=(X.rows, 1)).astype(np.int8), 1, 255)
    vals = torch.tensor([[float(v) for v in row] for row in ce_values(X)], dtype=torch.float64)
    up = torch.tensor(dY.mant, dtype=torch.float64)
    for six, fn in ((False, torch.relu), (True, torch.nn.functional.relu6)):
        x = vals.clone().requires_grad_(True)
        fn(x).backward(up)
        dX = oracle.relu_bwd(X, dY, six)
        assert (dX.exp == dY.exp).all()
        got = torch.tensor(dX.mant, dtype=torch.float64)
        for r, e in enumerate(X.exp[:, 0].tolist()):
            if six and e <= -5:
                # c = q_max: the page's mask 0 < C < c also drops C = q_max (value below 6)
                want = x.grad[r].clone()
                want[-1] = 0.0
                assert torch.equal(got[r], want), e
            elif six and e == 2:  # c = 1: no mantissa lies strictly between 0 and 1
                assert (got[r] == 0).all()
            else:
                assert torch.equal(got[r], x.grad[r]), (six, e)


@pytest.mark.parametrize("xw,yw", [((1, 0), (105, 20)), ((-3, 1), (230, 8)), ((512, 0), (-512, 30)),
                                   ((7, 64), (1, 0))])
def test_sum_scaled_matches_bruteforce(xw, yw):
    """FIT(xm 2^-xs X + ym 2^-ys Y) against exact rationals: the weight-decay form
    G + lambda W (lambda = 105 * 2^-20, about 1e-4) among others."""
    rng = np.random.default_rng(70 + xw[0] + yw[1])
    X = rand_ce(rng, 7, 32, 1, 16, elo=-20, ehi=-8, zero_groups=0.15)
    Y = rand_ce(rng, 7, 32, 1, 16, elo=-12, ehi=0, zero_groups=0.15)
    Z = oracle.sum_scaled(X, xw, Y, yw, 1, 16)
    vx, vy = ce_values(X), ce_values(Y)
    wx = Fraction(xw[0]) * pow2(-xw[1])
    wy = Fraction(yw[0]) * pow2(-yw[1])
    mant, exps = fit_matrix_brute([[wx * vx[i][j] + wy * vy[i][j] for j in range(32)] for i in range(7)], 1, 16)
    assert Z.mant.tolist() == mant and Z.exp.tolist() == exps


def test_sum_scaled_unit_weights_is_sum():
    rng = np.random.default_rng(71)
    X = rand_ce(rng, 5, 48, 1, 16, zero_groups=0.1)
    Y = rand_ce(rng, 5, 48, 1, 16, elo=-20, ehi=-5, zero_groups=0.1)
    a, b = oracle.sum_scaled(X, (1, 0), Y, (1, 0), 1, 16), oracle.sum_(X, Y, 1, 16)
    assert (a.mant == b.mant).all() and (a.exp == b.exp).all()
    with pytest.raises(oracle.OracleError):
        oracle.sum_scaled(X, (513, 0), Y, (1, 0), 1, 16)  # weights beyond 512 are refused


# --------------------------------------------------------------------- average pool


def _act(rng, n, h, w, c, g, elo=-9, ehi=-5):
    """NHWC activations with channel groups of g spanning all pixels."""
    npix = n * h * w
    m = rng.integers(-127, 128, size=(npix, c)).astype(np.int8)
    return with_groups(m, npix, g, lambda s: rng.integers(elo, ehi + 1, size=s))


@pytest.mark.parametrize("n,h,w,c,K,og", [(2, 4, 6, 32, 2, (1, 16)), (1, 6, 6, 16, 3, (4, 16)), (3, 7, 7, 32, 7, (1, 32)),
                                          (2, 5, 5, 16, 5, (2, 16)), (1, 4, 4, 16, 1, (16, 16))])
def test_avgpool_fwd_matches_bruteforce(n, h, w, c, K, og):
    rng = np.random.default_rng(80 + K + c)
    X = _act(rng, n, h, w, c, 16)
    g_rows = og[0] if og[0] != 16 else n * (h // K) * (w // K)
    Y = oracle.avgpool_fwd(X, n, h, w, K, g_rows, og[1])
    vx = ce_values(X)
    P, Q = h // K, w // K
    vals = [[sum(vx[(img * h + p * K + dy) * w + q * K + dx][ch] for dy in range(K) for dx in range(K)) / (K * K)
             for ch in range(c)] for img in range(n) for p in range(P) for q in range(Q)]
    mant, exps = fit_matrix_brute(vals, g_rows, og[1])
    assert Y.mant.tolist() == mant and Y.exp.tolist() == exps


def test_avgpool_power_of_two_window_is_a_requant():
    """D = 4: the average is the dyadic S 2^(e-2), so the pool equals the integer FIT of
    the window sums at exponent e - 2."""
    rng = np.random.default_rng(85)
    n, h, w, c = 2, 6, 4, 32
    X = _act(rng, n, h, w, c, 32)
    Y = oracle.avgpool_fwd(X, n, h, w, 2, 1, 16)
    S = X.mant.astype(np.int64).reshape(n, h // 2, 2, w // 2, 2, c).sum(axis=(2, 4)).reshape(-1, c)
    ref = oracle.requant(S, 1, 16, base_exp=-2, col_exp=np.repeat(X.exp[0], 32))
    assert (Y.mant == ref.mant).all() and (Y.exp == ref.exp).all()


@pytest.mark.parametrize("n,h,w,c,K,dyg,dxg", [(2, 4, 6, 32, 2, (1, 16), (48, 16)), (1, 6, 6, 16, 3, (4, 16), (1, 16)),
                                               (3, 7, 7, 32, 7, (1, 32), (147, 32))])
def test_avgpool_bwd_matches_bruteforce(n, h, w, c, K, dyg, dxg):
    rng = np.random.default_rng(90 + K)
    rows = n * (h // K) * (w // K)
    dY = rand_ce(rng, rows, c, *dyg, elo=-16, ehi=-8, zero_groups=0.1)
    dX = oracle.avgpool_bwd(dY, n, h, w, K, *dxg)
    vy = ce_values(dY)
    P, Q = h // K, w // K
    vals = [[vy[(img * P + y // K) * Q + x // K][ch] / (K * K) for ch in range(c)]
            for img in range(n) for y in range(h) for x in range(w)]
    mant, exps = fit_matrix_brute(vals, *dxg)
    assert dX.mant.tolist() == mant and dX.exp.tolist() == exps


# --------------------------------------------------------------------- depthwise convolution


@pytest.mark.parametrize("geom", [dict(), dict(stride=2), dict(r=5, s=5, pad=2), dict(h=4, w=4, r=1, s=1, pad=0)])
def test_depthwise_acc_matches_torch_grouped_conv(geom):
    """Depthwise sums against torch's grouped convolution (groups = channels) in float64
    on the exact mantissas, all three directions, and the exponents each sum carries."""
    torch = pytest.importorskip("torch")
    F = torch.nn.functional
    rng = np.random.default_rng(95)
    n, h, w, c = geom.get("n", 2), geom.get("h", 6), geom.get("w", 5), 8
    r, s, pad, stride = geom.get("r", 3), geom.get("s", 3), geom.get("pad", 1), geom.get("stride", 1)
    P, Q = (h + 2 * pad - r) // stride + 1, (w + 2 * pad - s) // stride + 1
    X = rand_ce(rng, n * h * w, c, n * h * w, 4, zero_groups=0.2)
    W = rand_ce(rng, c, r * s, 1, r * s)
    dY = rand_ce(rng, n * P * Q, c, n * P * Q, 2, zero_groups=0.2)
    d = dict(n=n, h=h, w=w, c=c, k=c, r=r, s=s, stride=stride, pad=pad)
    xt = torch.tensor(X.mant, dtype=torch.float64).reshape(n, h, w, c).permute(0, 3, 1, 2)
    wt = torch.tensor(W.mant, dtype=torch.float64).reshape(c, 1, r, s)
    yt = torch.tensor(dY.mant, dtype=torch.float64).reshape(n, P, Q, c).permute(0, 3, 1, 2)
    ex = np.repeat(X.exp[0], 4)[:c].astype(np.int32)
    ey = np.repeat(dY.exp[0], 2)[:c].astype(np.int32)
    ew = W.exp[:, 0].astype(np.int32)

    def esum(a, b):
        return np.where((a == E_ZERO) | (b == E_ZERO), 0, a + b)

    acc, rx = oracle.depthwise_acc(0, d, X, W)
    ref = F.conv2d(xt, wt, stride=stride, padding=pad, groups=c).permute(0, 2, 3, 1).reshape(-1, c)
    assert (acc == ref.numpy().astype(np.int64)).all()
    assert (rx == esum(ex, ew)[None, :]).all()
    acc, rx = oracle.depthwise_acc(1, d, dY, W)
    op = ((h + 2 * pad - r) % stride, (w + 2 * pad - s) % stride)
    ref = F.conv_transpose2d(yt, wt, stride=stride, padding=pad, output_padding=op, groups=c)
    assert (acc == ref.permute(0, 2, 3, 1).reshape(-1, c).numpy().astype(np.int64)).all()
    assert (rx == esum(ey, ew)[None, :]).all()
    acc, rx = oracle.depthwise_acc(2, d, dY, X)
    ref = torch.nn.grad.conv2d_weight(xt, (c, 1, r, s), yt, stride=stride, padding=pad, groups=c)
    assert (acc == ref.reshape(c, r * s).numpy().astype(np.int64)).all()
    assert (rx == esum(ey, ex)[:, None]).all()


def test_depthwise_outputs_match_bruteforce_fit():
    rng = np.random.default_rng(96)
    n, h, w, c, r = 1, 4, 4, 4, 3
    X = rand_ce(rng, n * h * w, c, n * h * w, 2)
    W = rand_ce(rng, c, r * r, 1, r * r)
    d = dict(n=n, h=h, w=w, c=c, k=c, r=r, s=r, stride=1, pad=1)
    Y = oracle.depthwise(0, d, X, W, n * h * w, 2)
    vx, vw = ce_values(X), ce_values(W)
    vals = [[sum(vx[(y + dy - 1) * w + (x + dx - 1)][ch] * vw[ch][dy * r + dx]
                 for dy in range(r) for dx in range(r) if 0 <= y + dy - 1 < h and 0 <= x + dx - 1 < w)
             for ch in range(c)] for y in range(h) for x in range(w)]
    mant, exps = fit_matrix_brute(vals, n * h * w, 2)
    assert Y.mant.tolist() == mant and Y.exp.tolist() == exps


# --------------------------------------------------------------------- B-bit mantissas (Table 4)


@pytest.mark.parametrize("bits", [4, 5, 6, 7, 8])
def test_requant_bits_matches_bruteforce(bits):
    rng = np.random.default_rng(100 + bits)
    x = rng.integers(-(2 ** 20), 2 ** 20, size=(6, 24)).astype(np.int64)
    x[rng.random(x.shape) < 0.15] = 0
    x[2] = 0  # an all-zero row: E_ZERO groups
    qmax = 2 ** (bits - 1) - 1
    out = oracle.requant_bits(x, bits, 1, 8, base_exp=-5)
    assert np.abs(out.mant).max() <= qmax
    mant = [[0] * 24 for _ in range(6)]
    exps = [[E_ZERO] * 3 for _ in range(6)]
    for gi, gj, cells in groups_of(6, 24, 1, 8):
        c, e = fit_brute([value(int(x[i, j]), -5) for i, j in cells], qmax=qmax)
        exps[gi][gj] = e
        for (i, j), cc in zip(cells, c):
            mant[i][j] = cc
    assert out.mant.tolist() == mant and out.exp.tolist() == exps


def test_requant_bits_8_is_requant():
    rng = np.random.default_rng(110)
    x = rng.integers(-(2 ** 30), 2 ** 30, size=(9, 40)).astype(np.int64)
    a, b = oracle.requant_bits(x, 8, 1, 8, base_exp=3), oracle.requant(x, 1, 8, base_exp=3)
    assert (a.mant == b.mant).all() and (a.exp == b.exp).all()


# --------------------------------------------------------------------- B-bit variants (Table 4)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 7, 8])
def test_linear_bits_match_bruteforce_fit(bits):
    """B-bit linear Products: the pinned exact accumulators, then the brute-force FIT with
    the clip bound q_max = 2^(B-1) - 1, on B-bit inputs."""
    q = (1 << (bits - 1)) - 1
    rng = np.random.default_rng(40 + bits)
    M, N, K = 6, 5, 7
    X = rand_ce(rng, M, K, 1, 3, mag=q)
    W = rand_ce(rng, N, K, 1, K, mag=q)
    dY = rand_ce(rng, M, N, 1, 2, mag=q)
    for op, accfn, args, shape in ((0, oracle.linear_fwd_acc, (X, W), (M, N)),
                                   (1, oracle.linear_bwd_data_acc, (dY, W), (M, K)),
                                   (2, oracle.linear_bwd_weight_acc, (dY, X), (N, K))):
        g = (1, max(1, shape[1] // 2))
        out = oracle.linear_bits(op, *args, bits, *g)
        acc, r = accfn(*args)
        vals = [[value(int(acc[i, j]), int(r[i, j])) for j in range(shape[1])] for i in range(shape[0])]
        mant, exps = fit_matrix_brute(vals, *g, qmax=q)
        assert out.mant.tolist() == mant and out.exp.tolist() == exps, (bits, op)
        assert np.abs(out.mant.astype(int)).max() <= q


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("erange", [(-16, -4), (-120, 0)])
def test_sgd_bits_matches_bruteforce(bits, erange):
    q = (1 << (bits - 1)) - 1
    rng = np.random.default_rng(900 + bits + erange[0])
    for trial in range(3):
        W = rand_ce(rng, 5, 8, 1, 8, elo=erange[0], ehi=erange[1], zero_groups=0.1, mag=q)
        V = rand_ce(rng, 5, 8, 1, 8, elo=erange[0], ehi=erange[1], zero_groups=0.3, mag=q)
        G = rand_ce(rng, 5, 8, 1, 8, elo=erange[0], ehi=erange[1], zero_groups=0.1, mag=q)
        mom, lr = (230, 8), [(1, 4), (205, 11), (3, 0)][trial]
        wm, we, vm, ve = _sgd_brute(W, V, G, mom, lr, q)
        if max(max(r) for r in we + ve) > 127:
            continue
        W2, V2 = oracle.sgd_step_bits(W, V, G, bits, mom, lr)
        assert V2.mant.tolist() == vm and V2.exp.tolist() == ve, (bits, trial)
        assert W2.mant.tolist() == wm and W2.exp.tolist() == we, (bits, trial)


def test_bits_8_is_the_int8_path():
    rng = np.random.default_rng(77)
    X, W = rand_ce(rng, 20, 64, 1, 16), rand_ce(rng, 12, 64, 1, 32)
    a, b = oracle.linear_bits(0, X, W, 8, 1, 4), oracle.linear_fwd(X, W, 1, 4)
    assert np.array_equal(a.mant, b.mant) and np.array_equal(a.exp, b.exp)
    V, G = rand_ce(rng, 12, 64, 1, 32), rand_ce(rng, 12, 64, 1, 32)
    for x, y in zip(oracle.sgd_step_bits(W, V, G, 8), oracle.sgd_step(W, V, G)):
        assert np.array_equal(x.mant, y.mant) and np.array_equal(x.exp, y.exp)
