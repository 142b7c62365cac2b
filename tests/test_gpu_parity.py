"""GPU parity: every entry point of libict.so against the CPU oracle, bit for bit.

Sizes span several 128-row tiles with ragged tails; group geometries cover per-tensor,
per-row, row-local (1, G) and pixel-uniform channel groups.  All arithmetic is integer,
so the comparison is exact equality of mantissas and exponent bytes.
"""
import numpy as np
import pytest

import oracle
from integer_only_nn_02_b200.workloads import CE, E_ZERO, clipped_laplace, with_groups
from tests.test_oracle_pins import rand_ce

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ict():
    from integer_only_nn_02_b200 import ict as _ict

    return _ict


def same(gpu_ce: CE, ref: CE, what=""):
    assert gpu_ce.mant.shape == ref.mant.shape, what
    bad = np.argwhere(gpu_ce.mant != ref.mant)
    assert bad.size == 0, f"{what}: {len(bad)} mantissas differ, first {bad[:5].tolist()}"
    bad = np.argwhere(gpu_ce.exp != ref.exp)
    assert bad.size == 0, f"{what}: {len(bad)} exponents differ, first {bad[:5].tolist()}"


def status_ok(ict):
    code, raw = ict.ict_get_device_status()
    assert code == 0, (code, raw)


# ------------------------------------------------------------------ requant / align


@pytest.mark.parametrize("rows,cols,G", [(5, 32, 32), (130, 96, 32), (64, 192, 64), (33, 768, 768), (7, 48, 16),
                                         (9, 192, 192), (4, 320, 160), (3, 3072, 3072), (6, 512, 256)])
def test_requant(ict, rows, cols, G):
    import torch

    rng = np.random.default_rng(rows + cols)
    for bits in (10, 24, 31):
        x = rng.integers(-(2 ** bits), 2 ** bits, size=(rows, cols)).astype(np.int64)
        x[rng.random(x.shape) < 0.1] = 0
        x[3 % rows] = 0  # an all-zero row -> E_ZERO groups
        re = rng.integers(-40, 20, size=rows).astype(np.int8)
        ce = rng.integers(-40, 20, size=cols).astype(np.int8)
        ref = oracle.requant(x, 1, G, base_exp=-5, row_exp=re, col_exp=ce)
        for dt in (torch.int32, torch.int64):
            if dt == torch.int32 and bits > 30:
                continue
            out = ict.DevCE.empty(rows, cols, 1, G)
            ict.ict_requant(torch.tensor(x, dtype=dt, device="cuda"), out, -5,
                            torch.tensor(re, device="cuda"), torch.tensor(ce, device="cuda"))
            same(out.to_host(), ref, f"requant {dt} bits={bits}")
    status_ok(ict)


@pytest.mark.parametrize("rows,cols,g", [(64, 128, (1, 32)), (200, 96, (1, 16)), (130, 64, (130, 32)),
                                         (48, 768, (1, 64)), (144, 32, (16, 32)), (100, 48, (1, 48))])
@pytest.mark.parametrize("axis,transpose", [(1, False), (0, True), (0, False), (1, True)])
def test_align(ict, rows, cols, g, axis, transpose):
    import torch

    rng = np.random.default_rng(rows * 3 + cols)
    t = rand_ce(rng, rows, cols, *g, elo=-20, ehi=5, zero_groups=0.1)
    ref_m, ref_e = oracle.align(t, axis, transpose)
    d = ict.DevCE.from_host(t)
    out_rows = cols if transpose else rows
    ld = -(-(rows if transpose else cols) // 16) * 16
    out = torch.zeros((out_rows, ld), dtype=torch.int8, device="cuda")
    e = torch.zeros(rows if axis == 1 else cols, dtype=torch.int8, device="cuda")
    ict.ict_align(d, axis, transpose, out, e)
    got = out.cpu().numpy()[:, : ref_m.shape[1]]
    assert (got == ref_m).all()
    assert (e.cpu().numpy() == ref_e).all()


# ------------------------------------------------------------------ linear

LINEAR_CASES = [
    # M, N, K, X groups, W groups, out group
    (64, 64, 128, (64, 128), (1, 128), 32),      # the single-layer config shapes
    (200, 192, 96, (1, 96), (1, 32), 32),
    (300, 320, 256, (1, 64), (1, 256), 64),
    (129, 256, 384, (1, 128), (4, 64), 256),
    (512, 448, 192, (1, 192), (1, 192), 64),
    (1000, 768, 768, (1, 64), (1, 64), 64),
    (2000, 64, 192, (1, 64), (1, 192), 64),       # long K: split-K slices, 192-wide dW rows
    (3000, 128, 320, (1, 32), (1, 320), 32),      # split-K, 320-wide dW rows
]


def _linear_inputs(M, N, K, gx, gw, seed):
    rng = np.random.default_rng(seed)
    X = rand_ce(rng, M, K, *gx, elo=-10, ehi=-4, zero_groups=0.05)
    W = rand_ce(rng, N, K, *gw, elo=-12, ehi=-6, zero_groups=0.05)
    dY = with_groups(clipped_laplace(rng, (M, N)), 1, 32, lambda g: rng.integers(-16, -10, size=g))
    return X, W, dY


@pytest.mark.parametrize("case", LINEAR_CASES)
def test_linear_fwd(ict, case):
    M, N, K, gx, gw, G = case
    X, W, _ = _linear_inputs(M, N, K, gx, gw, M + N + K)
    ref = oracle.linear_fwd(X, W, 1, G)
    got = ict.linear_fwd(ict.DevCE.from_host(X), ict.DevCE.from_host(W), G).to_host()
    same(got, ref, f"fwd {case}")
    status_ok(ict)


@pytest.mark.parametrize("case", LINEAR_CASES)
def test_linear_bwd_data(ict, case):
    M, N, K, gx, gw, G = case
    X, W, dY = _linear_inputs(M, N, K, gx, gw, M + 2 * N + K)
    ref = oracle.linear_bwd_data(dY, W, 1, G)
    got = ict.linear_bwd_data(ict.DevCE.from_host(dY), ict.DevCE.from_host(W), G).to_host()
    same(got, ref, f"bwd_data {case}")
    status_ok(ict)


@pytest.mark.parametrize("case", LINEAR_CASES)
@pytest.mark.parametrize("per_row", [True, False])
def test_linear_bwd_weight(ict, case, per_row):
    M, N, K, gx, gw, G = case
    X, W, dY = _linear_inputs(M, N, K, gx, gw, M + 3 * N + K)
    g = K if per_row else G
    ref = oracle.linear_bwd_weight(dY, X, 1, g)
    got = ict.linear_bwd_weight(ict.DevCE.from_host(dY), ict.DevCE.from_host(X), g).to_host()
    same(got, ref, f"bwd_weight {case} per_row={per_row}")
    status_ok(ict)


@pytest.mark.parametrize("M,N,K,xg,xspan", [
    (700, 400, 336, 64, (-10, -4)),     # dW 400 x 336: rows span 3 tiles, a 16-column overhang
    (896, 256, 528, 16, (-10, -4)),     # 16-column X groups: column exponents differ within a tile
    (500, 320, 640, 16, (-40, -4)),     # column exponents far apart: the exact per-element path
    (64, 144, 1024, 64, (-10, -4)),     # a 144-row dW with every row spanning 8 tiles
    (256, 4096, 768, 64, (-10, -4)),    # 192 tiles, more than the SMs: the int16 form and its row pass
    (300, 3312, 768, 16, (-40, -4)),    # the same with a ragged last tile and the per-element path
])
def test_linear_bwd_weight_row_groups_across_tiles(ict, M, N, K, xg, xspan):
    """dW = dY^T X with one output group per row spanning several tiles and no split K:
    the Product's int16 round-to-odd output with a need per (row, tile half), then the
    streaming pass that rounds each row to its group exponent, against the oracle (one
    tile per SM, and more tiles than SMs)."""
    rng = np.random.default_rng(M + N + K + xg)
    X = rand_ce(rng, M, K, 1, xg, elo=xspan[0], ehi=xspan[1], zero_groups=0.05)
    dY = with_groups(clipped_laplace(rng, (M, N)), 1, 32, lambda g: rng.integers(-16, -10, size=g))
    ref = oracle.linear_bwd_weight(dY, X, 1, K)
    got = ict.linear_bwd_weight(ict.DevCE.from_host(dY), ict.DevCE.from_host(X), K).to_host()
    same(got, ref, "bwd-weight, row groups across tiles")
    status_ok(ict)


@pytest.mark.parametrize("M,N,K,wspan", [
    (1000, 256, 192, (-12, -6)),    # ragged last M tile, two 128-wide tiles per row band
    (300, 768, 768, (-40, -6)),     # column exponents far apart: the exact per-element path, staged
    (64, 128, 64, (-12, -6)),       # fewer rows than one tile
    (2000, 384, 1024, (-12, -9)),   # the longest contraction on this plan
])
def test_linear_staged_single_cta(ict, M, N, K, wspan):
    """Short contractions with 32-column output groups: four epilogue warpgroups on
    alternate 128-wide tiles of single CTAs, each staging its 128 x 128 output tile in
    shared memory for two TMA stores, against the oracle (forward and backward-data)."""
    rng = np.random.default_rng(M + N + K)
    X = rand_ce(rng, M, K, 1, 64 if K % 64 == 0 else K, elo=-10, ehi=-4, zero_groups=0.05)
    W = rand_ce(rng, N, K, 1, K, elo=wspan[0], ehi=wspan[1], zero_groups=0.05)
    same(ict.linear_fwd(ict.DevCE.from_host(X), ict.DevCE.from_host(W), 32).to_host(), oracle.linear_fwd(X, W, 1, 32),
         "staged fwd")
    dY = with_groups(clipped_laplace(rng, (M, K)), 1, 32, lambda g: rng.integers(-16, -10, size=g))
    Wt = rand_ce(rng, K, N, 1, 64, elo=wspan[0], ehi=wspan[1])
    same(ict.linear_bwd_data(ict.DevCE.from_host(dY), ict.DevCE.from_host(Wt), 32).to_host(),
         oracle.linear_bwd_data(dY, Wt, 1, 32), "staged bwd-data")
    status_ok(ict)


@pytest.mark.parametrize("M,N,K,G,wspan", [
    (12000, 576, 256, 64, (-12, -6)),    # 192-wide pair tiles, ragged last M tile
    (12000, 576, 256, 64, (-40, -6)),    # the same with column exponents far apart: the exact per-element path
    (2600, 768, 256, 64, (-12, -6)),     # 128-wide tiles on single CTAs
    (3000, 512, 256, 128, (-12, -6)),    # 128-column groups (generic epilogue)
    (4200, 1024, 256, 64, (-12, -6)),    # 256-wide pair tiles, four epilogue warpgroups, TMA-store output
    (4100, 1024, 1280, 32, (-12, -6)),   # the same with 32-column groups; ragged last M tile
    (4160, 1024, 384, 64, (-40, -6)),    # staged output from the exact per-element path
])
def test_linear_pair_tiles(ict, M, N, K, G, wspan):
    """Products large enough to run on pairs of CTAs (256-row tiles, tcgen05 cta_group::2)
    against the oracle; on 256-wide tiles the FIT epilogue stages its output in shared
    memory and writes it with TMA stores."""
    rng = np.random.default_rng(M + N + K + G)
    X = rand_ce(rng, M, K, 1, 64, elo=-10, ehi=-4, zero_groups=0.05)
    W = rand_ce(rng, N, K, 1, K, elo=wspan[0], ehi=wspan[1], zero_groups=0.05)
    dY = with_groups(clipped_laplace(rng, (M, N)), 1, 32, lambda g: rng.integers(-16, -10, size=g))
    same(ict.linear_fwd(ict.DevCE.from_host(X), ict.DevCE.from_host(W), G).to_host(), oracle.linear_fwd(X, W, 1, G),
         "pair fwd")
    Wt = rand_ce(rng, N, K, 1, 64, elo=wspan[0], ehi=wspan[1])
    same(ict.linear_bwd_data(ict.DevCE.from_host(dY), ict.DevCE.from_host(Wt), G).to_host(),
         oracle.linear_bwd_data(dY, Wt, 1, G), "pair bwd-data")
    # the weight gradient (N output rows: single CTAs, split-K) of the same operands
    dW = ict.linear_bwd_weight(ict.DevCE.from_host(dY), ict.DevCE.from_host(X)).to_host()
    same(dW, oracle.linear_bwd_weight(dY, X, 1, K), "bwd-weight")
    status_ok(ict)


def test_linear_long_contraction_int64(ict):
    """K far beyond 2^17 products of 127^2: split-K int32 partials, int64 combine."""
    rng = np.random.default_rng(77)
    M, N, K = 160000, 64, 32
    dY = CE(np.full((M, N), 127, np.int8), np.zeros((1, 1), np.int8), M, N)
    X = CE(np.full((M, K), -127, np.int8), np.zeros((1, 1), np.int8), M, K)
    dY.mant[rng.random((M, N)) < 0.01] = -127
    ref = oracle.linear_bwd_weight(dY, X, 1, K)
    got = ict.linear_bwd_weight(ict.DevCE.from_host(dY), ict.DevCE.from_host(X), K).to_host()
    same(got, ref, "long K")
    status_ok(ict)


# ------------------------------------------------------------------ conv


def _conv_inputs(seed, n, h, w, c, k, gx=32):
    rng = np.random.default_rng(seed)
    npix = n * h * w
    X = with_groups(np.where(rng.random((npix, c)) < 0.5, 0, rng.integers(1, 128, size=(npix, c))).astype(np.int8),
                    npix, gx, lambda g: rng.integers(-8, -5, size=g))
    W = rand_ce(rng, k, 9 * c, 1, 9 * c, elo=-10, ehi=-6)
    dY = with_groups(clipped_laplace(rng, (npix, k)), npix, gx, lambda g: rng.integers(-14, -11, size=g))
    return X, W, dY, dict(n=n, h=h, w=w, c=c, k=k, r=3, s=3, stride=1, pad=1)


@pytest.mark.parametrize("shape", [(2, 8, 8, 64, 64), (3, 7, 56, 64, 64), (1, 9, 20, 128, 64),
                                   (2, 5, 12, 64, 128),
                                   # halo tiles with a one-row last tile; and with a box filling its slot
                                   (2, 9, 16, 64, 64), (1, 6, 64, 64, 64),
                                   # backward-data on halo tiles with 128 output channels (128-wide tiles)
                                   (2, 6, 16, 128, 64)])
@pytest.mark.parametrize("global_groups", [True, False])
def test_conv_fwd_and_bwd_data(ict, shape, global_groups):
    X, W, dY, d = _conv_inputs(sum(shape), *shape)
    npix = X.rows
    g_rows = npix if global_groups else 1
    for direction, a, b in ((ict.CONV_FWD, X, W), (ict.CONV_BWD_DATA, dY, W)):
        ref = oracle.conv(direction, d, a, b, g_rows, 32)
        got = ict.conv(direction, d, ict.DevCE.from_host(a), ict.DevCE.from_host(b), g_rows, 32).to_host()
        same(got, ref, f"conv dir={direction} {shape} global={global_groups}")
    # backward-weight: dW rows of r*s*c, per-row groups (or 64-wide groups)
    g = 9 * d["c"] if global_groups else 64
    ref = oracle.conv(ict.CONV_BWD_WEIGHT, d, dY, X, 1, g)
    got = ict.conv(ict.CONV_BWD_WEIGHT, d, ict.DevCE.from_host(dY), ict.DevCE.from_host(X), 1, g).to_host()
    same(got, ref, f"conv bwd-weight {shape} g={g}")
    status_ok(ict)


@pytest.mark.parametrize("n,h,w,c,k,G,wexp", [
    (2, 7, 7, 256, 512, 32, (-10, -6)),    # 16 group columns (forward), 8 (backward-data); two N tiles
    (2, 5, 12, 512, 128, 64, (-10, -6)),   # 512 contracted channels, 8 output groups backward
    (1, 9, 20, 128, 320, 32, (-10, -6)),   # 320 = 256 + 64: a ragged N tile
    (3, 6, 50, 64, 192, 192, (-10, -6)),   # one group over all channels, 100 of 128 tile rows
    (2, 8, 8, 64, 128, 32, (-24, -6)),     # weight exponents 18 apart: exact per-element epilogue
])
def test_conv_all_pixel_groups(ict, n, h, w, c, k, G, wexp):
    """Output groups spanning every pixel (Table 6 convolution, channel groups shared by
    the whole batch): the Product's int16 round-to-odd sums, the per-tile needs and the
    streaming rounding pass, forward and backward-data, with up to 16 group columns, two
    N tiles, a ragged N tile, partial M tiles, all-zero groups and the exact epilogue."""
    rng = np.random.default_rng(n * h + w + c + k + G)
    npix = n * h * w
    X = with_groups(np.where(rng.random((npix, c)) < 0.5, 0, rng.integers(1, 128, size=(npix, c))).astype(np.int8),
                    npix, 32, lambda g: rng.integers(-8, -5, size=g))
    W = rand_ce(rng, k, 9 * c, 1, 9 * c, elo=wexp[0], ehi=wexp[1])
    W.mant[k - 32:] = 0          # the last forward group column is all zero: E_ZERO
    W.exp[k - 32:] = E_ZERO
    dY = with_groups(clipped_laplace(rng, (npix, k)), npix, 32, lambda g: rng.integers(-14, -11, size=g))
    dY.mant[:, :32] = 0          # an all-zero input group: backward-data sums come from the others
    dY.exp[0, 0] = E_ZERO
    d = dict(n=n, h=h, w=w, c=c, k=k, r=3, s=3, stride=1, pad=1)
    for direction, a, b, out_c in ((ict.CONV_FWD, X, W, k), (ict.CONV_BWD_DATA, dY, W, c)):
        g = min(G, out_c)
        ref = oracle.conv(direction, d, a, b, npix, g)
        got = ict.conv(direction, d, ict.DevCE.from_host(a), ict.DevCE.from_host(b), npix, g).to_host()
        same(got, ref, f"conv dir={direction} n{n} {h}x{w} c{c} k{k} G{g}")
    status_ok(ict)


# ------------------------------------------------------------------ GELU


@pytest.mark.parametrize("rows,cols,G,erange", [(64, 768, 32, (-9, -5)), (130, 96, 32, (-30, 3)),
                                                (17, 64, 64, (-127, -100)), (40, 32, 32, (-3, 4))])
def test_gelu(ict, rows, cols, G, erange):
    rng = np.random.default_rng(rows + cols + G)
    H = rand_ce(rng, rows, cols, 1, G, elo=erange[0], ehi=erange[1], zero_groups=0.05)
    dG = rand_ce(rng, rows, cols, 1, G, elo=-16, ehi=-8, zero_groups=0.05)
    dHd, dGd = ict.DevCE.from_host(H), ict.DevCE.from_host(dG)
    same(ict.gelu_fwd(dHd).to_host(), oracle.gelu_fwd(H), "gelu fwd")
    same(ict.gelu_bwd(dHd, dGd).to_host(), oracle.gelu_bwd(H, dG, 1, G), "gelu bwd")
    status_ok(ict)


# ------------------------------------------------------------------ SGD


@pytest.mark.parametrize("rows,cols,G", [(64, 128, 128), (100, 64, 64), (12, 768, 768), (40, 192, 192),
                                         (9, 64, 16), (30, 200, 64)])
@pytest.mark.parametrize("erange", [(-16, -4), (-100, 40)])
def test_sgd(ict, rows, cols, G, erange):
    rng = np.random.default_rng(rows * cols + G + erange[0] + 200)
    W = rand_ce(rng, rows, cols, 1, G, *erange, zero_groups=0.05)
    V = rand_ce(rng, rows, cols, 1, G, *erange, zero_groups=0.3)
    Gr = rand_ce(rng, rows, cols, 1, G, *erange, zero_groups=0.05)
    for mom, lr in (((230, 8), (1, 4)), ((230, 8), (205, 11))):
        try:
            W2, V2 = oracle.sgd_step(W, V, Gr, mom, lr)
        except oracle.OracleError:
            continue
        dW, dV, dG = ict.DevCE.from_host(W), ict.DevCE.from_host(V), ict.DevCE.from_host(Gr)
        ict.ict_sgd_momentum_step(dW, dV, dG, mom, lr)
        same(dV.to_host(), V2, "velocity")
        same(dW.to_host(), W2, "weight")
    status_ok(ict)


def test_sgd_multi_matches_single(ict):
    rng = np.random.default_rng(5)
    shapes = [(64, 128, 128), (10, 64, 64), (3, 768, 64)]
    Ws, Vs, Gs, refs = [], [], [], []
    for r, c, g in shapes:
        W, V, G = (rand_ce(rng, r, c, 1, g, -16, -4) for _ in range(3))
        refs.append(oracle.sgd_step(W, V, G))
        Ws.append(ict.DevCE.from_host(W))
        Vs.append(ict.DevCE.from_host(V))
        Gs.append(ict.DevCE.from_host(G))
    ict.ict_sgd_momentum_step_multi(Ws, Vs, Gs)
    for (W2, V2), dW, dV in zip(refs, Ws, Vs):
        same(dW.to_host(), W2, "multi W")
        same(dV.to_host(), V2, "multi V")
    status_ok(ict)


# ------------------------------------------------------------------ errors


def test_argument_errors_return_before_launch(ict):
    X = ict.DevCE.from_host(CE(np.zeros((64, 128), np.int8), np.zeros((1, 1), np.int8), 64, 128))
    W = ict.DevCE.from_host(CE(np.zeros((64, 96), np.int8), np.zeros((64, 1), np.int8), 1, 96))
    Y = ict.DevCE.empty(64, 64, 1, 32)
    with pytest.raises(ict.IctError) as ei:
        ict.ict_linear_fwd(X, W, Y)
    assert ei.value.code == 1
    Yb = ict.DevCE.empty(64, 64, 2, 32)  # 2-row output groups are not row-local
    W2 = ict.DevCE.from_host(CE(np.zeros((64, 128), np.int8), np.zeros((64, 1), np.int8), 1, 128))
    with pytest.raises(ict.IctError) as ei:
        ict.ict_linear_fwd(X, W2, Yb)
    assert ei.value.code == 2
    Y = ict.DevCE.empty(64, 64, 1, 32)
    need = ict.ict_linear_workspace(ict.OP_LINEAR_FWD, X, W2, Y)
    assert need == 0  # both operands uniform along K, fused epilogue
    status_ok(ict)


def test_bounded_wait_timeout_leaves_context_usable(ict):
    """A wait that nothing completes runs out its bound, raises ICT_ERR_DEVICE_TIMEOUT in
    the status word and returns; the next calls run normally and bit-exact."""
    ict.ict_get_device_status()  # clear
    ict.ict_selftest_wait_timeout(2_000_000)  # 2 ms
    code, raw = ict.ict_get_device_status()
    assert code == 7, (code, raw)  # ICT_ERR_DEVICE_TIMEOUT
    from integer_only_nn_02_b200 import workloads as wl
    cfg = wl.single_linear(seed=3)
    X, W = cfg["X"], cfg["W"]
    Y = ict.linear_fwd(ict.DevCE.from_host(X), ict.DevCE.from_host(W), 32)
    ref = oracle.linear_fwd(X, W, 1, 32)
    h = Y.to_host()
    assert np.array_equal(h.mant, ref.mant) and np.array_equal(h.exp, ref.exp)
    code, raw = ict.ict_get_device_status()
    assert code == 0, (code, raw)


@pytest.mark.parametrize("r", [1, 5, 7])
@pytest.mark.parametrize("global_groups", [True, False])
def test_conv_other_odd_filters(ict, r, global_groups):
    """'Same' convolutions with other odd square filters (1x1: pad 0; 5x5: pad 2; 7x7:
    pad 3), all three directions, through the same implicit-GEMM kernels."""
    rng = np.random.default_rng(50 + r + global_groups)
    n, h, w, c, k = 2, 9, 12, 64, 128
    npix = n * h * w
    X = with_groups(np.where(rng.random((npix, c)) < 0.5, 0, rng.integers(1, 128, size=(npix, c))).astype(np.int8),
                    npix, 32, lambda g: rng.integers(-8, -5, size=g))
    W = rand_ce(rng, k, r * r * c, 1, r * r * c, elo=-10, ehi=-6)
    dY = with_groups(clipped_laplace(rng, (npix, k)), npix, 32, lambda g: rng.integers(-14, -11, size=g))
    d = dict(n=n, h=h, w=w, c=c, k=k, r=r, s=r, stride=1, pad=(r - 1) // 2)
    g_rows = npix if global_groups else 1
    for direction, a, b in ((ict.CONV_FWD, X, W), (ict.CONV_BWD_DATA, dY, W)):
        ref = oracle.conv(direction, d, a, b, g_rows, 32)
        got = ict.conv(direction, d, ict.DevCE.from_host(a), ict.DevCE.from_host(b), g_rows, 32).to_host()
        same(got, ref, f"conv {r}x{r} dir={direction} global={global_groups}")
    ref = oracle.conv(ict.CONV_BWD_WEIGHT, d, dY, X, 1, r * r * c)
    got = ict.conv(ict.CONV_BWD_WEIGHT, d, ict.DevCE.from_host(dY), ict.DevCE.from_host(X), 1, r * r * c).to_host()
    same(got, ref, f"conv {r}x{r} bwd-weight")
    status_ok(ict)


@pytest.mark.parametrize("n,h,w,c,P,G,k", [
    (2, 32, 32, 16, 16, 16, 64),     # channel groups of 16
    (2, 16, 48, 64, 8, 32, 96),      # two channel groups
    (2, 32, 32, 3, 16, 3, 64),       # RGB, one exponent, pixels packed (ld = 3)
])
def test_patch_embedding(ict, n, h, w, c, P, G, k):
    """ict_patchify then ict_linear_fwd equals the oracle's P x P, stride P convolution,
    and ict_linear_bwd_weight on the patches equals the convolution's weight gradient."""
    import torch

    rng = np.random.default_rng(n + h + c + P)
    npix = n * h * w
    X = with_groups(rng.integers(-127, 128, size=(npix, c)).astype(np.int8), npix, G,
                    lambda s: rng.integers(-9, -5, size=s))
    W = rand_ce(rng, k, P * P * c, 1, P * P * c, elo=-10, ehi=-6)
    d = dict(n=n, h=h, w=w, c=c, k=k, r=P, s=P, stride=P, pad=0)
    if c % 16:
        Xd = ict.DevCE(torch.from_numpy(X.mant.copy()).cuda(), torch.from_numpy(X.exp.copy()).cuda(), npix, G, cols=c)
    else:
        Xd = ict.DevCE.from_host(X)
    patches = ict.patchify(Xd, n, h, w, P)
    Y = ict.linear_fwd(patches, ict.DevCE.from_host(W), 32)
    same(Y.to_host(), oracle.conv(0, d, X, W, 1, 32), f"patch embedding {n}x{h}x{w}x{c} P={P}")
    # the patches themselves: the oracle's row alignment of X (one target for every
    # pixel), gathered into (dy, dx, channel) rows by reshaping
    xa, xe = oracle.align(X, axis=1)
    rows = n * (h // P) * (w // P)
    ref_m = xa.reshape(n, h // P, P, w // P, P, c).transpose(0, 1, 3, 2, 4, 5).reshape(rows, P * P * c)
    got = patches.to_host()
    assert np.array_equal(got.mant, ref_m) and int(got.exp[0, 0]) == int(xe[0]), "patches"
    # weight gradient on the patches
    dY = rand_ce(rng, rows, k, 1, 32, elo=-14, ehi=-10)
    ref_p = CE(np.ascontiguousarray(ref_m), np.array([[xe[0]]], np.int8), rows, P * P * c)
    dW = ict.linear_bwd_weight(ict.DevCE.from_host(dY), patches)
    same(dW.to_host(), oracle.linear_bwd_weight(dY, ref_p, 1, P * P * c), "patch embedding dW")
    status_ok(ict)


@pytest.mark.parametrize("geom", [dict(), dict(stride=2), dict(r=5, pad=2), dict(r=1, pad=0)])
@pytest.mark.parametrize("global_groups", [True, False])
def test_depthwise(ict, geom, global_groups):
    """Depthwise convolution (one filter per channel) in the three directions against the
    oracle, bit for bit."""
    rng = np.random.default_rng(60 + geom.get("r", 3) + geom.get("stride", 1) + global_groups)
    n, h, w, c = 2, 9, 10, 96
    r, pad, stride = geom.get("r", 3), geom.get("pad", 1), geom.get("stride", 1)
    P, Q = (h + 2 * pad - r) // stride + 1, (w + 2 * pad - r) // stride + 1
    X = rand_ce(rng, n * h * w, c, n * h * w, 32, elo=-8, ehi=-5, zero_groups=0.1)
    W = rand_ce(rng, c, r * r, 1, r * r, elo=-9, ehi=-6)
    dY = rand_ce(rng, n * P * Q, c, n * P * Q, 32, elo=-14, ehi=-11, zero_groups=0.1)
    d = dict(n=n, h=h, w=w, c=c, k=c, r=r, s=r, stride=stride, pad=pad)
    dev = ict.DevCE.from_host
    for direction, a, rows in ((0, X, n * P * Q), (1, dY, n * h * w)):
        g_rows = rows if global_groups else 1
        got = ict.depthwise(direction, d, dev(a), dev(W), g_rows, 32).to_host()
        same(got, oracle.depthwise(direction, d, a, W, g_rows, 32), f"depthwise dir={direction} {geom}")
    got = ict.depthwise(2, d, dev(dY), dev(X), 1, r * r).to_host()
    same(got, oracle.depthwise(2, d, dY, X, 1, r * r), f"depthwise dW {geom}")
    status_ok(ict)
