"""GPU parity of the pointwise primitives against the CPU oracle, bit for bit: ReLU /
ReLU6 forward and backward (the Clip primitive) and the Sum primitive (residual add),
on row-local and all-row (pixel-uniform) group partitions, with exponents chosen to
reach every ReLU6 bound case and every exponent-gap regime of the Sum (int32 fast path,
exact int64 path, sticky path beyond a 32-bit gap)."""
import numpy as np
import pytest

import oracle
from integer_only_nn_02_b200.workloads import CE, E_ZERO
from tests.test_oracle_pins import rand_ce

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ict():
    from integer_only_nn_02_b200 import ict as _ict

    return _ict


def same(got: CE, ref: CE, what=""):
    assert got.mant.shape == ref.mant.shape, what
    bad = np.argwhere(got.mant != ref.mant)
    assert bad.size == 0, f"{what}: {len(bad)} mantissas differ, first {bad[:5].tolist()}"
    bad = np.argwhere(got.exp != ref.exp)
    assert bad.size == 0, f"{what}: {len(bad)} exponents differ, first {bad[:5].tolist()}"


def status_ok(ict):
    code, raw = ict.ict_get_device_status()
    assert code == 0, (code, raw)


CLIP_CASES = [  # rows, cols, groups
    (300, 192, (1, 32)),
    (129, 768, (1, 768)),     # one group per row
    (1000, 64, (1000, 16)),   # pixel-uniform channel groups
    (7, 48, (7, 16)),
    (2048, 256, (1, 64)),
]


@pytest.mark.parametrize("case", CLIP_CASES)
@pytest.mark.parametrize("six", [False, True])
def test_relu_fwd_bwd(ict, case, six):
    rows, cols, g = case
    rng = np.random.default_rng(rows + cols + six)
    X = rand_ce(rng, rows, cols, *g, elo=-8, ehi=4, zero_groups=0.1)  # every ReLU6 bound case
    dY = rand_ce(rng, rows, cols, 1, 32 if cols % 32 == 0 else 16, elo=-20, ehi=-8, zero_groups=0.05)
    dX_ = ict.DevCE.from_host
    got = ict.relu_fwd(dX_(X), six).to_host()
    same(got, oracle.relu_fwd(X, six), f"fwd {case} six={six}")
    got = ict.relu_bwd(dX_(X), dX_(dY), six).to_host()
    same(got, oracle.relu_bwd(X, dY, six), f"bwd {case} six={six}")
    status_ok(ict)


SUM_CASES = [  # rows, cols, groups
    (300, 192, (1, 32)),
    (130, 768, (1, 64)),
    (64, 3072, (1, 3072)),    # one group per row: 32 lanes per group
    (5, 16, (1, 16)),
    (60, 256, (1, 128)),      # 8 lanes per group
    (70, 256, (1, 256)),      # 16 lanes
    (50, 512, (1, 512)),      # 32 lanes, one vector each
    (20, 1008, (1, 1008)),    # 32 lanes, two vectors each, the last lanes short
    (33, 2048, (1, 2048)),    # 32 lanes, four vectors each
    (2000, 64, (2000, 32)),   # pixel-uniform channel groups: two passes
    (777, 256, (777, 16)),
]
GAPS = [((-12, -2), (-12, -2)), ((-40, -30), (-5, 5)), ((-127, -90), (10, 40))]


@pytest.mark.parametrize("case", SUM_CASES)
@pytest.mark.parametrize("gaps", GAPS)
def test_sum(ict, case, gaps):
    rows, cols, g = case
    rng = np.random.default_rng(rows * 3 + cols + abs(gaps[0][0]))
    X = rand_ce(rng, rows, cols, *g, *gaps[0], zero_groups=0.1)
    Y = rand_ce(rng, rows, cols, *g, *gaps[1], zero_groups=0.1)
    d = ict.DevCE.from_host
    got = ict.sum_(d(X), d(Y)).to_host()
    same(got, oracle.sum_(X, Y, *g), f"sum {case} gaps={gaps}")
    got = ict.sum_(d(Y), d(X)).to_host()  # the Sum is symmetric
    same(got, oracle.sum_(X, Y, *g), f"sum (swapped) {case} gaps={gaps}")
    status_ok(ict)


def test_sum_edge_cases(ict):
    import torch

    d = ict.DevCE.from_host
    # both terms zero everywhere: E_ZERO groups
    Z = CE(np.zeros((40, 64), np.int8), np.full((40, 2), E_ZERO, np.int8), 1, 32)
    same(ict.sum_(d(Z), d(Z)).to_host(), oracle.sum_(Z, Z, 1, 32), "zeros")
    # x + (-x) = 0
    rng = np.random.default_rng(9)
    X = rand_ce(rng, 40, 64, 1, 32)
    N = CE((-X.mant.astype(np.int16)).astype(np.int8), X.exp.copy(), 1, 32)
    got = ict.sum_(d(X), d(N)).to_host()
    assert (got.mant == 0).all() and (got.exp == E_ZERO).all()
    # an empty tensor is a no-op
    E = ict.DevCE.empty(0, 64, 1, 32)
    ict.ict_sum(E, E, ict.DevCE.empty(0, 64, 1, 32))
    # mismatched partitions are refused
    A = d(rand_ce(rng, 40, 64, 1, 32))
    B = d(rand_ce(rng, 40, 64, 1, 16))
    with pytest.raises(ict.IctError) as ei:
        ict.ict_sum(A, B, ict.DevCE.empty(40, 64, 1, 32))
    assert ei.value.code == 2  # ICT_ERR_LAYOUT
    torch.cuda.synchronize()
    status_ok(ict)


def test_resnet_residual_and_relu_full_size(ict):
    """The ResNet-18 stage-1 block tail at full size: residual add of two
    128 x 56 x 56 x 64 activations (channel groups of 32 spanning all pixels), then ReLU,
    then the backward mask."""
    from integer_only_nn_02_b200 import workloads as wl

    cfg = wl.resnet18_conv3x3(seed=4)
    X, dY = cfg["X"], cfg["dY"]
    rng = np.random.default_rng(12)
    R = rand_ce(rng, X.rows, X.cols, X.rows, 32, elo=-9, ehi=-6)
    d = ict.DevCE.from_host
    S = ict.sum_(d(X), d(R))
    same(S.to_host(), oracle.sum_(X, R, X.rows, 32), "residual add")
    Sh = S.to_host()
    A = ict.relu_fwd(S)
    same(A.to_host(), oracle.relu_fwd(Sh), "relu")
    same(ict.relu_bwd(S, d(dY)).to_host(), oracle.relu_bwd(Sh, dY), "relu bwd")
    status_ok(ict)


@pytest.mark.parametrize("case", [(300, 192, (1, 32)), (2000, 64, (2000, 32)), (33, 2048, (1, 2048))])
@pytest.mark.parametrize("xw,yw", [((1, 0), (105, 20)), ((-3, 1), (230, 8)), ((512, 0), (-512, 30)),
                                   ((0, 0), (7, 3))])
def test_sum_scaled(ict, case, xw, yw):
    rows, cols, g = case
    rng = np.random.default_rng(rows + cols + xw[0] + yw[1])
    X = rand_ce(rng, rows, cols, *g, elo=-20, ehi=-8, zero_groups=0.1)
    Y = rand_ce(rng, rows, cols, *g, elo=-12, ehi=0, zero_groups=0.1)
    d = ict.DevCE.from_host
    Z = ict.DevCE.empty(rows, cols, *g)
    ict.ict_sum_scaled(d(X), xw, d(Y), yw, Z, ict._ws(ict.ict_sum_workspace(d(X), d(Y), Z)))
    same(Z.to_host(), oracle.sum_scaled(X, xw, Y, yw, *g), f"sum_scaled {case} {xw} {yw}")
    status_ok(ict)


def test_sgd_with_weight_decay(ict):
    """SGD with momentum and weight decay 1e-4 (105 2^-20): the weighted Sum G + lambda W
    then the momentum step, two steps, against the oracle's composition."""
    rng = np.random.default_rng(77)
    rows, cols, G = 96, 256, 64
    W = rand_ce(rng, rows, cols, 1, G, elo=-9, ehi=-6)
    V = rand_ce(rng, rows, cols, 1, G, elo=-14, ehi=-10, zero_groups=0.2)
    Gr = rand_ce(rng, rows, cols, 1, G, elo=-16, ehi=-12, zero_groups=0.05)
    d = ict.DevCE.from_host
    Wd, Vd, Gd = d(W), d(V), d(Gr)
    Gw = ict.DevCE.empty(rows, cols, 1, G)
    w_ref, v_ref = W, V
    for _ in range(2):
        ict.ict_sgd_momentum_step_wd(Wd, Vd, Gd, Gw, wd=(105, 20), mom=(230, 8), lr=(1, 4))
        g_ref = oracle.sum_scaled(Gr, (1, 0), w_ref, (105, 20), 1, G)
        w_ref, v_ref = oracle.sgd_step(w_ref, v_ref, g_ref, (230, 8), (1, 4))
    same(Wd.to_host(), w_ref, "W")
    same(Vd.to_host(), v_ref, "V")
    status_ok(ict)


POOL_CASES = [  # n, h, w, c, K, input groups (forward), output groups
    (2, 4, 6, 32, 2, 16, (1, 16)),
    (1, 6, 6, 16, 3, 16, (4, 16)),
    (3, 7, 7, 32, 7, 32, (1, 32)),
    (32, 7, 7, 512, 7, 32, (1, 32)),      # ResNet-18 head: global pool into the classifier's rows
    (4, 14, 14, 64, 2, 32, ("all", 32)),  # output groups spanning all pixels
]


@pytest.mark.parametrize("case", POOL_CASES)
def test_avgpool(ict, case):
    n, h, w, c, K, gin, og = case
    rng = np.random.default_rng(n + h + c + K)
    npix, nout = n * h * w, n * (h // K) * (w // K)
    X = rand_ce(rng, npix, c, npix, gin, elo=-9, ehi=-5, zero_groups=0.1)
    g_rows = nout if og[0] == "all" else og[0]
    d = ict.DevCE.from_host
    got = ict.avgpool_fwd(d(X), n, h, w, K, g_rows, og[1]).to_host()
    same(got, oracle.avgpool_fwd(X, n, h, w, K, g_rows, og[1]), f"avgpool fwd {case}")
    # backward: dY with the output's geometry, dX with pixel-uniform or row-local groups
    dY = rand_ce(rng, nout, c, g_rows, og[1], elo=-16, ehi=-8, zero_groups=0.1)
    for dxg in ((npix, gin), (1, gin)):
        got = ict.avgpool_bwd(d(dY), n, h, w, K, *dxg).to_host()
        same(got, oracle.avgpool_bwd(dY, n, h, w, K, *dxg), f"avgpool bwd {case} {dxg}")
    status_ok(ict)


@pytest.mark.parametrize("case", [(300, 192, (1, 32)), (2000, 64, (2000, 32)), (33, 2048, (1, 2048))])
@pytest.mark.parametrize("act", [1, 2])
def test_sum_act_fused(ict, case, act):
    """Residual add and ReLU / ReLU6 in one rounding pass; the backward mask taken from the
    fused output equals the one taken from the Sum before the activation."""
    rows, cols, g = case
    rng = np.random.default_rng(rows + cols + act)
    X = rand_ce(rng, rows, cols, *g, elo=-6, ehi=3, zero_groups=0.1)  # every ReLU6 bound case
    Y = rand_ce(rng, rows, cols, *g, elo=-8, ehi=1, zero_groups=0.1)
    dA = rand_ce(rng, rows, cols, 1, 16, elo=-16, ehi=-8)
    d = ict.DevCE.from_host
    Z = ict.DevCE.empty(rows, cols, *g)
    ict.ict_sum_act(d(X), d(Y), Z, act, ict._ws(ict.ict_sum_workspace(d(X), d(Y), Z)))
    S = oracle.sum_(X, Y, *g)
    six = act == 2
    same(Z.to_host(), oracle.relu_fwd(S, six), f"sum_act {case} act={act}")
    same(ict.relu_bwd(Z, d(dA), six).to_host(), oracle.relu_bwd(S, dA, six), f"mask from fused output {case}")
    status_ok(ict)


@pytest.mark.parametrize("global_groups", [True, False])
@pytest.mark.parametrize("act", [0, 1, 2])
def test_conv_fwd_act_fused(ict, global_groups, act):
    from integer_only_nn_02_b200.workloads import with_groups

    rng = np.random.default_rng(40 + act + global_groups)
    n, h, w, c, k, G = 2, 8, 8, 64, 64, 32
    npix = n * h * w
    X = with_groups(rng.integers(-127, 128, size=(npix, c)).astype(np.int8), npix, G,
                    lambda s: rng.integers(-6, -2, size=s))
    W = rand_ce(rng, k, 9 * c, 1, 9 * c, elo=-9, ehi=-6)
    d = dict(n=n, h=h, w=w, c=c, k=k, r=3, s=3, stride=1, pad=1)
    g_rows = npix if global_groups else 1
    Y = ict.DevCE.empty(npix, k, g_rows, G)
    ws = ict._ws(ict.ict_conv_workspace(0, d))
    ict.ict_conv_fwd_act(d, ict.DevCE.from_host(X), ict.DevCE.from_host(W), Y, act, ws)
    ref = oracle.conv(0, d, X, W, g_rows, G)
    if act:
        ref = oracle.relu_fwd(ref, act == 2)
    same(Y.to_host(), ref, f"conv fwd act={act} global={global_groups}")
    status_ok(ict)
