"""GPU parity of the data-parallel backward weight (ict_linear_bwd_weight_targets /
_partial + ict_requant): a batch split into shards, each shard's steps run on the one
GPU in turn, the MAX of the targets and the SUM of the integer sums taken by the test
between them (what the all-reduces of integer_only_nn_02_b200.dp do across GPUs).  The
result must equal the single-device oracle on the whole batch, bit for bit; at the
ViT-B size, where the oracle is too slow, it must equal the single-device GPU call,
which the parity suite checks against the oracle at that size."""
import numpy as np
import pytest

import oracle
from integer_only_nn_02_b200.workloads import CE
from tests.test_oracle_pins import rand_ce

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ict():
    from integer_only_nn_02_b200 import ict as _ict

    return _ict


def same(got: CE, ref: CE, what=""):
    bad = np.argwhere(got.mant != ref.mant)
    assert bad.size == 0, f"{what}: {len(bad)} mantissas differ, first {bad[:5].tolist()}"
    bad = np.argwhere(got.exp != ref.exp)
    assert bad.size == 0, f"{what}: {len(bad)} exponents differ, first {bad[:5].tolist()}"


def shard(t: CE, a: int, b: int) -> CE:
    return CE(t.mant[a:b].copy(), t.exp[a:b].copy(), 1, t.g_cols)


def split_batch_dw(ict, dY: CE, X: CE, cuts, bits, check_targets=True):
    """The five steps of the split-batch backward weight, shards run one after another."""
    import torch

    M, N = dY.cols, X.cols
    parts = [(shard(dY, a, b), shard(X, a, b)) for a, b in zip(cuts[:-1], cuts[1:])]
    devs = [(ict.DevCE.from_host(p), ict.DevCE.from_host(q)) for p, q in parts]
    ws = torch.empty(max(ict.ict_linear_bwd_weight_partial_workspace(a, b) for a, b in devs), dtype=torch.uint8,
                     device="cuda")
    targets = []
    for (hdy, hx), (ddy, dx) in zip(parts, devs):
        e_dy = torch.empty(M, dtype=torch.int8, device="cuda")
        e_x = torch.empty(N, dtype=torch.int8, device="cuda")
        ict.ict_linear_bwd_weight_targets(ddy, dx, e_dy, e_x, ws)
        if check_targets:
            assert np.array_equal(e_dy.cpu().numpy(), oracle.align(hdy, 0)[1]), "targets of dY"
            assert np.array_equal(e_x.cpu().numpy(), oracle.align(hx, 0)[1]), "targets of X"
        targets.append(torch.cat([e_dy, e_x]))
    e = torch.stack(targets).max(dim=0).values.contiguous()  # the MAX all-reduce
    e_dy, e_x = e[:M], e[M:]
    dt = torch.int32 if bits == 32 else torch.int64
    acc = torch.zeros((M, N), dtype=dt, device="cuda")
    part = torch.empty((M, N), dtype=dt, device="cuda")
    for ddy, dx in devs:
        part.fill_(0x5A5A)  # the call must write every element
        ict.ict_linear_bwd_weight_partial(ddy, dx, e_dy, e_x, part, ws)
        acc += part  # the SUM all-reduce
    dW = ict.DevCE.empty(M, N, 1, N)
    ict.ict_requant(acc, dW, 0, e_dy, e_x)
    torch.cuda.synchronize()
    code, raw = ict.ict_get_device_status()
    assert code == 0, (code, raw)
    return dW.to_host()


@pytest.mark.parametrize("K,M,N,g,cuts,bits", [
    (1000, 192, 768, 32, [0, 337, 337, 1000], 32),   # three shards, one of them empty
    (1000, 192, 768, 32, [0, 500, 1000], 64),
    (300, 64, 48, 16, [0, 7, 300], 64),              # a 7-row shard: one ragged tile
    (2100, 128, 96, 32, [0, 1, 1024, 2100], 32),     # a one-row shard
])
def test_split_batch_matches_oracle(ict, K, M, N, g, cuts, bits):
    rng = np.random.default_rng(K + M + N)
    dY = rand_ce(rng, K, M, 1, g, elo=-14, ehi=-3, zero_groups=0.1)
    X = rand_ce(rng, K, N, 1, g, elo=-9, ehi=-1, zero_groups=0.1)
    got = split_batch_dw(ict, dY, X, cuts, bits)
    same(got, oracle.linear_bwd_weight(dY, X), f"split {cuts}")


def test_split_batch_vit_b_matches_single_device(ict):
    """ViT-B fc1 backward weight (12 608 tokens, 3072 x 768) split over four shards."""
    from integer_only_nn_02_b200 import workloads as wl

    cfg = wl.vit_b_linear_trio(seed=3)
    dH, X = cfg["dY1"], cfg["X"]
    K = X.rows
    got = split_batch_dw(ict, dH, X, [0, 3152, 6304, 9456, K], 32, check_targets=False)
    dW = ict.linear_bwd_weight(ict.DevCE.from_host(dH), ict.DevCE.from_host(X))
    same(got, dW.to_host(), "ViT-B fc1 dW")


def test_linear_weight_grad_one_rank(ict):
    """dp.LinearWeightGrad without a process group (one rank) is ict_linear_bwd_weight."""
    from integer_only_nn_02_b200 import dp

    rng = np.random.default_rng(5)
    dY = ict.DevCE.from_host(rand_ce(rng, 777, 192, 1, 32, elo=-14, ehi=-3, zero_groups=0.05))
    X = ict.DevCE.from_host(rand_ce(rng, 777, 768, 1, 32, elo=-9, ehi=-1, zero_groups=0.05))
    for total in (777, None):
        g = dp.LinearWeightGrad(dY, X, total_rows=total)
        assert g.bits == (32 if total else 64)
        dW = ict.DevCE.empty(192, 768, 1, 768)
        g(dY, X, dW)
        same(dW.to_host(), ict.linear_bwd_weight(dY, X).to_host(), f"bits {g.bits}")


# ------------------------------------------------------------------ convolution


def _rows(t: CE, a: int, b: int) -> CE:
    """Pixel rows [a, b) of an activation whose groups span all pixels (one exponent row)."""
    return CE(t.mant[a:b].copy(), t.exp.copy(), max(1, b - a), t.g_cols)


@pytest.mark.parametrize("shape,G,cuts", [
    ((3, 8, 8, 64, 64), 32, [0, 1, 3]),
    ((4, 7, 20, 128, 256), 32, [0, 2, 3, 4]),       # eight output group columns
    ((5, 6, 12, 64, 128), 64, [0, 1, 2, 5]),
])
def test_conv_split_batch_matches_oracle(ict, shape, G, cuts):
    """Images split between shards: forward and backward-data rounding with the MAX of the
    shards' group needs, backward weight from the SUM of their int64 sums."""
    import torch

    from integer_only_nn_02_b200 import dp
    from integer_only_nn_02_b200.workloads import clipped_laplace, relu_like, with_groups

    n, h, w, c, k = shape
    rng = np.random.default_rng(sum(shape) + G)
    npix = n * h * w
    X = with_groups(relu_like(rng, (npix, c)), npix, G, lambda g: rng.integers(-9, -5, size=g))
    W = rand_ce(rng, k, 9 * c, 1, 64, elo=-11, ehi=-6, zero_groups=0.05)
    dY = with_groups(clipped_laplace(rng, (npix, k)), npix, G, lambda g: rng.integers(-14, -11, size=g))
    d_full = dict(n=n, h=h, w=w, c=c, k=k, r=3, s=3, stride=1, pad=1)
    hw = h * w
    shards = list(zip(cuts[:-1], cuts[1:]))
    Wd = ict.DevCE.from_host(W)
    for direction, act, out_c in ((ict.CONV_FWD, X, k), (ict.CONV_BWD_DATA, dY, c)):
        parts = []
        for i0, i1 in shards:
            d_r = dict(d_full, n=i1 - i0)
            a_r = ict.DevCE.from_host(_rows(act, i0 * hw, i1 * hw))
            out_r = ict.DevCE.empty((i1 - i0) * hw, out_c, (i1 - i0) * hw, G)
            split = dp.ConvSplit(direction, d_r, a_r, Wd, out_r)
            parts.append((d_r, a_r, out_r, split))
        for d_r, a_r, out_r, split in parts:  # phase 1 on every shard
            ict.ict_conv_split_begin(direction, d_r, a_r, Wd, out_r, split.need, split.ws)
        need = torch.stack([p[3].need for p in parts]).max(dim=0).values  # the MAX all-reduce
        for d_r, a_r, out_r, split in parts:  # phase 2 with the whole batch's needs
            ict.ict_conv_split_end(direction, d_r, a_r, Wd, out_r, need, split.ws)
        hosts = [p[2].to_host() for p in parts]
        got = CE(np.concatenate([t.mant for t in hosts]), hosts[0].exp, npix, G)
        for t in hosts[1:]:
            assert np.array_equal(t.exp, hosts[0].exp), "every shard rounds with the same exponents"
        same(got, oracle.conv(direction, d_full, act, W, npix, G), f"dir={direction} {shape} cuts={cuts}")
    # backward weight
    RSC = 9 * c
    acc = torch.zeros((k, RSC), dtype=torch.int64, device="cuda")
    for i0, i1 in shards:
        d_r = dict(d_full, n=i1 - i0)
        g = dp.ConvWeightGrad(d_r)
        g.acc.fill_(77)  # the call must write every sum
        ict.ict_conv_bwd_weight_partial(d_r, ict.DevCE.from_host(_rows(dY, i0 * hw, i1 * hw)),
                                        ict.DevCE.from_host(_rows(X, i0 * hw, i1 * hw)), g.acc, g.e_k, g.e_rsc, g.ws)
        acc += g.acc  # the SUM all-reduce
    dW = ict.DevCE.empty(k, RSC, 1, RSC)
    ict.ict_requant(acc, dW, 0, g.e_k, g.e_rsc)
    same(dW.to_host(), oracle.conv(ict.CONV_BWD_WEIGHT, d_full, dY, X, 1, RSC), f"dW {shape} cuts={cuts}")
    torch.cuda.synchronize()
    code, raw = ict.ict_get_device_status()
    assert code == 0, (code, raw)


def test_conv_split_classes_one_rank(ict):
    """dp.ConvSplit and dp.ConvWeightGrad without a process group equal the single calls."""
    from integer_only_nn_02_b200 import dp
    from integer_only_nn_02_b200.workloads import clipped_laplace, relu_like, with_groups

    rng = np.random.default_rng(31)
    n, h, w, c, k, G = 2, 8, 8, 64, 64, 32
    npix = n * h * w
    d = dict(n=n, h=h, w=w, c=c, k=k, r=3, s=3, stride=1, pad=1)
    X = ict.DevCE.from_host(with_groups(relu_like(rng, (npix, c)), npix, G, lambda g: rng.integers(-9, -5, size=g)))
    W = ict.DevCE.from_host(rand_ce(rng, k, 9 * c, 1, 64, elo=-11, ehi=-6))
    dY = ict.DevCE.from_host(with_groups(clipped_laplace(rng, (npix, k)), npix, G,
                                         lambda g: rng.integers(-14, -11, size=g)))
    Y = ict.DevCE.empty(npix, k, npix, G)
    dp.ConvSplit(ict.CONV_FWD, d, X, W, Y)(X, W, Y)
    same(Y.to_host(), ict.conv(ict.CONV_FWD, d, X, W, npix, G).to_host(), "fwd")
    dW = ict.DevCE.empty(k, 9 * c, 1, 9 * c)
    dp.ConvWeightGrad(d)(dY, X, dW)
    same(dW.to_host(), ict.conv(ict.CONV_BWD_WEIGHT, d, dY, X, 1, 9 * c).to_host(), "dW")


def test_sharded_update_one_rank_and_row_blocks(ict):
    """dp.ShardedLinearUpdate on one rank equals ict_linear_bwd_weight + the SGD step; the
    per-rank pieces it runs (FIT of a block of rows of the sums, SGD on a block of rows of
    W and V) run here on two row blocks of one GPU and give the same W and V."""
    import torch

    from integer_only_nn_02_b200 import dp

    rng = np.random.default_rng(21)
    K, M, N, G = 777, 192, 768, 768
    dYh = rand_ce(rng, K, M, 1, 32, elo=-14, ehi=-3, zero_groups=0.05)
    Xh = rand_ce(rng, K, N, 1, 32, elo=-9, ehi=-1, zero_groups=0.05)
    Wh = rand_ce(rng, M, N, 1, G, elo=-9, ehi=-6)
    Vh = rand_ce(rng, M, N, 1, G, elo=-14, ehi=-10)
    d = ict.DevCE.from_host
    dY, X = d(dYh), d(Xh)
    upd = dp.ShardedLinearUpdate(dY, X, d(Wh), d(Vh), total_rows=K)
    upd(dY, X)
    W2, V2 = oracle.sgd_step(Wh, Vh, oracle.linear_bwd_weight(dYh, Xh, 1, G))
    same(upd.W.to_host(), W2, "W, one rank")
    same(upd.V_shard.to_host(), V2, "V, one rank")
    # the same rounds on two row blocks
    g = dp.LinearWeightGrad(dY, X, total_rows=K)
    ict.ict_linear_bwd_weight_targets(dY, X, g.e_dy, g.e_x, g.ws)
    ict.ict_linear_bwd_weight_partial(dY, X, g.e_dy, g.e_x, g.acc, g.ws)
    Wd, Vd = d(Wh), d(Vh)
    for r0, r1 in ((0, 96), (96, M)):
        rows = lambda t: ict.DevCE(t.mant[r0:r1], t.exp[r0:r1], 1, G, cols=N)
        dWs = ict.DevCE.empty(r1 - r0, N, 1, G)
        ict.ict_requant(g.acc[r0:r1], dWs, 0, g.e_dy[r0:r1], g.e_x)
        ict.ict_sgd_momentum_step(rows(Wd), rows(Vd), dWs)
    torch.cuda.synchronize()
    same(Wd.to_host(), W2, "W, two row blocks")
    same(Vd.to_host(), V2, "V, two row blocks")
    code, raw = ict.ict_get_device_status()
    assert code == 0, (code, raw)
