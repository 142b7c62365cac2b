"""Full-size parity at the benchmark configurations, in the launch configurations
bench.py times (same shapes and group geometries, hence the same tiling plans).

* single linear layer 64x128: the whole training step, every tensor.
* ViT-Ti MLP block (12608 tokens): the whole step, every tensor (the oracle runs the
  full step on the host cores in a few seconds).
* ResNet-18 3x3 conv (128x56x56x64): all three directions, every output.
* ViT-B linear trio (12608 x 768 x 3072): fc1 forward and both weight gradients in
  full (every row of dW1 3072 x 768 and dW2 768 x 3072, each a contraction over all
  12608 tokens), fc2 forward and both backward-data Products on sampled rows (row
  alignment and (1, 64) output groups are row-local, so a row subset is exact).
* ResNet-50 SGD arena (25 557 032 parameters): the whole update.
* ResNet-18 block tail (residual add fused with ReLU, ReLU backward, gradient merge on
  128x56x56x64): every output.
"""
import numpy as np
import pytest

import oracle
from integer_only_nn_02_b200 import workloads as wl
from integer_only_nn_02_b200.workloads import CE

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def ict():
    from integer_only_nn_02_b200 import ict as _ict

    return _ict


def same(got: CE, ref: CE, what):
    assert got.mant.shape == ref.mant.shape, what
    bad = np.argwhere(got.mant != ref.mant)
    assert bad.size == 0, f"{what}: {len(bad)} mantissas differ, first {bad[:5].tolist()}"
    bad = np.argwhere(got.exp != ref.exp)
    assert bad.size == 0, f"{what}: {len(bad)} exponents differ, first {bad[:5].tolist()}"


def rows_of(t: CE, rows) -> CE:
    """Row subset of a tensor with row-local (g_rows = 1) or tensor-wide row groups."""
    assert t.g_rows == 1 or t.g_rows >= t.rows
    exp = t.exp[rows] if t.g_rows == 1 else t.exp
    return CE(np.ascontiguousarray(t.mant[rows]), np.ascontiguousarray(exp), 1 if t.g_rows == 1 else len(rows),
              t.g_cols)


def cols_of(t: CE, c0, c1) -> CE:
    """Column slice [c0, c1) made of whole column groups."""
    assert c0 % t.g_cols == 0 and (c1 % t.g_cols == 0 or c1 == t.cols)
    return CE(np.ascontiguousarray(t.mant[:, c0:c1]), np.ascontiguousarray(t.exp[:, c0 // t.g_cols:-(-c1 // t.g_cols)]),
              t.g_rows, t.g_cols)


def status_ok(ict):
    code, raw = ict.ict_get_device_status()
    assert code == 0, (code, raw)


def test_single_linear_step_full(ict):
    cfg = wl.single_linear(seed=0)
    X, W, dY, V = cfg["X"], cfg["W"], cfg["dY"], cfg["V"]
    G, mom, lr = cfg["out_group"], cfg["sgd"]["mom"], cfg["sgd"]["lr"]
    dX_, dW_, ddY, dV_ = (ict.DevCE.from_host(t) for t in (X, W, dY, V))
    Y = ict.linear_fwd(dX_, dW_, G)
    dXg = ict.linear_bwd_data(ddY, dW_, G)
    dWg = ict.linear_bwd_weight(ddY, dX_)
    ict.ict_sgd_momentum_step(dW_, dV_, dWg, mom, lr)
    dW_ref = oracle.linear_bwd_weight(dY, X, 1, X.cols)
    W2, V2 = oracle.sgd_step(W, V, dW_ref, mom, lr)
    same(Y.to_host(), oracle.linear_fwd(X, W, 1, G), "Y")
    same(dXg.to_host(), oracle.linear_bwd_data(dY, W, 1, G), "dX")
    same(dWg.to_host(), dW_ref, "dW")
    same(dW_.to_host(), W2, "W'")
    same(dV_.to_host(), V2, "V'")
    status_ok(ict)


def test_vit_ti_mlp_step_full(ict):
    cfg = wl.vit_ti_mlp(seed=0)
    X, W1, W2, dY2, V1, V2 = (cfg[k] for k in ("X", "W1", "W2", "dY2", "V1", "V2"))
    G, mom, lr = cfg["out_group"], cfg["sgd"]["mom"], cfg["sgd"]["lr"]
    D = {k: ict.DevCE.from_host(cfg[k]) for k in ("X", "W1", "W2", "dY2", "V1", "V2")}
    H = ict.linear_fwd(D["X"], D["W1"], G)
    Gl = ict.gelu_fwd(H)
    Y = ict.linear_fwd(Gl, D["W2"], G)
    dG = ict.linear_bwd_data(D["dY2"], D["W2"], G)
    dW2 = ict.linear_bwd_weight(D["dY2"], Gl)
    dH = ict.gelu_bwd(H, dG)
    dX = ict.linear_bwd_data(dH, D["W1"], G)
    dW1 = ict.linear_bwd_weight(dH, D["X"])
    ict.ict_sgd_momentum_step(D["W1"], D["V1"], dW1, mom, lr)
    ict.ict_sgd_momentum_step(D["W2"], D["V2"], dW2, mom, lr)
    status_ok(ict)

    rH = oracle.linear_fwd(X, W1, 1, G)
    rG = oracle.gelu_fwd(rH)
    rY = oracle.linear_fwd(rG, W2, 1, G)
    rdG = oracle.linear_bwd_data(dY2, W2, 1, G)
    rdW2 = oracle.linear_bwd_weight(dY2, rG, 1, W2.cols)
    rdH = oracle.gelu_bwd(rH, rdG, 1, G)
    rdX = oracle.linear_bwd_data(rdH, W1, 1, G)
    rdW1 = oracle.linear_bwd_weight(rdH, X, 1, W1.cols)
    rW1, rV1 = oracle.sgd_step(W1, V1, rdW1, mom, lr)
    rW2, rV2 = oracle.sgd_step(W2, V2, rdW2, mom, lr)
    for name, got, ref in (("H", H, rH), ("GELU", Gl, rG), ("Y", Y, rY), ("dG", dG, rdG), ("dW2", dW2, rdW2),
                           ("dH", dH, rdH), ("dX", dX, rdX), ("dW1", dW1, rdW1), ("W1'", D["W1"], rW1),
                           ("V1'", D["V1"], rV1), ("W2'", D["W2"], rW2), ("V2'", D["V2"], rV2)):
        same(got.to_host(), ref, name)


def test_resnet18_conv_full(ict):
    cfg = wl.resnet18_conv3x3(seed=0)
    X, W, dY, d, G = cfg["X"], cfg["W"], cfg["dY"], cfg["conv"], cfg["out_group"]
    npix = X.rows
    dX_, dW_, ddY = ict.DevCE.from_host(X), ict.DevCE.from_host(W), ict.DevCE.from_host(dY)
    Y = ict.conv(ict.CONV_FWD, d, dX_, dW_, npix, G)
    dXg = ict.conv(ict.CONV_BWD_DATA, d, ddY, dW_, npix, G)
    dWg = ict.conv(ict.CONV_BWD_WEIGHT, d, ddY, dX_, 1, W.cols)
    status_ok(ict)
    same(Y.to_host(), oracle.conv(oracle.CONV_FWD, d, X, W, npix, G), "conv Y")
    same(dXg.to_host(), oracle.conv(oracle.CONV_BWD_DATA, d, dY, W, npix, G), "conv dX")
    same(dWg.to_host(), oracle.conv(oracle.CONV_BWD_WEIGHT, d, dY, X, 1, W.cols), "conv dW")


def test_vit_b_trio(ict):
    cfg = wl.vit_b_linear_trio(seed=0)
    X, W1, W2, dY1, dY2 = (cfg[k] for k in ("X", "W1", "W2", "dY1", "dY2"))
    G = cfg["out_group"]
    D = {k: ict.DevCE.from_host(cfg[k]) for k in ("X", "W1", "W2", "dY1", "dY2")}
    H1 = ict.linear_fwd(D["X"], D["W1"], G)
    rH1 = oracle.linear_fwd(X, W1, 1, G)
    same(H1.to_host(), rH1, "fc1 fwd (every row)")
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([rng.choice(X.rows, 200, replace=False), np.arange(X.rows - 40, X.rows)]))
    Y2 = ict.linear_fwd(H1, D["W2"], G).to_host()
    same(rows_of(Y2, rows), oracle.linear_fwd(rows_of(rH1, rows), W2, 1, G), "fc2 fwd rows")
    dH = ict.linear_bwd_data(D["dY2"], D["W2"], G).to_host()
    same(rows_of(dH, rows), oracle.linear_bwd_data(rows_of(dY2, rows), W2, 1, G), "fc2 bwd-data rows")
    dXo = ict.linear_bwd_data(D["dY1"], D["W1"], G).to_host()
    same(rows_of(dXo, rows), oracle.linear_bwd_data(rows_of(dY1, rows), W1, 1, G), "fc1 bwd-data rows")
    # both weight gradients in full: contractions over all 12608 tokens, split-K on the GPU
    dW1 = ict.linear_bwd_weight(D["dY1"], D["X"]).to_host()
    same(dW1, oracle.linear_bwd_weight(dY1, X, 1, X.cols), "fc1 bwd-weight (3072 x 768)")
    dW2 = ict.linear_bwd_weight(D["dY2"], H1).to_host()
    same(dW2, oracle.linear_bwd_weight(dY2, rH1, 1, rH1.cols), "fc2 bwd-weight (768 x 3072)")
    status_ok(ict)


def test_resnet50_sgd_full(ict):
    c5 = wl.resnet50_sgd_arena(seed=0)
    W, V, G = c5["W"], c5["V"], c5["G"]
    mom, lr = c5["sgd"]["mom"], c5["sgd"]["lr"]
    Wd, Vd, Gd = (ict.DevCE.from_host(t) for t in (W, V, G))
    ict.ict_sgd_momentum_step(Wd, Vd, Gd, mom, lr)
    rW, rV = oracle.sgd_step(W, V, G, mom, lr)
    same(Vd.to_host(), rV, "V'")
    same(Wd.to_host(), rW, "W'")
    status_ok(ict)


def test_resnet18_block_tail_full(ict):
    """The block tail bench.py times (residual add fused with ReLU, ReLU backward from the
    fused output, gradient merge on 128 x 56 x 56 x 64 with all-pixel channel groups of
    32), every output, against the oracle's unfused composition."""
    cfg = wl.resnet18_block_tail(seed=0)
    d = ict.DevCE.from_host
    Y, X, dA, dXc = (cfg[k] for k in ("Y", "X", "dA", "dXc"))
    g = (Y.rows, cfg["group"])
    A = ict.DevCE.empty(Y.rows, Y.cols, *g)
    Yd, Xd = d(Y), d(X)
    ict.ict_sum_act(Yd, Xd, A, ict.ACT_RELU, ict._ws(ict.ict_sum_workspace(Yd, Xd, A)))
    Sr = oracle.sum_(Y, X, *g)
    same(A.to_host(), oracle.relu_fwd(Sr), "residual add + relu")
    dS = ict.relu_bwd(A, d(dA))
    dSr = oracle.relu_bwd(Sr, dA)
    same(dS.to_host(), dSr, "relu backward")
    same(ict.sum_(d(dXc), dS).to_host(), oracle.sum_(dXc, dSr, *g), "gradient merge")
    code, raw = ict.ict_get_device_status()
    assert code == 0, (code, raw)
