"""The seeded synthetic inputs are what the design documents: shapes, group geometries,
exponent ranges and value distributions of the configurations, reproducible by seed."""
import numpy as np

from integer_only_nn_02_b200 import workloads as wl


def _check(t, rows, cols, g_rows, g_cols, elo, ehi):
    assert t.mant.shape == (rows, cols) and t.mant.dtype == np.int8
    assert (t.g_rows, t.g_cols) == (g_rows, g_cols)
    assert t.exp.shape == (-(-rows // g_rows), -(-cols // g_cols))
    assert np.abs(t.mant.astype(int)).max() <= 127
    assert t.exp.min() >= elo and t.exp.max() <= ehi


def test_vit_ti_mlp_small():
    cfg = wl.vit_ti_mlp(seed=3, tokens=500)
    _check(cfg["X"], 500, 192, 1, 192, -8, -6)
    _check(cfg["W1"], 768, 192, 1, 192, -10, -6)
    _check(cfg["W2"], 192, 768, 1, 768, -10, -6)
    _check(cfg["dY2"], 500, 192, 1, 192, -14, -12)
    assert (cfg["V1"].exp == wl.E_ZERO).all() and (cfg["V1"].mant == 0).all()
    again = wl.vit_ti_mlp(seed=3, tokens=500)
    assert all(np.array_equal(cfg[k].mant, again[k].mant) and np.array_equal(cfg[k].exp, again[k].exp)
               for k in ("X", "W1", "W2", "dY2"))
    assert not np.array_equal(cfg["X"].mant, wl.vit_ti_mlp(seed=4, tokens=500)["X"].mant)


def test_resnet18_shapes_and_relu_like_input():
    cfg = wl.resnet18_conv3x3(seed=1, n=2)
    npix = 2 * 56 * 56
    _check(cfg["X"], npix, 64, npix, 32, -8, -6)
    _check(cfg["W"], 64, 576, 1, 576, -10, -6)
    _check(cfg["dY"], npix, 64, npix, 32, -14, -12)
    zeros = (cfg["X"].mant == 0).mean()
    assert 0.45 < zeros < 0.55 and cfg["X"].mant.min() >= 0  # post-ReLU: half zeros, rest in [1, 127]
    tail = wl.resnet18_block_tail(seed=1, n=2)
    for k in ("Y", "X", "dA", "dXc"):
        assert tail[k].mant.shape == (npix, 64) and tail[k].g_rows == npix and tail[k].g_cols == 32


def test_vit_b_trio_small():
    cfg = wl.vit_b_linear_trio(seed=2, tokens=300)
    _check(cfg["X"], 300, 768, 1, 64, -9, -7)
    _check(cfg["W1"], 3072, 768, 1, 64, -10, -8)
    _check(cfg["dY1"], 300, 3072, 1, 64, -14, -12)


def test_resnet50_arena():
    shapes = wl.resnet50_param_shapes()
    assert len(shapes) == 161
    assert sum(int(np.prod(s)) for s in shapes) == 25_557_032
