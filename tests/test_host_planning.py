"""Host-side argument checking and planning of libict, without a GPU: the *_workspace
queries run the same validation and tiling plans as the entry points (dry, nothing is
dereferenced or launched) and return 0 for arguments the entry point would refuse."""
import ctypes

import pytest

from integer_only_nn_02_b200 import ict

A16 = 0x100000  # a 16-byte aligned fake address: the planner only inspects pointer values


def T(rows, cols, g_rows, g_cols, ld=None, addr=A16):
    return ict.ict_tensor(addr, addr, rows, cols, ld if ld is not None else cols, g_rows, g_cols)


def lin_ws(op, a, b, out):
    return ict.lib.ict_linear_workspace(op, ctypes.byref(a), ctypes.byref(b), ctypes.byref(out))


def test_linear_workspace_accepts_and_sizes():
    # forward with both operands uniform along K: fused epilogue, no scratch
    assert lin_ws(0, T(64, 128, 64, 128), T(64, 128, 1, 128), T(64, 64, 1, 32)) == 0
    # forward with (1, 32) groups along K: the aligned copy of X (rows x K) and its exponents
    need = lin_ws(0, T(100, 128, 1, 32), T(64, 128, 1, 128), T(100, 64, 1, 32))
    assert need >= 100 * 128 + 100
    # backward weight: both operands aligned per column and transposed, plus split-K slices
    need = lin_ws(2, T(12608, 192, 1, 32), T(12608, 768, 1, 32), T(192, 768, 1, 768))
    assert need >= 192 * 12608 + 768 * 12608


@pytest.mark.parametrize("args", [
    (0, T(64, 128, 1, 128), T(64, 96, 1, 96), T(64, 64, 1, 32)),        # K mismatch
    (0, T(64, 128, 1, 128), T(64, 128, 1, 128), T(64, 48, 1, 32)),      # output width mismatch
    (0, T(64, 128, 1, 128), T(64, 128, 1, 128), T(64, 64, 2, 32)),      # output groups not row-local
    (0, T(64, 120, 1, 120), T(64, 120, 1, 120), T(64, 64, 1, 32)),      # K not a multiple of 16
    (0, T(64, 128, 1, 128, ld=136), T(64, 128, 1, 128), T(64, 64, 1, 32)),  # ld not 16-aligned
    (0, T(64, 128, 1, 128, addr=A16 + 8), T(64, 128, 1, 128), T(64, 64, 1, 32)),  # misaligned base
    (0, T(64, 128, 1, 24), T(64, 128, 1, 128), T(64, 64, 1, 32)),       # groups of 24 along K
    (1, T(64, 64, 1, 64), T(48, 128, 1, 128), T(64, 128, 1, 32)),       # bwd-data: N mismatch
    (2, T(64, 64, 1, 64), T(65, 128, 1, 128), T(64, 128, 1, 128)),      # bwd-weight: M mismatch
    (5, T(64, 128, 1, 128), T(64, 128, 1, 128), T(64, 64, 1, 32)),      # unknown op
])
def test_linear_workspace_refuses(args):
    op, a, b, out = args
    assert lin_ws(op, a, b, out) == 0


def test_split_batch_workspace():
    f = ict.lib.ict_linear_bwd_weight_partial_workspace
    assert f(ctypes.byref(T(1000, 192, 1, 32)), ctypes.byref(T(1000, 768, 1, 32))) > 0
    assert f(ctypes.byref(T(1000, 192, 1, 32)), ctypes.byref(T(999, 768, 1, 32))) == 0  # batch mismatch
    assert f(ctypes.byref(T(0, 192, 1, 32)), ctypes.byref(T(0, 768, 1, 32))) > 0       # an empty shard


def test_sum_and_pool_workspaces():
    s = ict.lib.ict_sum_workspace
    row = T(300, 192, 1, 32)
    assert s(ctypes.byref(row), ctypes.byref(row), ctypes.byref(row)) == 0  # row-local: no scratch
    glob = T(2000, 64, 2000, 32)
    assert s(ctypes.byref(glob), ctypes.byref(glob), ctypes.byref(glob)) == 256  # 2 group columns, rounded up
    p = ict.lib.ict_avgpool_workspace
    X, Y = T(2 * 14 * 14, 64, 2 * 14 * 14, 32), T(2 * 7 * 7, 64, 1, 32)
    assert p(0, ctypes.byref(X), 2, 14, 14, 2, ctypes.byref(Y)) >= 98 * 2 * 4
    assert p(0, ctypes.byref(X), 2, 14, 14, 3, ctypes.byref(Y)) == 0  # 14 is not a multiple of 3


def test_conv_workspace():
    d = ict.conv_desc(dict(n=4, h=56, w=56, c=64, k=64, r=3, s=3, stride=1, pad=1))
    for direction in (0, 1, 2):
        assert ict.lib.ict_conv_workspace(direction, ctypes.byref(d)) > 0


def test_library_lookup_tables_equal_the_oracles():
    """The library builds its lookup tables (Tables 7 and 8) on the host, independently
    of the oracle (long double libm against 90-digit decimals); every entry agrees."""
    import numpy as np

    from oracle import luts

    mine, ref = ict.ict_lut_tables(), luts.tables()
    for name in ("exp", "log", "gelu_fwd", "gelu_bwd"):
        assert mine[name].shape == ref[name].shape and np.array_equal(mine[name], ref[name]), name
