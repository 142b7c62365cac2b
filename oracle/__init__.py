"""Python access to the CPU oracle ``libict_oracle.so`` (test infrastructure only).

The oracle is the plain int64 C implementation in ``ict_oracle.c``.  Only the tests,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` import this
module; the CUDA library never does.  Inputs and outputs are
``integer_only_nn_02_b200.workloads.CE`` containers (numpy arrays).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from integer_only_nn_02_b200.workloads import CE, empty_ce

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ict_oracle.c")
LIB = os.path.join(HERE, "libict_oracle.so")

ORC_OK, ORC_ERR_ARG, ORC_ERR_LAYOUT, ORC_ERR_EXP_RANGE = 0, 1, 2, 8


class OracleError(RuntimeError):
    def __init__(self, code, what):
        super().__init__(f"oracle {what} failed with status {code}")
        self.code = code


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP over independent output rows)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.run(
            ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=gnu11", "-o", tmp, SRC],
            check=True,
        )
        os.replace(tmp, LIB)
    return LIB


class _OT(ctypes.Structure):
    _fields_ = [
        ("mant", ctypes.c_void_p),
        ("exp", ctypes.c_void_p),
        ("rows", ctypes.c_int64),
        ("cols", ctypes.c_int64),
        ("ld", ctypes.c_int64),
        ("g_rows", ctypes.c_int32),
        ("g_cols", ctypes.c_int32),
    ]


class _Conv(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("n", "h", "w", "c", "k", "r", "s", "stride", "pad")]


class _Sgd(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("mom_mul", "mom_shift", "lr_mul", "lr_shift")]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.POINTER
        L = _lib
        L.oracle_requant.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64,
                                     ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, P(_OT)]
        L.oracle_requant_bits.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64,
                                          ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, P(_OT)]
        L.oracle_align_to.argtypes = [P(_OT), ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_int64, ctypes.c_int]
        L.oracle_align.argtypes = [P(_OT), ctypes.c_int, ctypes.c_void_p, ctypes.c_int64,
                                   ctypes.c_int, ctypes.c_void_p]
        for name in ("oracle_linear_fwd", "oracle_linear_bwd_data", "oracle_linear_bwd_weight",
                     "oracle_gelu_bwd"):
            getattr(L, name).argtypes = [P(_OT), P(_OT), P(_OT)]
        for name in ("oracle_linear_fwd_acc", "oracle_linear_bwd_data_acc",
                     "oracle_linear_bwd_weight_acc"):
            getattr(L, name).argtypes = [P(_OT), P(_OT), ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_gelu_fwd.argtypes = [P(_OT), P(_OT)]
        L.oracle_sum.argtypes = [P(_OT), P(_OT), P(_OT)]
        L.oracle_sum_scaled.argtypes = [P(_OT), ctypes.c_int32, ctypes.c_int32, P(_OT), ctypes.c_int32,
                                        ctypes.c_int32, P(_OT)]
        L.oracle_relu_fwd.argtypes = [P(_OT), ctypes.c_int, P(_OT)]
        L.oracle_avgpool_fwd.argtypes = [P(_OT)] + [ctypes.c_int] * 4 + [P(_OT)]
        L.oracle_depthwise.argtypes = [ctypes.c_int, P(_Conv), P(_OT), P(_OT), P(_OT)]
        L.oracle_depthwise_acc.argtypes = [ctypes.c_int, P(_Conv), P(_OT), P(_OT), ctypes.c_void_p,
                                           ctypes.c_void_p]
        L.oracle_avgpool_bwd.argtypes = [P(_OT)] + [ctypes.c_int] * 4 + [P(_OT)]
        L.oracle_relu_bwd.argtypes = [P(_OT), P(_OT), ctypes.c_int, P(_OT)]
        L.oracle_conv.argtypes = [ctypes.c_int, P(_Conv), P(_OT), P(_OT), P(_OT)]
        L.oracle_conv_acc.argtypes = [ctypes.c_int, P(_Conv), P(_OT), P(_OT), ctypes.c_void_p,
                                      ctypes.c_void_p]
        L.oracle_sgd_step.argtypes = [P(_OT), P(_OT), P(_OT), P(_Sgd)]
        L.oracle_need64.argtypes = [ctypes.c_int64, ctypes.c_int32]
        L.oracle_rne_shift64.argtypes = [ctypes.c_int64, ctypes.c_int32]
        L.oracle_rne_shift64.restype = ctypes.c_int64
        L.oracle_fit_two_term.argtypes = [ctypes.c_int64] + [ctypes.c_void_p] * 5
        L.oracle_linear_bits.argtypes = [ctypes.c_int, P(_OT), P(_OT), P(_OT), ctypes.c_int32]
        L.oracle_sgd_step_bits.argtypes = [P(_OT), P(_OT), P(_OT), P(_Sgd), ctypes.c_int32]
        L.oracle_softmax_ce.argtypes = [P(_OT), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p, P(_OT)]
        L.oracle_gelu_lut_fwd.argtypes = [P(_OT), ctypes.c_void_p, P(_OT)]
        L.oracle_gelu_lut_bwd.argtypes = [P(_OT), P(_OT), ctypes.c_void_p, P(_OT)]
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _ot(t: CE) -> _OT:
    assert t.mant.dtype == np.int8 and t.exp.dtype == np.int8
    assert t.mant.flags.c_contiguous and t.exp.flags.c_contiguous
    return _OT(_ptr(t.mant), _ptr(t.exp), t.rows, t.cols, t.cols, t.g_rows, t.g_cols)


def _check(code, what):
    if code != ORC_OK:
        raise OracleError(code, what)


def num_threads() -> int:
    return int(lib().oracle_num_threads())


# ------------------------------------------------------------------ primitives


def need(x: int, r: int) -> int:
    """Smallest exponent at which RNE(x * 2^(r-e)) fits in [-127, 127]; -128 for x = 0."""
    return int(lib().oracle_need64(int(x), int(r)))


def rne_shift(x: int, k: int) -> int:
    """RNE(x * 2^k)."""
    return int(lib().oracle_rne_shift64(int(x), int(k)))


def fit_two_term(a, pa, b, pb):
    """FIT of one group of values a*2^pa + b*2^pb; returns (mantissas, exponent)."""
    a = np.ascontiguousarray(a, np.int64)
    b = np.ascontiguousarray(b, np.int64)
    pa = np.ascontiguousarray(pa, np.int32)
    pb = np.ascontiguousarray(pb, np.int32)
    out = np.zeros(a.shape[0], np.int8)
    e = lib().oracle_fit_two_term(a.shape[0], _ptr(a), _ptr(pa), _ptr(b), _ptr(pb), _ptr(out))
    return out, int(e)


def requant(x: np.ndarray, g_rows: int, g_cols: int, base_exp: int = 0,
            row_exp: np.ndarray | None = None, col_exp: np.ndarray | None = None) -> CE:
    x = np.ascontiguousarray(x, np.int64)
    rows, cols = x.shape
    out = empty_ce(rows, cols, g_rows, g_cols)
    re = None if row_exp is None else np.ascontiguousarray(row_exp, np.int8)
    ce = None if col_exp is None else np.ascontiguousarray(col_exp, np.int8)
    code = lib().oracle_requant(rows, cols, _ptr(x), cols, base_exp,
                                None if re is None else _ptr(re),
                                None if ce is None else _ptr(ce), ctypes.byref(_ot(out)))
    _check(code, "requant")
    return out


def requant_bits(x: np.ndarray, bits: int, g_rows: int, g_cols: int, base_exp: int = 0) -> CE:
    """FIT with B-bit mantissas (clip bound 2^(bits-1) - 1)."""
    x = np.ascontiguousarray(x, np.int64)
    rows, cols = x.shape
    out = empty_ce(rows, cols, g_rows, g_cols)
    _check(lib().oracle_requant_bits(rows, cols, _ptr(x), cols, base_exp, None, None, int(bits),
                                     ctypes.byref(_ot(out))), "requant_bits")
    return out


def align(t: CE, axis: int, transpose: bool = False):
    """ALIGN_MAX; returns (aligned mantissas, exponent vector)."""
    shape = (t.cols, t.rows) if transpose else (t.rows, t.cols)
    out = np.zeros(shape, np.int8)
    e = np.zeros(t.rows if axis == 1 else t.cols, np.int8)
    code = lib().oracle_align(ctypes.byref(_ot(t)), axis, _ptr(out), shape[1], int(transpose), _ptr(e))
    _check(code, "align")
    return out, e


def align_to(t: CE, axis: int, e_target: np.ndarray, transpose: bool = False) -> np.ndarray:
    """ALIGN_MAX to given target exponents (one per non-contracted index, each at least
    the group exponents it covers); returns the aligned mantissas."""
    shape = (t.cols, t.rows) if transpose else (t.rows, t.cols)
    out = np.zeros(shape, np.int8)
    e = np.ascontiguousarray(e_target, np.int8)
    assert e.shape == ((t.rows if axis == 1 else t.cols),)
    code = lib().oracle_align_to(ctypes.byref(_ot(t)), axis, _ptr(e), _ptr(out), shape[1], int(transpose))
    _check(code, "align_to")
    return out


def _product(name, a, b, rows, cols, g_rows, g_cols):
    out = empty_ce(rows, cols, g_rows, g_cols)
    _check(getattr(lib(), name)(ctypes.byref(_ot(a)), ctypes.byref(_ot(b)), ctypes.byref(_ot(out))), name)
    return out


def linear_fwd(X: CE, W: CE, g_rows=1, g_cols=32) -> CE:
    """Y = X * W^T, requantised into (g_rows, g_cols) groups."""
    return _product("oracle_linear_fwd", X, W, X.rows, W.rows, g_rows, g_cols)


def linear_bwd_data(dY: CE, W: CE, g_rows=1, g_cols=32) -> CE:
    """dX = dY * W."""
    return _product("oracle_linear_bwd_data", dY, W, dY.rows, W.cols, g_rows, g_cols)


def linear_bwd_weight(dY: CE, X: CE, g_rows=1, g_cols=None) -> CE:
    """dW = dY^T * X (default groups: one per row)."""
    cols = X.cols
    return _product("oracle_linear_bwd_weight", dY, X, dY.cols, cols, g_rows, g_cols or cols)


def _acc(name, a, b, rows, cols):
    acc = np.zeros((rows, cols), np.int64)
    r = np.zeros((rows, cols), np.int32)
    _check(getattr(lib(), name)(ctypes.byref(_ot(a)), ctypes.byref(_ot(b)), _ptr(acc), _ptr(r)), name)
    return acc, r


def linear_fwd_acc(X, W):
    return _acc("oracle_linear_fwd_acc", X, W, X.rows, W.rows)


def linear_bwd_data_acc(dY, W):
    return _acc("oracle_linear_bwd_data_acc", dY, W, dY.rows, W.cols)


def linear_bwd_weight_acc(dY, X):
    return _acc("oracle_linear_bwd_weight_acc", dY, X, dY.cols, X.cols)


CONV_FWD, CONV_BWD_DATA, CONV_BWD_WEIGHT = 0, 1, 2


def _conv_out_shape(direction, d):
    P = (d["h"] + 2 * d["pad"] - d["r"]) // d["stride"] + 1
    Q = (d["w"] + 2 * d["pad"] - d["s"]) // d["stride"] + 1
    if direction == CONV_FWD:
        return d["n"] * P * Q, d["k"]
    if direction == CONV_BWD_DATA:
        return d["n"] * d["h"] * d["w"], d["c"]
    return d["k"], d["r"] * d["s"] * d["c"]


def conv(direction: int, d: dict, a: CE, b: CE, g_rows: int, g_cols: int) -> CE:
    rows, cols = _conv_out_shape(direction, d)
    out = empty_ce(rows, cols, g_rows, g_cols)
    cd = _Conv(*[int(d[k]) for k in ("n", "h", "w", "c", "k", "r", "s", "stride", "pad")])
    _check(lib().oracle_conv(direction, ctypes.byref(cd), ctypes.byref(_ot(a)), ctypes.byref(_ot(b)),
                             ctypes.byref(_ot(out))), "conv")
    return out


def conv_acc(direction: int, d: dict, a: CE, b: CE):
    rows, cols = _conv_out_shape(direction, d)
    acc = np.zeros((rows, cols), np.int64)
    r = np.zeros((rows, cols), np.int32)
    cd = _Conv(*[int(d[k]) for k in ("n", "h", "w", "c", "k", "r", "s", "stride", "pad")])
    _check(lib().oracle_conv_acc(direction, ctypes.byref(cd), ctypes.byref(_ot(a)), ctypes.byref(_ot(b)),
                                 _ptr(acc), _ptr(r)), "conv_acc")
    return acc, r


def sgd_step(W: CE, V: CE, G: CE, mom=(230, 8), lr=(1, 4)):
    """One integer SGD-momentum step; returns new (W, V) (inputs untouched)."""
    W2, V2 = W.copy(), V.copy()
    p = _Sgd(mom[0], mom[1], lr[0], lr[1])
    _check(lib().oracle_sgd_step(ctypes.byref(_ot(W2)), ctypes.byref(_ot(V2)), ctypes.byref(_ot(G)),
                                 ctypes.byref(p)), "sgd_step")
    return W2, V2


def linear_bits(op: int, a: CE, b: CE, bits: int, g_rows: int = 1, g_cols: int = 32) -> CE:
    """A linear Product with B-bit outputs (op 0 forward, 1 backward-data, 2 backward-weight)."""
    rows = a.cols if op == 2 else a.rows
    cols = b.rows if op == 0 else b.cols
    out = empty_ce(rows, cols, g_rows, g_cols)
    _check(lib().oracle_linear_bits(op, ctypes.byref(_ot(a)), ctypes.byref(_ot(b)), ctypes.byref(_ot(out)),
                                    int(bits)), "linear_bits")
    return out


def sgd_step_bits(W: CE, V: CE, G: CE, bits: int, mom=(230, 8), lr=(1, 4)):
    """The momentum step with B-bit mantissas; returns new copies of (W, V)."""
    W2, V2 = W.copy(), V.copy()
    p = _Sgd(int(mom[0]), int(mom[1]), int(lr[0]), int(lr[1]))
    _check(lib().oracle_sgd_step_bits(ctypes.byref(_ot(W2)), ctypes.byref(_ot(V2)), ctypes.byref(_ot(G)),
                                      ctypes.byref(p), int(bits)), "sgd_step_bits")
    return W2, V2


def gelu_fwd(H: CE) -> CE:
    out = empty_ce(H.rows, H.cols, H.g_rows, H.g_cols)
    _check(lib().oracle_gelu_fwd(ctypes.byref(_ot(H)), ctypes.byref(_ot(out))), "gelu_fwd")
    return out


def gelu_bwd(H: CE, dG: CE, g_rows=1, g_cols=32) -> CE:
    return _product("oracle_gelu_bwd", H, dG, H.rows, H.cols, g_rows, g_cols)


# ------------------------------------------------------------------ lookup-table nonlinearities


def softmax_ce(Z: CE, target: np.ndarray, g_rows: int = 1, g_cols: int = None):
    """Output head through LUT_exp / LUT_log (Table 8): (loss per row as integers at
    scale 2^-5, gradient of the summed loss as a (C,e) tensor in (g_rows, g_cols) groups)."""
    from oracle import luts

    t = luts.tables()
    tgt = np.ascontiguousarray(target, dtype=np.int32)
    loss = np.zeros(Z.rows, np.int32)
    dZ = empty_ce(Z.rows, Z.cols, g_rows, g_cols or Z.cols)
    _check(lib().oracle_softmax_ce(ctypes.byref(_ot(Z)), _ptr(tgt), _ptr(t["exp"]), _ptr(t["log"]), _ptr(loss),
                                   ctypes.byref(_ot(dZ))), "softmax_ce")
    return loss, dZ


def gelu_lut_fwd(H: CE) -> CE:
    """GELU forward through LUT_fwd (Table 7), exponents carried unchanged."""
    from oracle import luts

    out = empty_ce(H.rows, H.cols, H.g_rows, H.g_cols)
    _check(lib().oracle_gelu_lut_fwd(ctypes.byref(_ot(H)), _ptr(luts.tables()["gelu_fwd"]), ctypes.byref(_ot(out))),
           "gelu_lut_fwd")
    return out


def gelu_lut_bwd(H: CE, dY: CE, g_rows=1, g_cols=32) -> CE:
    """GELU backward through LUT_bwd (Table 7): FIT(dY * LUT_bwd[e, C] * 2^-6)."""
    from oracle import luts

    out = empty_ce(H.rows, H.cols, g_rows, g_cols)
    _check(lib().oracle_gelu_lut_bwd(ctypes.byref(_ot(H)), ctypes.byref(_ot(dY)), _ptr(luts.tables()["gelu_bwd"]),
                                     ctypes.byref(_ot(out))), "gelu_lut_bwd")
    return out


def sum_(X: CE, Y: CE, g_rows: int, g_cols: int) -> CE:
    """The Sum primitive: FIT(X + Y) into (g_rows, g_cols) groups."""
    out = empty_ce(X.rows, X.cols, g_rows, g_cols)
    _check(lib().oracle_sum(ctypes.byref(_ot(X)), ctypes.byref(_ot(Y)), ctypes.byref(_ot(out))), "sum")
    return out


def sum_scaled(X: CE, xw, Y: CE, yw, g_rows: int, g_cols: int) -> CE:
    """FIT(xm 2^-xs X + ym 2^-ys Y) for weights xw = (xm, xs), yw = (ym, ys)."""
    out = empty_ce(X.rows, X.cols, g_rows, g_cols)
    _check(lib().oracle_sum_scaled(ctypes.byref(_ot(X)), int(xw[0]), int(xw[1]), ctypes.byref(_ot(Y)), int(yw[0]),
                                   int(yw[1]), ctypes.byref(_ot(out))), "sum_scaled")
    return out


def relu_fwd(X: CE, six: bool = False) -> CE:
    """ReLU (or ReLU6) on the mantissas; the exponents are carried through."""
    out = empty_ce(X.rows, X.cols, X.g_rows, X.g_cols)
    _check(lib().oracle_relu_fwd(ctypes.byref(_ot(X)), int(six), ctypes.byref(_ot(out))), "relu_fwd")
    return out


def relu_bwd(X: CE, dY: CE, six: bool = False) -> CE:
    """dY masked where the forward input passed the ReLU (ReLU6); dY's exponents."""
    out = empty_ce(dY.rows, dY.cols, dY.g_rows, dY.g_cols)
    _check(lib().oracle_relu_bwd(ctypes.byref(_ot(X)), ctypes.byref(_ot(dY)), int(six), ctypes.byref(_ot(out))),
           "relu_bwd")
    return out


def avgpool_fwd(X: CE, n: int, h: int, w: int, K: int, g_rows: int, g_cols: int) -> CE:
    """K x K average pool, stride K, of NHWC X [n*h*w][c]: FIT(window sum / K^2)."""
    out = empty_ce(n * (h // K) * (w // K), X.cols, g_rows, g_cols)
    _check(lib().oracle_avgpool_fwd(ctypes.byref(_ot(X)), n, h, w, K, ctypes.byref(_ot(out))), "avgpool_fwd")
    return out


def avgpool_bwd(dY: CE, n: int, h: int, w: int, K: int, g_rows: int, g_cols: int) -> CE:
    """Backward of the K x K average pool: FIT(dY of the window / K^2) at every pixel."""
    out = empty_ce(n * h * w, dY.cols, g_rows, g_cols)
    _check(lib().oracle_avgpool_bwd(ctypes.byref(_ot(dY)), n, h, w, K, ctypes.byref(_ot(out))), "avgpool_bwd")
    return out


def _dw_shape(direction, d):
    P = (d["h"] + 2 * d["pad"] - d["r"]) // d["stride"] + 1
    Q = (d["w"] + 2 * d["pad"] - d["s"]) // d["stride"] + 1
    if direction == CONV_FWD:
        return d["n"] * P * Q, d["c"]
    if direction == CONV_BWD_DATA:
        return d["n"] * d["h"] * d["w"], d["c"]
    return d["c"], d["r"] * d["s"]


def depthwise(direction: int, d: dict, a: CE, b: CE, g_rows: int, g_cols: int) -> CE:
    """Depthwise convolution (one filter per channel, d["k"] == d["c"]), FIT into groups."""
    rows, cols = _dw_shape(direction, d)
    out = empty_ce(rows, cols, g_rows, g_cols)
    cd = _Conv(*[int(d[k]) for k in ("n", "h", "w", "c", "k", "r", "s", "stride", "pad")])
    _check(lib().oracle_depthwise(direction, ctypes.byref(cd), ctypes.byref(_ot(a)), ctypes.byref(_ot(b)),
                                  ctypes.byref(_ot(out))), "depthwise")
    return out


def depthwise_acc(direction: int, d: dict, a: CE, b: CE):
    rows, cols = _dw_shape(direction, d)
    acc = np.zeros((rows, cols), np.int64)
    r = np.zeros((rows, cols), np.int32)
    cd = _Conv(*[int(d[k]) for k in ("n", "h", "w", "c", "k", "r", "s", "stride", "pad")])
    _check(lib().oracle_depthwise_acc(direction, ctypes.byref(cd), ctypes.byref(_ot(a)), ctypes.byref(_ot(b)),
                                      _ptr(acc), _ptr(r)), "depthwise_acc")
    return acc, r
