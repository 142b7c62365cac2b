"""Thin Python binding of libict.so (argument marshalling only).

Every entry point of ``include/ict.h`` is exposed under the same name and takes the
same arguments, with :class:`DevCE` (a (C,e) tensor on the GPU: torch int8 mantissas
plus an int8 exponent grid) in place of ``ict_tensor``.  PyTorch supplies device memory
and streams; all arithmetic runs in the library's kernels.  Importing this module
loads ``libict.so`` and raises if it has not been built; there is no other code path.

Convenience wrappers (``linear_fwd`` ...) allocate outputs and workspace with torch
and then make exactly one library call.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from .workloads import CE, cdiv

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libict.so")

ICT_OK = 0
NOALLOC_SCRATCH_BYTES = 16 << 20  # ICT_NOALLOC_SCRATCH_BYTES in include/ict.h
STATUS_NAMES = {
    0: "ICT_OK", 1: "ICT_ERR_INVALID_ARG", 2: "ICT_ERR_LAYOUT", 3: "ICT_ERR_ALIGNMENT",
    4: "ICT_ERR_WORKSPACE", 5: "ICT_ERR_UNSUPPORTED_ARCH", 6: "ICT_ERR_CUDA",
    7: "ICT_ERR_DEVICE_TIMEOUT", 8: "ICT_ERR_EXP_RANGE",
}
OP_LINEAR_FWD, OP_LINEAR_BWD_DATA, OP_LINEAR_BWD_WEIGHT = 0, 1, 2
CONV_FWD, CONV_BWD_DATA, CONV_BWD_WEIGHT = 0, 1, 2

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libict.so not found at {LIB_PATH}: build it with "
        "`python -m integer_only_nn_02_b200.csrc.build` (nvcc, sm_100a)")
lib = ctypes.CDLL(LIB_PATH)


class ict_tensor(ctypes.Structure):
    _fields_ = [("mant", ctypes.c_void_p), ("exp", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("ld", ctypes.c_int64), ("g_rows", ctypes.c_int32),
                ("g_cols", ctypes.c_int32)]


class ict_sgd_params(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("mom_mul", "mom_shift", "lr_mul", "lr_shift")]


class ict_conv_desc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("n", "h", "w", "c", "k", "r", "s", "stride", "pad")]


_P = ctypes.POINTER
_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_SIGS = {
    "ict_status_string": ([_i32], ctypes.c_char_p),
    "ict_version": ([], ctypes.c_char_p),
    "ict_get_device_status": ([_P(_i32), _vp], _i32),
    "ict_set_wait_limit_ns": ([ctypes.c_uint64], _i32),
    "ict_selftest_wait_timeout": ([ctypes.c_uint64, _vp], _i32),
    "ict_launch_count": ([], ctypes.c_uint64),
    "ict_timing_enable": ([_i32], _i32),
    "ict_timing_read": ([_i32, _P(ctypes.c_double), _P(_i64), _P(ctypes.c_double), _i32], _i32),
    "ict_requant": ([_vp, _i32, _i64, _i64, _i64, _i32, _vp, _vp, _P(ict_tensor), _vp], _i32),
    "ict_align": ([_P(ict_tensor), _i32, _i32, _vp, _i64, _vp, _vp], _i32),
    "ict_linear_workspace": ([_i32, _P(ict_tensor), _P(ict_tensor), _P(ict_tensor)], _sz),
    "ict_linear_fwd": ([_P(ict_tensor)] * 3 + [_vp, _sz, _vp], _i32),
    "ict_linear_fwd_noalloc": ([_P(ict_tensor)] * 3 + [_vp], _i32),
    "ict_linear_bwd_data": ([_P(ict_tensor)] * 3 + [_vp, _sz, _vp], _i32),
    "ict_linear_bwd_weight": ([_P(ict_tensor)] * 3 + [_vp, _sz, _vp], _i32),
    "ict_linear_bwd_weight_partial_workspace": ([_P(ict_tensor)] * 2, _sz),
    "ict_linear_bwd_weight_targets": ([_P(ict_tensor)] * 2 + [_vp, _vp, _vp, _sz, _vp], _i32),
    "ict_linear_bwd_weight_partial": ([_P(ict_tensor)] * 2 + [_vp, _vp, _vp, _i32, _i64, _vp, _sz, _vp], _i32),
    "ict_conv_workspace": ([_i32, _P(ict_conv_desc)], _sz),
    "ict_conv_implicit_gemm": ([_i32, _P(ict_conv_desc)] + [_P(ict_tensor)] * 3 + [_vp, _sz, _vp], _i32),
    "ict_conv_split_begin": ([_i32, _P(ict_conv_desc)] + [_P(ict_tensor)] * 3 + [_vp, _vp, _sz, _vp], _i32),
    "ict_conv_split_end": ([_i32, _P(ict_conv_desc)] + [_P(ict_tensor)] * 3 + [_vp, _vp, _sz, _vp], _i32),
    "ict_conv_bwd_weight_partial": ([_P(ict_conv_desc)] + [_P(ict_tensor)] * 2 + [_vp, _i64, _vp, _vp, _vp, _sz,
                                                                                   _vp], _i32),
    "ict_sgd_momentum_step": ([_P(ict_tensor), _P(ict_tensor), _P(ict_tensor), _P(ict_sgd_params), _vp], _i32),
    "ict_sgd_momentum_step_multi": ([_i32, _P(_P(ict_tensor)), _P(_P(ict_tensor)), _P(_P(ict_tensor)),
                                     _P(ict_sgd_params), _vp], _i32),
    "ict_gelu_fwd": ([_P(ict_tensor), _P(ict_tensor), _vp], _i32),
    "ict_gelu_bwd": ([_P(ict_tensor)] * 3 + [_vp], _i32),
    "ict_relu_fwd": ([_P(ict_tensor), _i32, _P(ict_tensor), _vp], _i32),
    "ict_relu_bwd": ([_P(ict_tensor), _P(ict_tensor), _i32, _P(ict_tensor), _vp], _i32),
    "ict_sum_workspace": ([_P(ict_tensor)] * 3, _sz),
    "ict_sum": ([_P(ict_tensor)] * 3 + [_vp, _sz, _vp], _i32),
    "ict_avgpool_workspace": ([_i32, _P(ict_tensor), _i32, _i32, _i32, _i32, _P(ict_tensor)], _sz),
    "ict_avgpool_fwd": ([_P(ict_tensor), _i32, _i32, _i32, _i32, _P(ict_tensor), _vp, _sz, _vp], _i32),
    "ict_avgpool_bwd": ([_P(ict_tensor), _i32, _i32, _i32, _i32, _P(ict_tensor), _vp, _sz, _vp], _i32),
    "ict_sum_act": ([_P(ict_tensor)] * 3 + [_i32, _vp, _sz, _vp], _i32),
    "ict_conv_fwd_act": ([_P(ict_conv_desc)] + [_P(ict_tensor)] * 3 + [_i32, _vp, _sz, _vp], _i32),
    "ict_depthwise_workspace": ([_i32, _P(ict_conv_desc), _P(ict_tensor)], _sz),
    "ict_depthwise": ([_i32, _P(ict_conv_desc)] + [_P(ict_tensor)] * 3 + [_vp, _sz, _vp], _i32),
    "ict_patchify": ([_P(ict_tensor), _i32, _i32, _i32, _i32, _P(ict_tensor), _vp], _i32),
    "ict_sum_scaled": ([_P(ict_tensor), _i32, _i32, _P(ict_tensor), _i32, _i32, _P(ict_tensor), _vp, _sz, _vp], _i32),
    "ict_lut_tables": ([_vp, _vp, _vp, _vp], _i32),
    "ict_set_mantissa_bits": ([_i32], _i32),
    "ict_get_mantissa_bits": ([], _i32),
    "ict_gelu_lut_fwd": ([_P(ict_tensor), _P(ict_tensor), _vp], _i32),
    "ict_gelu_lut_bwd": ([_P(ict_tensor)] * 3 + [_vp], _i32),
    "ict_softmax_ce": ([_P(ict_tensor), _vp, _vp, _P(ict_tensor), _vp], _i32),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = _res

EXPORTED = tuple(_SIGS)


class IctError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)}")
        self.code = code


def _check(code: int, what: str) -> None:
    if code != ICT_OK:
        raise IctError(code, what)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor | None):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


class DevCE:
    """A (C,e) tensor on the GPU: int8 mantissas [rows, ld] (first ``cols`` used) and an
    int8 exponent grid [cdiv(rows, g_rows), cdiv(cols, g_cols)]."""

    def __init__(self, mant: torch.Tensor, exp: torch.Tensor, g_rows: int, g_cols: int, cols=None):
        assert mant.dtype == torch.int8 and exp.dtype == torch.int8 and mant.is_cuda
        self.mant, self.exp = mant, exp
        self.rows = int(mant.shape[0])
        self.cols = int(cols if cols is not None else mant.shape[1])
        self.ld = int(mant.stride(0)) if mant.dim() == 2 and self.rows > 1 else int(mant.shape[1])
        self.g_rows, self.g_cols = int(g_rows), int(g_cols)

    @staticmethod
    def empty(rows, cols, g_rows, g_cols, device="cuda"):
        g_rows = max(1, min(g_rows, rows)) if rows else max(1, g_rows)
        g_cols = max(1, min(g_cols, cols)) if cols else max(1, g_cols)
        ld = -(-cols // 16) * 16 if cols else 16
        mant = torch.empty((rows, ld), dtype=torch.int8, device=device)
        exp = torch.empty((cdiv(rows, g_rows), cdiv(cols, g_cols)), dtype=torch.int8, device=device)
        return DevCE(mant, exp, g_rows, g_cols, cols=cols)

    @staticmethod
    def from_host(t: CE, device="cuda", pin=False):
        rows, cols = t.rows, t.cols
        ld = -(-cols // 16) * 16 if cols else 16
        m = np.zeros((rows, ld), np.int8)
        m[:, :cols] = t.mant
        mt = torch.from_numpy(m)
        et = torch.from_numpy(np.ascontiguousarray(t.exp))
        if pin:
            mt, et = mt.pin_memory(), et.pin_memory()
        return DevCE(mt.to(device, non_blocking=pin), et.to(device, non_blocking=pin),
                     t.g_rows, t.g_cols, cols=cols)

    def to_host(self) -> CE:
        m = self.mant[:, : self.cols].cpu().numpy().copy()
        return CE(np.ascontiguousarray(m), self.exp.cpu().numpy().copy(), self.g_rows, self.g_cols)

    def c(self) -> ict_tensor:
        return ict_tensor(self.mant.data_ptr(), self.exp.data_ptr(), self.rows, self.cols, self.ld,
                          self.g_rows, self.g_cols)


def _ws(nbytes: int, device="cuda") -> torch.Tensor | None:
    if nbytes == 0:
        return None
    return torch.empty(int(nbytes), dtype=torch.uint8, device=device)  # 256-aligned by torch


# ----------------------------------------------------------------- raw entry points

def ict_status_string(code: int) -> str:
    return lib.ict_status_string(code).decode()


def ict_version() -> str:
    return lib.ict_version().decode()


def ict_get_device_status(stream=None):
    v = ctypes.c_int32(0)
    code = lib.ict_get_device_status(ctypes.byref(v), _stream(stream))
    return code, v.value


def ict_launch_count() -> int:
    return int(lib.ict_launch_count())


KERNEL_CLASSES = {"gemm": 0, "sgd": 1, "align": 2, "requant": 3, "gelu": 4, "estar": 5, "other": 6, "pointwise": 7}


def ict_timing_enable(on: bool) -> None:
    _check(lib.ict_timing_enable(int(bool(on))), "ict_timing_enable")


def ict_timing_read(kernel_class: int, reset: bool = False):
    """(device ms, launches, algorithmic work) accumulated for one kernel class."""
    ms, n, w = ctypes.c_double(0), ctypes.c_int64(0), ctypes.c_double(0)
    _check(lib.ict_timing_read(int(kernel_class), ctypes.byref(ms), ctypes.byref(n), ctypes.byref(w),
                               int(bool(reset))), "ict_timing_read")
    return ms.value, n.value, w.value


def ict_set_wait_limit_ns(ns: int) -> None:
    _check(lib.ict_set_wait_limit_ns(int(ns)), "ict_set_wait_limit_ns")


def ict_selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    _check(lib.ict_selftest_wait_timeout(int(limit_ns), _stream(stream)), "ict_selftest_wait_timeout")


def ict_requant(vals: torch.Tensor, out: DevCE, base_exp=0, row_exp=None, col_exp=None, stream=None):
    bits = {torch.int32: 32, torch.int64: 64}[vals.dtype]
    rows, cols = vals.shape
    o = out.c()
    _check(lib.ict_requant(_ptr(vals), bits, rows, cols, vals.stride(0), base_exp, _ptr(row_exp),
                           _ptr(col_exp), ctypes.byref(o), _stream(stream)), "ict_requant")


def ict_align(t: DevCE, axis: int, transpose: bool, out: torch.Tensor, e_star: torch.Tensor, stream=None):
    c = t.c()
    _check(lib.ict_align(ctypes.byref(c), axis, int(transpose), _ptr(out), out.stride(0), _ptr(e_star),
                         _stream(stream)), "ict_align")


def ict_linear_workspace(op: int, a: DevCE, b: DevCE, out: DevCE) -> int:
    ca, cb, co = a.c(), b.c(), out.c()
    return int(lib.ict_linear_workspace(op, ctypes.byref(ca), ctypes.byref(cb), ctypes.byref(co)))


def _linear(fn, name, a, b, out, ws, stream):
    ca, cb, co = a.c(), b.c(), out.c()
    nbytes = 0 if ws is None else ws.numel()
    _check(fn(ctypes.byref(ca), ctypes.byref(cb), ctypes.byref(co), _ptr(ws), nbytes, _stream(stream)), name)


def ict_linear_fwd(X: DevCE, W: DevCE, Y: DevCE, ws=None, stream=None):
    _linear(lib.ict_linear_fwd, "ict_linear_fwd", X, W, Y, ws, stream)


def ict_linear_fwd_noalloc(X: DevCE, W: DevCE, Y: DevCE, stream=None):
    """Forward Product with the library's fixed internal scratch instead of a workspace."""
    cx, cw, cy = X.c(), W.c(), Y.c()
    _check(lib.ict_linear_fwd_noalloc(ctypes.byref(cx), ctypes.byref(cw), ctypes.byref(cy), _stream(stream)),
           "ict_linear_fwd_noalloc")


def ict_linear_bwd_data(dY: DevCE, W: DevCE, dX: DevCE, ws=None, stream=None):
    _linear(lib.ict_linear_bwd_data, "ict_linear_bwd_data", dY, W, dX, ws, stream)


def ict_linear_bwd_weight(dY: DevCE, X: DevCE, dW: DevCE, ws=None, stream=None):
    _linear(lib.ict_linear_bwd_weight, "ict_linear_bwd_weight", dY, X, dW, ws, stream)


def ict_linear_bwd_weight_partial_workspace(dY: DevCE, X: DevCE) -> int:
    cy, cx = dY.c(), X.c()
    return int(lib.ict_linear_bwd_weight_partial_workspace(ctypes.byref(cy), ctypes.byref(cx)))


def ict_linear_bwd_weight_targets(dY: DevCE, X: DevCE, e_dy: torch.Tensor, e_x: torch.Tensor, ws, stream=None):
    cy, cx = dY.c(), X.c()
    _check(lib.ict_linear_bwd_weight_targets(ctypes.byref(cy), ctypes.byref(cx), _ptr(e_dy), _ptr(e_x), _ptr(ws),
                                             ws.numel(), _stream(stream)), "ict_linear_bwd_weight_targets")


def ict_linear_bwd_weight_partial(dY: DevCE, X: DevCE, e_dy: torch.Tensor, e_x: torch.Tensor, acc: torch.Tensor,
                                  ws, stream=None):
    bits = {torch.int32: 32, torch.int64: 64}[acc.dtype]
    cy, cx = dY.c(), X.c()
    _check(lib.ict_linear_bwd_weight_partial(ctypes.byref(cy), ctypes.byref(cx), _ptr(e_dy), _ptr(e_x), _ptr(acc),
                                             bits, acc.stride(0), _ptr(ws), ws.numel(), _stream(stream)),
           "ict_linear_bwd_weight_partial")


def conv_desc(d: dict) -> ict_conv_desc:
    return ict_conv_desc(*[int(d[k]) for k in ("n", "h", "w", "c", "k", "r", "s", "stride", "pad")])


def ict_conv_workspace(direction: int, d: dict) -> int:
    cd = conv_desc(d)
    return int(lib.ict_conv_workspace(direction, ctypes.byref(cd)))


def ict_conv_implicit_gemm(direction: int, d: dict, a: DevCE, b: DevCE, out: DevCE, ws=None, stream=None):
    cd, ca, cb, co = conv_desc(d), a.c(), b.c(), out.c()
    nbytes = 0 if ws is None else ws.numel()
    _check(lib.ict_conv_implicit_gemm(direction, ctypes.byref(cd), ctypes.byref(ca), ctypes.byref(cb),
                                      ctypes.byref(co), _ptr(ws), nbytes, _stream(stream)),
           "ict_conv_implicit_gemm")


def _conv_split(fn, name, direction, d, a, b, out, need, ws, stream):
    cd, ca, cb, co = conv_desc(d), a.c(), b.c(), out.c()
    _check(fn(direction, ctypes.byref(cd), ctypes.byref(ca), ctypes.byref(cb), ctypes.byref(co), _ptr(need), _ptr(ws),
              ws.numel(), _stream(stream)), name)


def ict_conv_split_begin(direction: int, d: dict, a: DevCE, b: DevCE, out: DevCE, need: torch.Tensor, ws,
                         stream=None):
    _conv_split(lib.ict_conv_split_begin, "ict_conv_split_begin", direction, d, a, b, out, need, ws, stream)


def ict_conv_split_end(direction: int, d: dict, a: DevCE, b: DevCE, out: DevCE, need: torch.Tensor, ws,
                       stream=None):
    _conv_split(lib.ict_conv_split_end, "ict_conv_split_end", direction, d, a, b, out, need, ws, stream)


def ict_conv_bwd_weight_partial(d: dict, dY: DevCE, X: DevCE, acc: torch.Tensor, e_k: torch.Tensor,
                                e_rsc: torch.Tensor, ws, stream=None):
    cd, cy, cx = conv_desc(d), dY.c(), X.c()
    _check(lib.ict_conv_bwd_weight_partial(ctypes.byref(cd), ctypes.byref(cy), ctypes.byref(cx), _ptr(acc),
                                           acc.stride(0), _ptr(e_k), _ptr(e_rsc), _ptr(ws), ws.numel(),
                                           _stream(stream)), "ict_conv_bwd_weight_partial")


def sgd_params(mom=(230, 8), lr=(1, 4)) -> ict_sgd_params:
    return ict_sgd_params(int(mom[0]), int(mom[1]), int(lr[0]), int(lr[1]))


def ict_sgd_momentum_step(W: DevCE, V: DevCE, G: DevCE, mom=(230, 8), lr=(1, 4), stream=None):
    cw, cv, cg, p = W.c(), V.c(), G.c(), sgd_params(mom, lr)
    _check(lib.ict_sgd_momentum_step(ctypes.byref(cw), ctypes.byref(cv), ctypes.byref(cg), ctypes.byref(p),
                                      _stream(stream)), "ict_sgd_momentum_step")


def ict_sgd_momentum_step_multi(Ws, Vs, Gs, mom=(230, 8), lr=(1, 4), stream=None):
    n = len(Ws)
    cw = [w.c() for w in Ws]
    cv = [v.c() for v in Vs]
    cg = [g.c() for g in Gs]
    arr = _P(ict_tensor) * n
    pw = arr(*[ctypes.pointer(x) for x in cw])
    pv = arr(*[ctypes.pointer(x) for x in cv])
    pg = arr(*[ctypes.pointer(x) for x in cg])
    p = sgd_params(mom, lr)
    _check(lib.ict_sgd_momentum_step_multi(n, pw, pv, pg, ctypes.byref(p), _stream(stream)),
           "ict_sgd_momentum_step_multi")


def ict_gelu_fwd(H: DevCE, out: DevCE, stream=None):
    ch, co = H.c(), out.c()
    _check(lib.ict_gelu_fwd(ctypes.byref(ch), ctypes.byref(co), _stream(stream)), "ict_gelu_fwd")


def ict_gelu_bwd(H: DevCE, dG: DevCE, dH: DevCE, stream=None):
    ch, cd, co = H.c(), dG.c(), dH.c()
    _check(lib.ict_gelu_bwd(ctypes.byref(ch), ctypes.byref(cd), ctypes.byref(co), _stream(stream)),
           "ict_gelu_bwd")


def ict_set_mantissa_bits(bits: int):
    _check(lib.ict_set_mantissa_bits(int(bits)), "ict_set_mantissa_bits")


def ict_get_mantissa_bits() -> int:
    return int(lib.ict_get_mantissa_bits())


def ict_lut_tables():
    """The library's own lookup tables (host memory): LUT_exp [30][256] uint8, LUT_log
    [256] uint8, GELU forward and backward [30][256] int8."""
    ex, lg = np.zeros((30, 256), np.uint8), np.zeros(256, np.uint8)
    gf, gb = np.zeros((30, 256), np.int8), np.zeros((30, 256), np.int8)
    _check(lib.ict_lut_tables(ex.ctypes.data, lg.ctypes.data, gf.ctypes.data, gb.ctypes.data), "ict_lut_tables")
    return {"exp": ex, "log": lg, "gelu_fwd": gf, "gelu_bwd": gb}


def ict_gelu_lut_fwd(H: DevCE, out: DevCE, stream=None):
    ch, co = H.c(), out.c()
    _check(lib.ict_gelu_lut_fwd(ctypes.byref(ch), ctypes.byref(co), _stream(stream)), "ict_gelu_lut_fwd")


def ict_gelu_lut_bwd(H: DevCE, dY: DevCE, dH: DevCE, stream=None):
    ch, cd, co = H.c(), dY.c(), dH.c()
    _check(lib.ict_gelu_lut_bwd(ctypes.byref(ch), ctypes.byref(cd), ctypes.byref(co), _stream(stream)),
           "ict_gelu_lut_bwd")


def ict_softmax_ce(Z: DevCE, target: torch.Tensor, loss: torch.Tensor, dZ: DevCE, stream=None):
    assert target.dtype == torch.int32 and loss.dtype == torch.int32 and target.is_cuda and loss.is_cuda
    cz, cd = Z.c(), dZ.c()
    _check(lib.ict_softmax_ce(ctypes.byref(cz), _ptr(target), _ptr(loss), ctypes.byref(cd), _stream(stream)),
           "ict_softmax_ce")


# ----------------------------------------------------------------- conveniences

def ict_relu_fwd(X: DevCE, six: bool, Z: DevCE, stream=None):
    cx, cz = X.c(), Z.c()
    _check(lib.ict_relu_fwd(ctypes.byref(cx), int(six), ctypes.byref(cz), _stream(stream)), "ict_relu_fwd")


def ict_relu_bwd(X: DevCE, dY: DevCE, six: bool, dX: DevCE, stream=None):
    cx, cy, cd = X.c(), dY.c(), dX.c()
    _check(lib.ict_relu_bwd(ctypes.byref(cx), ctypes.byref(cy), int(six), ctypes.byref(cd), _stream(stream)),
           "ict_relu_bwd")


def ict_sum_workspace(X: DevCE, Y: DevCE, Z: DevCE) -> int:
    cx, cy, cz = X.c(), Y.c(), Z.c()
    return int(lib.ict_sum_workspace(ctypes.byref(cx), ctypes.byref(cy), ctypes.byref(cz)))


def ict_sum(X: DevCE, Y: DevCE, Z: DevCE, ws=None, stream=None):
    cx, cy, cz = X.c(), Y.c(), Z.c()
    nbytes = 0 if ws is None else ws.numel()
    _check(lib.ict_sum(ctypes.byref(cx), ctypes.byref(cy), ctypes.byref(cz), _ptr(ws), nbytes, _stream(stream)),
           "ict_sum")


def ict_sum_scaled(X: DevCE, xw, Y: DevCE, yw, Z: DevCE, ws=None, stream=None):
    """Z = FIT(xw[0] 2^-xw[1] X + yw[0] 2^-yw[1] Y)."""
    cx, cy, cz = X.c(), Y.c(), Z.c()
    nbytes = 0 if ws is None else ws.numel()
    _check(lib.ict_sum_scaled(ctypes.byref(cx), int(xw[0]), int(xw[1]), ctypes.byref(cy), int(yw[0]), int(yw[1]),
                              ctypes.byref(cz), _ptr(ws), nbytes, _stream(stream)), "ict_sum_scaled")


ACT_NONE, ACT_RELU, ACT_RELU6 = 0, 1, 2


def ict_sum_act(X: DevCE, Y: DevCE, Z: DevCE, act: int, ws=None, stream=None):
    cx, cy, cz = X.c(), Y.c(), Z.c()
    nbytes = 0 if ws is None else ws.numel()
    _check(lib.ict_sum_act(ctypes.byref(cx), ctypes.byref(cy), ctypes.byref(cz), int(act), _ptr(ws), nbytes,
                           _stream(stream)), "ict_sum_act")


def ict_conv_fwd_act(d: dict, X: DevCE, W: DevCE, Y: DevCE, act: int, ws=None, stream=None):
    cd, cx, cw, cy = conv_desc(d), X.c(), W.c(), Y.c()
    nbytes = 0 if ws is None else ws.numel()
    _check(lib.ict_conv_fwd_act(ctypes.byref(cd), ctypes.byref(cx), ctypes.byref(cw), ctypes.byref(cy), int(act),
                                _ptr(ws), nbytes, _stream(stream)), "ict_conv_fwd_act")


def ict_sgd_momentum_step_wd(W: DevCE, V: DevCE, G: DevCE, Gd: DevCE, wd=(105, 20), mom=(230, 8), lr=(1, 4),
                             stream=None):
    """SGD with momentum and weight decay: Gd = FIT(G + wd W) (the weighted Sum, into G's
    groups; wd = 105 2^-20 is 1e-4), then the momentum step on Gd."""
    ict_sum_scaled(G, (1, 0), W, wd, Gd, _ws(ict_sum_workspace(G, W, Gd)), stream)
    ict_sgd_momentum_step(W, V, Gd, mom, lr, stream)


def linear_fwd(X: DevCE, W: DevCE, g_cols=32, stream=None) -> DevCE:
    Y = DevCE.empty(X.rows, W.rows, 1, g_cols)
    ict_linear_fwd(X, W, Y, _ws(ict_linear_workspace(OP_LINEAR_FWD, X, W, Y)), stream)
    return Y


def linear_bwd_data(dY: DevCE, W: DevCE, g_cols=32, stream=None) -> DevCE:
    dX = DevCE.empty(dY.rows, W.cols, 1, g_cols)
    ict_linear_bwd_data(dY, W, dX, _ws(ict_linear_workspace(OP_LINEAR_BWD_DATA, dY, W, dX)), stream)
    return dX


def linear_bwd_weight(dY: DevCE, X: DevCE, g_cols=None, stream=None) -> DevCE:
    dW = DevCE.empty(dY.cols, X.cols, 1, g_cols or X.cols)
    ict_linear_bwd_weight(dY, X, dW, _ws(ict_linear_workspace(OP_LINEAR_BWD_WEIGHT, dY, X, dW)), stream)
    return dW


def conv(direction: int, d: dict, a: DevCE, b: DevCE, g_rows: int, g_cols: int, stream=None) -> DevCE:
    P = (d["h"] + 2 * d["pad"] - d["r"]) // d["stride"] + 1
    Q = (d["w"] + 2 * d["pad"] - d["s"]) // d["stride"] + 1
    if direction == CONV_FWD:
        rows, cols = d["n"] * P * Q, d["k"]
    elif direction == CONV_BWD_DATA:
        rows, cols = d["n"] * d["h"] * d["w"], d["c"]
    else:
        rows, cols = d["k"], d["r"] * d["s"] * d["c"]
    out = DevCE.empty(rows, cols, g_rows, g_cols)
    ict_conv_implicit_gemm(direction, d, a, b, out, _ws(ict_conv_workspace(direction, d)), stream)
    return out


def gelu_fwd(H: DevCE, stream=None) -> DevCE:
    out = DevCE.empty(H.rows, H.cols, H.g_rows, H.g_cols)
    ict_gelu_fwd(H, out, stream)
    return out


def gelu_bwd(H: DevCE, dG: DevCE, stream=None) -> DevCE:
    dH = DevCE.empty(H.rows, H.cols, 1, H.g_cols)
    ict_gelu_bwd(H, dG, dH, stream)
    return dH


def gelu_lut_fwd(H: DevCE, stream=None) -> DevCE:
    out = DevCE.empty(H.rows, H.cols, H.g_rows, H.g_cols)
    ict_gelu_lut_fwd(H, out, stream)
    return out


def gelu_lut_bwd(H: DevCE, dY: DevCE, stream=None) -> DevCE:
    dH = DevCE.empty(H.rows, H.cols, 1, H.g_cols)
    ict_gelu_lut_bwd(H, dY, dH, stream)
    return dH


def softmax_ce(Z: DevCE, target: torch.Tensor, g_cols: int | None = None, stream=None):
    """(loss per row, int32 at scale 2^-5; gradient of the summed loss in (1, g_cols) groups)."""
    loss = torch.empty(Z.rows, dtype=torch.int32, device="cuda")
    dZ = DevCE.empty(Z.rows, Z.cols, 1, g_cols or Z.cols)
    ict_softmax_ce(Z, target.to(device="cuda", dtype=torch.int32), loss, dZ, stream)
    return loss, dZ


def device_status(stream=None) -> int:
    code, _ = ict_get_device_status(stream)
    return code


class StepGraph:
    """A fixed sequence of library calls (for instance one training step) captured into
    one CUDA graph and replayed with a single launch.

    ``fn`` issues the calls on torch's current stream.  It runs ``warmup`` times eagerly
    on a side stream first (one-time host setup such as kernel attributes happens
    there), then once under capture.  Every tensor and workspace ``fn`` touches must
    stay alive, at the same address, for the life of the graph; each replay reruns all
    calls, including in-place updates (an SGD step advances the weights every replay).
    """

    def __init__(self, fn, warmup: int = 1):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(warmup):
                fn()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        n0 = ict_launch_count()
        with torch.cuda.graph(self.graph, capture_error_mode="relaxed"):
            fn()
        self.launches = ict_launch_count() - n0  # kernels in one replay

    def replay(self) -> None:
        self.graph.replay()


def relu_fwd(X: DevCE, six=False, stream=None) -> DevCE:
    Z = DevCE.empty(X.rows, X.cols, X.g_rows, X.g_cols)
    ict_relu_fwd(X, six, Z, stream)
    return Z


def relu_bwd(X: DevCE, dY: DevCE, six=False, stream=None) -> DevCE:
    dX = DevCE.empty(dY.rows, dY.cols, dY.g_rows, dY.g_cols)
    ict_relu_bwd(X, dY, six, dX, stream)
    return dX


def sum_(X: DevCE, Y: DevCE, stream=None) -> DevCE:
    """FIT(X + Y) into X's (and Y's) group partition."""
    Z = DevCE.empty(X.rows, X.cols, X.g_rows, X.g_cols)
    ict_sum(X, Y, Z, _ws(ict_sum_workspace(X, Y, Z)), stream)
    return Z


def ict_avgpool_workspace(direction: int, src: DevCE, n, h, w, K, out: DevCE) -> int:
    ci, co = src.c(), out.c()
    return int(lib.ict_avgpool_workspace(direction, ctypes.byref(ci), n, h, w, K, ctypes.byref(co)))


def ict_avgpool_fwd(X: DevCE, n, h, w, K, Y: DevCE, ws, stream=None):
    cx, cy = X.c(), Y.c()
    _check(lib.ict_avgpool_fwd(ctypes.byref(cx), n, h, w, K, ctypes.byref(cy), _ptr(ws), 0 if ws is None else ws.numel(),
                               _stream(stream)), "ict_avgpool_fwd")


def ict_avgpool_bwd(dY: DevCE, n, h, w, K, dX: DevCE, ws, stream=None):
    cy, cx = dY.c(), dX.c()
    _check(lib.ict_avgpool_bwd(ctypes.byref(cy), n, h, w, K, ctypes.byref(cx), _ptr(ws), 0 if ws is None else ws.numel(),
                               _stream(stream)), "ict_avgpool_bwd")


def _avgpool(direction, src: DevCE, n, h, w, K, out: DevCE, stream):
    ws = _ws(ict_avgpool_workspace(direction, src, n, h, w, K, out))
    (ict_avgpool_fwd if direction == 0 else ict_avgpool_bwd)(src, n, h, w, K, out, ws, stream)


def avgpool_fwd(X: DevCE, n, h, w, K, g_rows, g_cols, stream=None) -> DevCE:
    """K x K average pool, stride K, of NHWC X [n*h*w][c]: FIT(window sum / K^2)."""
    Y = DevCE.empty(n * (h // K) * (w // K), X.cols, g_rows, g_cols)
    _avgpool(0, X, n, h, w, K, Y, stream)
    return Y


def avgpool_bwd(dY: DevCE, n, h, w, K, g_rows, g_cols, stream=None) -> DevCE:
    """Backward of the K x K average pool: FIT(window gradient / K^2) at every pixel."""
    dX = DevCE.empty(n * h * w, dY.cols, g_rows, g_cols)
    _avgpool(1, dY, n, h, w, K, dX, stream)
    return dX


def ict_patchify(X: DevCE, n, h, w, P, out: DevCE, stream=None):
    cx, co = X.c(), out.c()
    _check(lib.ict_patchify(ctypes.byref(cx), n, h, w, P, ctypes.byref(co), _stream(stream)), "ict_patchify")


def patchify(X: DevCE, n, h, w, P, stream=None) -> DevCE:
    """Non-overlapping P x P patches as the aligned rows of one (C,e) tensor."""
    rows, K = n * (h // P) * (w // P), P * P * X.cols
    out = DevCE.empty(rows, K, rows, K)
    ict_patchify(X, n, h, w, P, out, stream)
    return out


def ict_depthwise_workspace(direction: int, d: dict, out: DevCE) -> int:
    cd, co = conv_desc(d), out.c()
    return int(lib.ict_depthwise_workspace(direction, ctypes.byref(cd), ctypes.byref(co)))


def ict_depthwise(direction: int, d: dict, a: DevCE, b: DevCE, out: DevCE, ws=None, stream=None):
    cd, ca, cb, co = conv_desc(d), a.c(), b.c(), out.c()
    nbytes = 0 if ws is None else ws.numel()
    _check(lib.ict_depthwise(direction, ctypes.byref(cd), ctypes.byref(ca), ctypes.byref(cb), ctypes.byref(co),
                             _ptr(ws), nbytes, _stream(stream)), "ict_depthwise")


def depthwise(direction: int, d: dict, a: DevCE, b: DevCE, g_rows: int, g_cols: int, stream=None) -> DevCE:
    P = (d["h"] + 2 * d["pad"] - d["r"]) // d["stride"] + 1
    Q = (d["w"] + 2 * d["pad"] - d["s"]) // d["stride"] + 1
    if direction == CONV_FWD:
        rows, cols = d["n"] * P * Q, d["c"]
    elif direction == CONV_BWD_DATA:
        rows, cols = d["n"] * d["h"] * d["w"], d["c"]
    else:
        rows, cols = d["c"], d["r"] * d["s"]
    out = DevCE.empty(rows, cols, g_rows, g_cols)
    ict_depthwise(direction, d, a, b, out, _ws(max(256, ict_depthwise_workspace(direction, d, out))), stream)
    return out
