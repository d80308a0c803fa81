"""CPU oracle for the microscaling quantized-linear hot path.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
(``microscaling_bit_quantization_b200``) never imports it, and this package
imports nothing from the library: the two are independent implementations
compared element by element.

The arithmetic lives in ``mxq_oracle.c`` (plain scalar C11, IEEE binary32,
no FMA contraction); this module marshals numpy arrays, and computes the
GEMM reference in binary64 with numpy's matmul over exactly dequantized
operands (the only library primitive used as a step).

Formats and their scale layouts (canonical, row-major) are documented in
``mxq_oracle.c``.  Every function cites the page passage it follows there.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mxq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# Format ids (same values as the library's public enum).
MXFP8, MXFP4, NVFP4, INT4_G32, INT4_G64, INT8_ROW, FP8_TENSOR = range(7)
FORMATS = {
    "MXFP8": MXFP8, "MXFP4": MXFP4, "NVFP4": NVFP4, "INT4_G32": INT4_G32,
    "INT4_G64": INT4_G64, "INT8_ROW": INT8_ROW, "FP8_TENSOR": FP8_TENSOR,
}
BLOCK = {MXFP8: 32, MXFP4: 32, NVFP4: 16, INT4_G32: 32, INT4_G64: 64, INT8_ROW: 0, FP8_TENSOR: 0}
IS_4BIT = {MXFP8: False, MXFP4: True, NVFP4: True, INT4_G32: True, INT4_G64: True,
           INT8_ROW: False, FP8_TENSOR: False}


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (C11, no fast-math, no FMA contraction)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-fopenmp", "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i64, i32, u8, u32 = ctypes.c_int64, ctypes.c_int, ctypes.c_uint8, ctypes.c_uint32
        L.orc_e2m1_value.restype = ctypes.c_double
        L.orc_e2m1_value.argtypes = [u8]
        L.orc_e4m3_value.restype = ctypes.c_double
        L.orc_e4m3_value.argtypes = [u8]
        L.orc_e8m0_value.restype = ctypes.c_double
        L.orc_e8m0_value.argtypes = [u8]
        L.orc_to_e4m3.restype = u8
        L.orc_to_e4m3.argtypes = [ctypes.c_float]
        L.orc_to_e2m1.restype = u8
        L.orc_to_e2m1.argtypes = [ctypes.c_float]
        L.orc_round_bf16.restype = ctypes.c_float
        L.orc_round_bf16.argtypes = [ctypes.c_float]
        L.orc_cast_range.restype = None
        L.orc_cast_range.argtypes = [u32, i64, i32, P]
        L.orc_hadamard_norm.restype = ctypes.c_float
        L.orc_hadamard_norm.argtypes = [i32]
        L.orc_hadamard.restype = i32
        L.orc_hadamard.argtypes = [P, P, i64, i64, i32]
        L.orc_quantize.restype = i32
        L.orc_quantize.argtypes = [P, i64, i64, i32, i32, P, P, P, P]
        L.orc_dequantize.restype = i32
        L.orc_dequantize.argtypes = [P, P, P, i64, i64, i32, P]
        L.orc_select.restype = i32
        L.orc_select.argtypes = [P, i64, i64, P, i32, P, P, P, P, P]
        L.orc_quantize_mse_nvfp4.restype = i32
        L.orc_quantize_mse_nvfp4.argtypes = [P, i64, i64, i32, P, P, P, P]
        L.orc_mse_nvfp4_blocks.restype = i32
        L.orc_mse_nvfp4_blocks.argtypes = [P, i64, i64, ctypes.c_float, P, P, P]
        L.orc_quantize_mx_grid.restype = i32
        L.orc_quantize_mx_grid.argtypes = [P, i64, i64, i32, i32, ctypes.c_float, P, P, P]
        L.orc_mx_grid_sse.restype = i32
        L.orc_mx_grid_sse.argtypes = [P, i64, i64, i32, i32, P, i32, P, P, P, P]
        L.orc_calibrate_activation.restype = i32
        L.orc_calibrate_activation.argtypes = [P, i64, i64, P, i32, P, P, P, P, P, P, P]
        L.orc_w4a16_weights.restype = i32
        L.orc_w4a16_weights.argtypes = [P, P, i64, i64, i32, P]
        L.orc_lowrank_down.restype = i32
        L.orc_lowrank_down.argtypes = [P, P, i64, i64, i32, P]
        L.orc_route.restype = i32
        L.orc_route.argtypes = [P, i32, i32, i32, i32, i32]
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


class OracleError(ValueError):
    pass


# ---------------------------------------------------------------- codecs

def e2m1_value(code: int) -> float:
    return lib().orc_e2m1_value(code)


def e4m3_value(code: int) -> float:
    return lib().orc_e4m3_value(code)


def e8m0_value(b: int) -> float:
    return lib().orc_e8m0_value(b)


def to_e4m3(v: float) -> int:
    return lib().orc_to_e4m3(v)


def to_e2m1(v: float) -> int:
    return lib().orc_to_e2m1(v)


def round_bf16(v: float) -> float:
    return lib().orc_round_bf16(v)


def round_bf16_array(x) -> np.ndarray:
    """bf16 rounding (RNE) of an fp32 array, through the oracle's scalar routine."""
    x = _f32(x)
    f = lib().orc_round_bf16
    return np.array([f(float(v)) for v in x.ravel()], dtype=np.float32).reshape(x.shape)


def cast_range(first_bits: int, count: int, elem: str) -> np.ndarray:
    """Convert `count` consecutive binary32 bit patterns; elem 'e4m3' or 'e2m1'."""
    out = np.empty(count, dtype=np.uint8)
    lib().orc_cast_range(first_bits, count, 0 if elem == "e4m3" else 1, _ptr(out))
    return out


# ---------------------------------------------------------------- transforms

def hadamard_norm(b: int) -> float:
    return lib().orc_hadamard_norm(b)


def hadamard(x, b: int) -> np.ndarray:
    x = _f32(x)
    rows, cols = x.shape
    y = np.empty_like(x)
    if lib().orc_hadamard(_ptr(x), _ptr(y), rows, cols, b) != 0:
        raise OracleError("bad hadamard arguments")
    return y


# ---------------------------------------------------------------- quantizers

class QTensor:
    """Oracle quantized tensor: codes (packed as in the library's canonical
    layout), scales (canonical row-major), tensor scale, and the format."""

    def __init__(self, fmt, rows, cols, codes, scales, tensor_scale):
        self.fmt, self.rows, self.cols = fmt, rows, cols
        self.codes, self.scales, self.tensor_scale = codes, scales, tensor_scale

    def dequantize(self) -> np.ndarray:
        out = np.empty((self.rows, self.cols), dtype=np.float64)
        ts = np.array([self.tensor_scale], dtype=np.float32)
        sc = self.scales if self.scales is not None else np.zeros(1, np.uint8)
        st = lib().orc_dequantize(_ptr(self.codes), _ptr(sc), _ptr(ts), self.rows, self.cols,
                                  self.fmt, _ptr(out))
        if st != 0:
            raise OracleError("bad dequantize arguments")
        return out


def scales_shape_dtype(fmt: int, rows: int, cols: int):
    if fmt in (MXFP8, MXFP4):
        return (rows, cols // 32), np.uint8
    if fmt == NVFP4:
        return (rows, cols // 16), np.uint8
    if fmt in (INT4_G32, INT4_G64):
        return (rows, cols // BLOCK[fmt]), np.float32
    if fmt == INT8_ROW:
        return (rows,), np.float32
    return None, None


def codes_shape(fmt: int, rows: int, cols: int):
    return (rows, cols // 2) if IS_4BIT[fmt] else (rows, cols)


def quantize(x, fmt: int, hadamard_b: int = 0) -> QTensor:
    x = _f32(x)
    rows, cols = x.shape
    codes = np.zeros(codes_shape(fmt, rows, cols), dtype=np.uint8)
    sshape, sdt = scales_shape_dtype(fmt, rows, cols)
    scales = np.zeros(sshape, dtype=sdt) if sshape is not None else None
    ts = np.zeros(1, dtype=np.float32)
    work = np.empty_like(x) if hadamard_b else np.empty(1, np.float32)
    st = lib().orc_quantize(_ptr(x), rows, cols, fmt, hadamard_b, _ptr(work), _ptr(codes),
                            _ptr(scales) if scales is not None else None, _ptr(ts))
    if st != 0:
        raise OracleError("bad quantize arguments")
    return QTensor(fmt, rows, cols, codes, scales, float(ts[0]))


def dequantize_f32(q: QTensor) -> np.ndarray:
    """Dequantized values rounded once to fp32 (each exact product is
    representable in fp32 except for the final rounding of NVFP4's tensor
    scale product and the INT scales, so this is RN_f32 of the exact value)."""
    return q.dequantize().astype(np.float32)


# ---------------------------------------------------------------- selection

def select_weight_format(w, candidates):
    w = _f32(w)
    n, k = w.shape
    cands = np.ascontiguousarray(np.asarray(candidates, dtype=np.int32))
    codes = np.empty(n * k, np.uint8)
    scales = np.empty(n * k * 4, np.uint8)
    deq = np.empty(n * k, np.float64)
    choice = np.empty(n, np.uint8)
    sse = np.empty((n, len(cands)), np.float64)
    st = lib().orc_select(_ptr(w), n, k, _ptr(cands), len(cands), _ptr(codes), _ptr(scales),
                          _ptr(deq), _ptr(choice), _ptr(sse))
    if st != 0:
        raise OracleError("bad select arguments")
    return choice, sse


# ---------------------------------------------------------------- MSE-fitted NVFP4 scales

def quantize_mse_nvfp4(x, iters: int):
    """NVFP4 with block and tensor scales fitted to the squared error
    (mxq_oracle.c, orc_quantize_mse_nvfp4).  Returns (QTensor, total error)."""
    x = _f32(x)
    rows, cols = x.shape
    codes = np.zeros(codes_shape(NVFP4, rows, cols), dtype=np.uint8)
    scales = np.zeros((rows, cols // 16), dtype=np.uint8)
    ts = np.zeros(1, dtype=np.float32)
    sse = np.zeros(1, dtype=np.float64)
    st = lib().orc_quantize_mse_nvfp4(_ptr(x), rows, cols, iters, _ptr(codes), _ptr(scales), _ptr(ts), _ptr(sse))
    if st != 0:
        raise OracleError("bad quantize_mse_nvfp4 arguments")
    return QTensor(NVFP4, rows, cols, codes, scales, float(ts[0])), float(sse[0])


def mse_nvfp4_blocks(x, s_t: float):
    """Block step of quantize_mse_nvfp4 under a given tensor scale: (QTensor,
    per-row errors)."""
    x = _f32(x)
    rows, cols = x.shape
    codes = np.zeros(codes_shape(NVFP4, rows, cols), dtype=np.uint8)
    scales = np.zeros((rows, cols // 16), dtype=np.uint8)
    row_err = np.zeros(rows, dtype=np.float64)
    st = lib().orc_mse_nvfp4_blocks(_ptr(x), rows, cols, float(s_t), _ptr(codes), _ptr(scales), _ptr(row_err))
    if st != 0:
        raise OracleError("bad mse_nvfp4_blocks arguments")
    return QTensor(NVFP4, rows, cols, codes, scales, float(s_t)), row_err


# ---------------------------------------------------------------- MX fixed grid scale

def quantize_mx_grid(x, fmt: int, g: float, hadamard_b: int = 0) -> QTensor:
    """MXFP4 / MXFP8 with the exponent taken from RN32(g amax) (mxq_oracle.c,
    orc_quantize_mx_grid)."""
    x = _f32(x)
    rows, cols = x.shape
    codes = np.zeros(codes_shape(fmt, rows, cols), dtype=np.uint8)
    scales = np.zeros((rows, cols // 32), dtype=np.uint8)
    work = np.empty_like(x) if hadamard_b else np.empty(1, np.float32)
    st = lib().orc_quantize_mx_grid(_ptr(x), rows, cols, fmt, hadamard_b, float(g), _ptr(work), _ptr(codes),
                                    _ptr(scales))
    if st != 0:
        raise OracleError("bad quantize_mx_grid arguments")
    return QTensor(fmt, rows, cols, codes, scales, 0.0)


def mx_grid_sse(x, fmt: int, grid_scales, hadamard_b: int = 0) -> np.ndarray:
    """Squared error of the (rotated) tensor for each candidate grid scale."""
    x = _f32(x)
    rows, cols = x.shape
    gs = np.ascontiguousarray(np.asarray(grid_scales, dtype=np.float32))
    codes = np.zeros(codes_shape(fmt, rows, cols), dtype=np.uint8)
    scales = np.zeros((rows, cols // 32), dtype=np.uint8)
    work = np.empty_like(x) if hadamard_b else np.empty(1, np.float32)
    sse = np.zeros(len(gs), dtype=np.float64)
    st = lib().orc_mx_grid_sse(_ptr(x), rows, cols, fmt, hadamard_b, _ptr(gs), len(gs), _ptr(work), _ptr(codes),
                               _ptr(scales), _ptr(sse))
    if st != 0:
        raise OracleError("bad mx_grid_sse arguments")
    return sse


# ---------------------------------------------------------------- activation-format calibration

def calibrate_activation(x, candidates, sse_accum: np.ndarray, moments_accum: np.ndarray):
    """Adds x's per-candidate squared error and (sum x^2, sum x^4) to the
    accumulators (mxq_oracle.c, orc_calibrate_activation)."""
    x = _f32(x)
    n, k = x.shape
    cands = np.ascontiguousarray(np.asarray(candidates, dtype=np.int32))
    codes = np.empty(max(n * k, 1), np.uint8)
    scales = np.empty(max(n * k * 4, 1), np.uint8)
    deq = np.empty(max(n * k, 1), np.float64)
    choice = np.empty(max(n, 1), np.uint8)
    sse_rows = np.empty(max(n * len(cands), 1), np.float64)
    assert sse_accum.dtype == np.float64 and moments_accum.dtype == np.float64
    st = lib().orc_calibrate_activation(_ptr(x), n, k, _ptr(cands), len(cands), _ptr(codes), _ptr(scales),
                                        _ptr(deq), _ptr(choice), _ptr(sse_rows), _ptr(sse_accum),
                                        _ptr(moments_accum))
    if st != 0:
        raise OracleError("bad calibrate_activation arguments")


def calibrate_pick(sse_accum, candidates, forced_fmt: int = -1) -> int:
    """Table entry: forced_fmt if >= 0, else the candidate with the least
    accumulated error (ties to the lower candidate index)."""
    if forced_fmt >= 0:
        return forced_fmt
    return int(candidates[int(np.argmin(np.asarray(sse_accum)))])


# ---------------------------------------------------------------- low rank + GEMM

def lowrank_down(x, l1) -> np.ndarray:
    """T = bf16(X) . L1 in binary64 (L1 given as fp32 copies of bf16)."""
    x, l1 = _f32(x), _f32(l1)
    m, k = x.shape
    r = l1.shape[1]
    t = np.empty((m, r), np.float64)
    lib().orc_lowrank_down(_ptr(x), _ptr(l1), m, k, r, _ptr(t))
    return t


def lowrank_down_rows(x, l1, rows) -> np.ndarray:
    x = _f32(x)
    return lowrank_down(x[np.asarray(rows)], l1)


def qlinear(xq: QTensor, wq: QTensor, t=None, l2=None, rows=None) -> np.ndarray:
    """Y = deq(Xq) . deq(Wq)^T (+ T . L2), all in binary64 over exactly
    dequantized operands.  `rows` restricts the result to those rows of X
    (T, if given, must already hold just those rows)."""
    xd = xq.dequantize()
    if rows is not None:
        xd = xd[np.asarray(rows)]
    y = xd @ wq.dequantize().T
    if t is not None:
        y = y + np.asarray(t, np.float64) @ np.asarray(l2, np.float64)
    return y


def w4a16_weights(wq: QTensor) -> np.ndarray:
    """bf16(RN32(q s)) of every weight of an INT4-g32/g64 tensor (mxq_oracle.c,
    orc_w4a16_weights), as fp32 values."""
    g = BLOCK[wq.fmt]
    w = np.empty((wq.rows, wq.cols), np.float32)
    st = lib().orc_w4a16_weights(_ptr(wq.codes), _ptr(np.ascontiguousarray(wq.scales, np.float32)), wq.rows, wq.cols,
                                 g, _ptr(w))
    if st != 0:
        raise OracleError("bad w4a16 arguments")
    return w


def w4a16(x, wq: QTensor, rows=None) -> np.ndarray:
    """Y = bf16(X) . W16^T in binary64, W16 = w4a16_weights(wq)."""
    xb = round_bf16_array(x).astype(np.float64)
    if rows is not None:
        xb = xb[np.asarray(rows)]
    return xb @ w4a16_weights(wq).astype(np.float64).T


# ---------------------------------------------------------------- per-channel mixed weight formats

def qlinear_mixed(x, w, choice, rows=None) -> np.ndarray:
    """Linear layer whose weight keeps a format per output channel (Chameleon
    article, section "the format is chosen by the value distribution": each
    output channel of a weight takes the format with the least reconstruction
    error; its W8A8 / W4A8 settings quantize activations to 8 bits, here
    MXFP8).  Y[m, n] = sum_k deq(MXFP8(X))[m, k] * deq_f(W)[n, k] with
    f = choice[n], in binary64 over exactly dequantized operands.  Each
    weight format quantizes the whole W, so a tensor-scaled format (NVFP4)
    takes the tensor scale of the whole weight, as the selection measures it.
    `rows` restricts the result to those rows of X."""
    x, w = _f32(x), _f32(w)
    choice = np.asarray(choice, dtype=np.uint8)
    if choice.shape != (w.shape[0],):
        raise OracleError("one format per output channel")
    wd = np.zeros(w.shape, np.float64)
    for f in np.unique(choice):
        sel = choice == f
        wd[sel] = quantize(w, int(f)).dequantize()[sel]
    xd = quantize(x, MXFP8).dequantize()
    if rows is not None:
        xd = xd[np.asarray(rows)]
    return xd @ wd.T


# ---------------------------------------------------------------- routing

def route(table, n_layers: int, n_intervals: int, layer: int, step: int, n_steps: int) -> int:
    table = np.ascontiguousarray(np.asarray(table, dtype=np.uint8))
    return lib().orc_route(_ptr(table), n_layers, n_intervals, layer, step, n_steps)
