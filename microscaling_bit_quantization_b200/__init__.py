"""Python binding of libmxq, the B200 (sm_100a) microscaling quantized-linear
library.  Argument marshalling only: every step runs in the library's CUDA
kernels.  torch provides device memory and the current stream.

The C ABI is declared in ``include/mxq.h``; functions here carry the same
names.  Importing this module loads ``libmxq.so`` from the package directory
and raises ImportError if it has not been built (``python -m
microscaling_bit_quantization_b200.build`` or ``__graft_entry__.build()``).
There is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmxq.so")

MXFP8, MXFP4, NVFP4, INT4_G32, INT4_G64, INT8_ROW, FP8_TENSOR = range(7)
FORMATS = {"MXFP8": MXFP8, "MXFP4": MXFP4, "NVFP4": NVFP4, "INT4_G32": INT4_G32, "INT4_G64": INT4_G64,
           "INT8_ROW": INT8_ROW, "FP8_TENSOR": FP8_TENSOR}
FORMAT_NAMES = {v: k for k, v in FORMATS.items()}
CANONICAL, MMA = 0, 1
F32, BF16 = 0, 1
STATUS = {0: "MXQ_OK", 1: "MXQ_EINVAL", 2: "MXQ_EUNSUPPORTED", 3: "MXQ_ECUDA", 4: "MXQ_ETIMEOUT", 5: "MXQ_ENOSPACE"}

# Every entry point the header declares.
EXPORTS = ("mxq_status_string", "mxq_last_cuda_error_string", "mxq_device_supported", "mxq_check",
           "mxq_selftest_wait_timeout", "mxq_codes_bytes", "mxq_scales_bytes",
           "mxq_quantize_workspace_bytes", "mxq_quantize", "mxq_dequantize", "mxq_hadamard_block", "mxq_cast",
           "mxq_select_workspace_bytes", "mxq_select_weight_format", "mxq_quantize_mse_workspace_bytes",
           "mxq_quantize_mse", "mxq_quantize_mx_grid", "mxq_fit_mx_grid_workspace_bytes", "mxq_fit_mx_grid",
           "mxq_calibrate_workspace_bytes", "mxq_calibrate_activation", "mxq_calibrate_pick",
           "mxq_lowrank_down", "mxq_lowrank_packed_bytes",
           "mxq_lowrank_down_packed", "mxq_lowrank_pack_t", "mxq_lowrank_pack_l2", "mxq_qlinear", "mxq_qlinear_w4a16",
           "mxq_qlinear_w4a16_workspace_bytes", "mxq_route",
           "mxq_quantize_lowrank_workspace_bytes", "mxq_quantize_lowrank", "mxq_quantize_lowrank_noalloc",
           "mxq_qlinear_routed_workspace_bytes", "mxq_qlinear_routed", "mxq_mixed_plan", "mxq_mixed_weight_bytes",
           "mxq_mixed_prepare", "mxq_qlinear_mixed_workspace_bytes", "mxq_qlinear_mixed")


class MxqError(RuntimeError):
    def __init__(self, status: int, what: str):
        detail = _lib.mxq_status_string(status).decode()
        if status == 3:   # MXQ_ECUDA: name the CUDA error
            detail += ": " + _lib.mxq_last_cuda_error_string().decode()
        super().__init__("%s failed: %s (%s)" % (what, STATUS.get(status, status), detail))
        self.status = status


class _QTensorC(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("layout", ctypes.c_int32), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("tensor_scale", ctypes.c_void_p)]


class _LayerC(ctypes.Structure):
    _fields_ = [("w", _QTensorC * 7), ("l1", ctypes.c_void_p), ("l2p", ctypes.c_void_p), ("r", ctypes.c_int32),
                ("hadamard_b", ctypes.c_int32)]


class _MixedC(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("n_group", ctypes.c_int64 * 3),
                ("choice", ctypes.c_void_p), ("group_index", ctypes.c_void_p), ("mx_codes", ctypes.c_void_p),
                ("mx_scales", ctypes.c_void_p), ("i4_codes", ctypes.c_void_p), ("i4_scales", ctypes.c_void_p),
                ("nv_values", ctypes.c_void_p), ("nv_tensor_scale", ctypes.c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libmxq.so is not built at %s; run __graft_entry__.build()" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    psz = ctypes.POINTER(ctypes.c_size_t)
    sig = {
        "mxq_status_string": (ctypes.c_char_p, [i32]),
        "mxq_last_cuda_error_string": (ctypes.c_char_p, []),
        "mxq_device_supported": (ctypes.c_int, [ctypes.c_int]),
        "mxq_check": (i32, [P]),
        "mxq_codes_bytes": (i32, [i32, i64, i64, i32, psz]),
        "mxq_scales_bytes": (i32, [i32, i64, i64, i32, psz]),
        "mxq_quantize_workspace_bytes": (i32, [i32, psz]),
        "mxq_quantize": (i32, [P, i32, i64, i64, i32, i32, i32, P, P, P, P, sz, P]),
        "mxq_selftest_wait_timeout": (i32, [ctypes.c_uint32, P]),
        "mxq_dequantize": (i32, [ctypes.POINTER(_QTensorC), P, i32, P]),
        "mxq_hadamard_block": (i32, [P, P, i32, i64, i64, i32, P]),
        "mxq_cast": (i32, [P, i64, i32, P, P]),
        "mxq_select_workspace_bytes": (i32, [P, i32, psz]),
        "mxq_select_weight_format": (i32, [P, i32, i64, i64, P, i32, P, P, P, sz, P]),
        "mxq_quantize_mse_workspace_bytes": (i32, [i64, i64, psz]),
        "mxq_quantize_mse": (i32, [P, i32, i64, i64, i32, i32, i32, P, P, P, P, P, sz, P]),
        "mxq_quantize_mx_grid": (i32, [P, i32, i64, i64, i32, i32, ctypes.c_float, i32, P, P, P]),
        "mxq_fit_mx_grid_workspace_bytes": (i32, [i64, i64, i32, psz]),
        "mxq_fit_mx_grid": (i32, [P, i32, i64, i64, i32, i32, P, i32, P, P, sz, P]),
        "mxq_calibrate_workspace_bytes": (i32, [i64, i64, i32, psz]),
        "mxq_calibrate_activation": (i32, [P, i32, i64, i64, P, i32, P, P, P, sz, P]),
        "mxq_calibrate_pick": (i32, [P, P, i32, i32, P, P]),
        "mxq_lowrank_down": (i32, [P, i32, i64, i64, P, i32, P, P]),
        "mxq_lowrank_packed_bytes": (i32, [i64, psz]),
        "mxq_lowrank_down_packed": (i32, [P, i32, i64, i64, P, i32, P, P, P, P]),
        "mxq_lowrank_pack_t": (i32, [P, i32, i64, P, P, P, P]),
        "mxq_lowrank_pack_l2": (i32, [P, i32, i64, P, P]),
        "mxq_qlinear": (i32, [ctypes.POINTER(_QTensorC), ctypes.POINTER(_QTensorC), P, P, P, i32, P]),
        "mxq_qlinear_w4a16": (i32, [P, i64, i64, ctypes.POINTER(_QTensorC), P, i32, P, sz, P]),
        "mxq_qlinear_w4a16_workspace_bytes": (i32, [i64, i64, i64, psz]),
        "mxq_route": (i32, [P, i32, i32, i32, i32, i32]),
        "mxq_quantize_lowrank_workspace_bytes": (i32, [i64, i32, psz]),
        "mxq_quantize_lowrank": (i32, [P, i32, i64, i64, i32, i32, P, i32, P, P, P, P, P, P, sz, P]),
        "mxq_quantize_lowrank_noalloc": (i32, [P, i32, i64, i64, i32, i32, P, i32, P, P, P, P, P, P]),
        "mxq_qlinear_routed_workspace_bytes": (i32, [i64, i64, i32, psz]),
        "mxq_mixed_plan": (i32, [P, i64, ctypes.POINTER(i64), P]),
        "mxq_mixed_weight_bytes": (i32, [ctypes.POINTER(i64), i64, psz]),
        "mxq_mixed_prepare": (i32, [ctypes.POINTER(_QTensorC), ctypes.POINTER(_QTensorC), ctypes.POINTER(_QTensorC),
                                    ctypes.POINTER(_MixedC), P]),
        "mxq_qlinear_mixed_workspace_bytes": (i32, [i64, ctypes.POINTER(_MixedC), i32, psz]),
        "mxq_qlinear_mixed": (i32, [ctypes.POINTER(_QTensorC), ctypes.POINTER(_MixedC), P, i32, P, sz, P]),
        "mxq_qlinear_routed": (i32, [P, i32, i64, i64, ctypes.POINTER(_LayerC), P, i32, i32, i32, i32, i32, P, i32,
                                     ctypes.POINTER(ctypes.c_int32), P, sz, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype, f.argtypes = res, args
    return L


_lib = _load()


def lib():
    return _lib


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None and t.numel() > 0 else None


def _ok(st: int, what: str):
    if st != 0:
        raise MxqError(st, what)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError("expected float32 or bfloat16, got %s" % t.dtype)


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device (there is no CPU path)")


def _size(fn, *args) -> int:
    out = ctypes.c_size_t(0)
    _ok(fn(*args, ctypes.byref(out)), fn.__name__)
    return out.value


@dataclass
class QTensor:
    """A quantized matrix: device tensors for codes, scales, tensor scale."""
    fmt: int
    layout: int
    rows: int
    cols: int
    codes: torch.Tensor
    scales: Optional[torch.Tensor]
    tensor_scale: Optional[torch.Tensor]

    def c(self) -> _QTensorC:
        return _QTensorC(self.fmt, self.layout, self.rows, self.cols, _ptr(self.codes), _ptr(self.scales),
                         _ptr(self.tensor_scale))


def codes_bytes(fmt, rows, cols, layout=CANONICAL) -> int:
    return _size(_lib.mxq_codes_bytes, fmt, rows, cols, layout)


def scales_bytes(fmt, rows, cols, layout=CANONICAL) -> int:
    return _size(_lib.mxq_scales_bytes, fmt, rows, cols, layout)


def alloc_qtensor(fmt, rows, cols, layout=CANONICAL, device="cuda") -> QTensor:
    cb = codes_bytes(fmt, rows, cols, layout)
    sb = scales_bytes(fmt, rows, cols, layout)
    codes = torch.empty(cb, dtype=torch.uint8, device=device)
    scales = torch.empty(max(sb, 1), dtype=torch.uint8, device=device) if sb else None
    ts = torch.empty(1, dtype=torch.float32, device=device) if fmt in (NVFP4, FP8_TENSOR) else None
    return QTensor(fmt, layout, rows, cols, codes, scales, ts)


def quantize_workspace_bytes(fmt) -> int:
    return _size(_lib.mxq_quantize_workspace_bytes, fmt)


def quantize(x: torch.Tensor, fmt: int, hadamard_b: int = 0, layout: int = CANONICAL, out: QTensor = None,
             workspace: torch.Tensor = None, stream=None) -> QTensor:
    """Block-scaled quantization of a 2-D CUDA tensor (fp32 or bf16)."""
    _require_cuda(x)
    x = x.contiguous()
    rows, cols = x.shape
    q = out if out is not None else alloc_qtensor(fmt, rows, cols, layout, x.device)
    wsb = quantize_workspace_bytes(fmt)
    if wsb and workspace is None:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=x.device)
    _ok(_lib.mxq_quantize(_ptr(x), _dtype_code(x), rows, cols, fmt, hadamard_b, layout, _ptr(q.codes),
                          _ptr(q.scales), _ptr(q.tensor_scale), _ptr(workspace), wsb, _stream(stream)),
        "mxq_quantize")
    return q


def dequantize(q: QTensor, dtype=torch.float32, stream=None) -> torch.Tensor:
    y = torch.empty((q.rows, q.cols), dtype=dtype, device=q.codes.device)
    qc = q.c()
    _ok(_lib.mxq_dequantize(ctypes.byref(qc), _ptr(y), _dtype_code(y), _stream(stream)), "mxq_dequantize")
    return y


def hadamard_block(x: torch.Tensor, b: int, out: torch.Tensor = None, stream=None) -> torch.Tensor:
    _require_cuda(x)
    x = x.contiguous()
    y = out if out is not None else torch.empty_like(x)
    rows, cols = x.shape
    _ok(_lib.mxq_hadamard_block(_ptr(x), _ptr(y), _dtype_code(x), rows, cols, b, _stream(stream)),
        "mxq_hadamard_block")
    return y


def cast(x: torch.Tensor, elem: str, out: torch.Tensor = None, stream=None) -> torch.Tensor:
    """Element conversion of fp32 values: 'e4m3' byte or 'e2m1' nibble per element."""
    _require_cuda(x)
    assert x.dtype == torch.float32 and x.is_contiguous()
    y = out if out is not None else torch.empty(x.numel(), dtype=torch.uint8, device=x.device)
    _ok(_lib.mxq_cast(_ptr(x), x.numel(), 0 if elem == "e4m3" else 1, _ptr(y), _stream(stream)), "mxq_cast")
    return y


def select_weight_format(w: torch.Tensor, candidates: Sequence[int], want_sse: bool = True, stream=None):
    """Per-output-channel format choice; returns (uint8 formats, float64 errors or None)."""
    _require_cuda(w)
    w = w.contiguous()
    n, k = w.shape
    cands = (ctypes.c_int32 * len(candidates))(*candidates)
    wsb = _size(_lib.mxq_select_workspace_bytes, cands, len(candidates))
    ws = torch.empty(wsb, dtype=torch.uint8, device=w.device)
    choice = torch.empty(n, dtype=torch.uint8, device=w.device)
    sse = torch.empty((n, len(candidates)), dtype=torch.float64, device=w.device) if want_sse else None
    _ok(_lib.mxq_select_weight_format(_ptr(w), _dtype_code(w), n, k, cands, len(candidates), _ptr(choice),
                                      _ptr(sse), _ptr(ws), wsb, _stream(stream)), "mxq_select_weight_format")
    return choice, sse


def quantize_mse_workspace_bytes(rows: int, cols: int) -> int:
    return _size(_lib.mxq_quantize_mse_workspace_bytes, rows, cols)


def quantize_mse(w: torch.Tensor, iters: int = 2, layout: int = CANONICAL, out: QTensor = None,
                 workspace: torch.Tensor = None, want_sse: bool = True, stream=None):
    """NVFP4 with block and tensor scales fitted to the squared error;
    returns (QTensor, device float64 total error or None)."""
    _require_cuda(w)
    w = w.contiguous()
    rows, cols = w.shape
    q = out if out is not None else alloc_qtensor(NVFP4, rows, cols, layout, w.device)
    wsb = quantize_mse_workspace_bytes(rows, cols)
    ws = workspace if workspace is not None else torch.empty(wsb, dtype=torch.uint8, device=w.device)
    sse = torch.empty(1, dtype=torch.float64, device=w.device) if want_sse else None
    _ok(_lib.mxq_quantize_mse(_ptr(w), _dtype_code(w), rows, cols, NVFP4, iters, layout, _ptr(q.codes),
                              _ptr(q.scales), _ptr(q.tensor_scale), _ptr(sse), _ptr(ws), ws.numel(), _stream(stream)),
        "mxq_quantize_mse")
    return q, sse


def quantize_mx_grid(x: torch.Tensor, fmt: int, grid_scale: float, hadamard_b: int = 0, layout: int = CANONICAL,
                     out: QTensor = None, stream=None) -> QTensor:
    """MXFP4 / MXFP8 with a fixed grid scale g in [1, 2] (g = 1: mxq_quantize)."""
    _require_cuda(x)
    x = x.contiguous()
    rows, cols = x.shape
    q = out if out is not None else alloc_qtensor(fmt, rows, cols, layout, x.device)
    _ok(_lib.mxq_quantize_mx_grid(_ptr(x), _dtype_code(x), rows, cols, fmt, hadamard_b, float(grid_scale), layout,
                                  _ptr(q.codes), _ptr(q.scales), _stream(stream)), "mxq_quantize_mx_grid")
    return q


def fit_mx_grid_workspace_bytes(rows: int, cols: int, n: int) -> int:
    return _size(_lib.mxq_fit_mx_grid_workspace_bytes, rows, cols, n)


def fit_mx_grid(w: torch.Tensor, fmt: int, grid_scales: Sequence[float], hadamard_b: int = 0,
                workspace: torch.Tensor = None, sse: torch.Tensor = None, stream=None):
    """Squared error of w under each candidate grid scale; returns (the
    least-error grid scale, device float64 errors)."""
    _require_cuda(w)
    w = w.contiguous()
    rows, cols = w.shape
    n = len(grid_scales)
    gs = (ctypes.c_float * n)(*grid_scales)
    ws = workspace if workspace is not None else torch.empty(fit_mx_grid_workspace_bytes(rows, cols, n),
                                                             dtype=torch.uint8, device=w.device)
    sse = sse if sse is not None else torch.empty(n, dtype=torch.float64, device=w.device)
    _ok(_lib.mxq_fit_mx_grid(_ptr(w), _dtype_code(w), rows, cols, fmt, hadamard_b, gs, n, _ptr(sse), _ptr(ws),
                             ws.numel(), _stream(stream)), "mxq_fit_mx_grid")
    return None if torch.cuda.is_current_stream_capturing() else grid_scales[int(torch.argmin(sse).item())], sse


def calibrate_workspace_bytes(rows: int, cols: int, ncand: int) -> int:
    return _size(_lib.mxq_calibrate_workspace_bytes, rows, cols, ncand)


def calibrate_activation(x: torch.Tensor, candidates: Sequence[int], sse_accum: torch.Tensor,
                         moments_accum: torch.Tensor, workspace: torch.Tensor = None, stream=None):
    """Adds x's per-candidate squared error to sse_accum (float64[ncand]) and
    (sum x^2, sum x^4) to moments_accum (float64[2])."""
    _require_cuda(x)
    x = x.contiguous()
    rows, cols = x.shape
    n = len(candidates)
    cands = (ctypes.c_int32 * n)(*candidates)
    ws = workspace if workspace is not None else torch.empty(calibrate_workspace_bytes(rows, cols, n),
                                                             dtype=torch.uint8, device=x.device)
    _ok(_lib.mxq_calibrate_activation(_ptr(x), _dtype_code(x), rows, cols, cands, n, _ptr(sse_accum),
                                      _ptr(moments_accum), _ptr(ws), ws.numel(), _stream(stream)),
        "mxq_calibrate_activation")


def calibrate_pick(sse_accum: torch.Tensor, candidates: Sequence[int], entry: torch.Tensor, forced_fmt: int = -1,
                   stream=None):
    """Writes the table entry (a device uint8 view) for the accumulated errors."""
    n = len(candidates)
    cands = (ctypes.c_int32 * n)(*candidates)
    _ok(_lib.mxq_calibrate_pick(_ptr(sse_accum), cands, n, forced_fmt, _ptr(entry), _stream(stream)),
        "mxq_calibrate_pick")


def lowrank_down(x: torch.Tensor, l1: torch.Tensor, out: torch.Tensor = None, stream=None) -> torch.Tensor:
    """t = bf16(x) . l1 in fp32 (l1: k x r bf16)."""
    _require_cuda(x, l1)
    x, l1 = x.contiguous(), l1.contiguous()
    assert l1.dtype == torch.bfloat16
    m, k = x.shape
    r = l1.shape[1]
    t = out if out is not None else torch.empty((m, r), dtype=torch.float32, device=x.device)
    _ok(_lib.mxq_lowrank_down(_ptr(x), _dtype_code(x), m, k, _ptr(l1), r, _ptr(t), _stream(stream)),
        "mxq_lowrank_down")
    return t


def lowrank_pack_l2(l2: torch.Tensor, stream=None) -> torch.Tensor:
    """Packs the up-projection (r x n bf16) as the GEMM operand (n x 64 bf16)."""
    _require_cuda(l2)
    l2 = l2.contiguous()
    assert l2.dtype == torch.bfloat16
    r, n = l2.shape
    l2p = torch.empty((n, 64), dtype=torch.bfloat16, device=l2.device)
    _ok(_lib.mxq_lowrank_pack_l2(_ptr(l2), r, n, _ptr(l2p), _stream(stream)), "mxq_lowrank_pack_l2")
    return l2p


def lowrank_packed_bytes(m: int) -> int:
    return _size(_lib.mxq_lowrank_packed_bytes, m)


def _scales_of(xq: Optional[QTensor], wq: Optional[QTensor]):
    if xq is None or xq.tensor_scale is None:
        return None, None
    return _ptr(xq.tensor_scale), _ptr(wq.tensor_scale)


def lowrank_down_packed(x: torch.Tensor, l1: torch.Tensor, xq: QTensor = None, wq: QTensor = None,
                        out: torch.Tensor = None, stream=None) -> torch.Tensor:
    """Packed low-rank activation (m x 64 bf16) for qlinear, divided by the
    tensor scales of xq and wq when their format has them."""
    _require_cuda(x, l1)
    x, l1 = x.contiguous(), l1.contiguous()
    m, k = x.shape
    r = l1.shape[1]
    tp = out if out is not None else torch.empty((m, 64), dtype=torch.bfloat16, device=x.device)
    xs, ws = _scales_of(xq, wq)
    _ok(_lib.mxq_lowrank_down_packed(_ptr(x), _dtype_code(x), m, k, _ptr(l1), r, xs, ws, _ptr(tp), _stream(stream)),
        "mxq_lowrank_down_packed")
    return tp


def lowrank_pack_t(t: torch.Tensor, xq: QTensor = None, wq: QTensor = None, out: torch.Tensor = None,
                   stream=None) -> torch.Tensor:
    _require_cuda(t)
    t = t.contiguous()
    m, r = t.shape
    tp = out if out is not None else torch.empty((m, 64), dtype=torch.bfloat16, device=t.device)
    xs, ws = _scales_of(xq, wq)
    _ok(_lib.mxq_lowrank_pack_t(_ptr(t), r, m, xs, ws, _ptr(tp), _stream(stream)), "mxq_lowrank_pack_t")
    return tp


def quantize_lowrank_workspace_bytes(m: int, r: int) -> int:
    return _size(_lib.mxq_quantize_lowrank_workspace_bytes, m, r)


def quantize_lowrank(x: torch.Tensor, fmt: int, l1: torch.Tensor, wq: QTensor, hadamard_b: int = 0,
                     out: QTensor = None, tp: torch.Tensor = None, workspace: torch.Tensor = None, stream=None):
    """Quantized activation (MMA layout) and packed low-rank operand in one call; returns (xq, tp)."""
    _require_cuda(x, l1)
    x, l1 = x.contiguous(), l1.contiguous()
    m, k = x.shape
    r = l1.shape[1]
    q = out if out is not None else alloc_qtensor(fmt, m, k, MMA, x.device)
    if tp is None:
        tp = torch.empty((m, 64), dtype=torch.bfloat16, device=x.device)
    wsb = quantize_lowrank_workspace_bytes(m, r)
    if workspace is None:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=x.device)
    _ok(_lib.mxq_quantize_lowrank(_ptr(x), _dtype_code(x), m, k, fmt, hadamard_b, _ptr(l1), r,
                                  _ptr(wq.tensor_scale) if wq is not None else None, _ptr(q.codes), _ptr(q.scales),
                                  _ptr(q.tensor_scale), _ptr(tp), _ptr(workspace), wsb, _stream(stream)),
        "mxq_quantize_lowrank")
    return q, tp


def quantize_lowrank_noalloc(x: torch.Tensor, fmt: int, l1: torch.Tensor, wq: QTensor, hadamard_b: int = 0,
                             out: QTensor = None, tp: torch.Tensor = None, stream=None):
    """quantize_lowrank without a workspace: the library's own 4 MiB device
    scratch array is used (see mxq_quantize_lowrank_noalloc in mxq.h)."""
    _require_cuda(x, l1)
    x, l1 = x.contiguous(), l1.contiguous()
    m, k = x.shape
    r = l1.shape[1]
    q = out if out is not None else alloc_qtensor(fmt, m, k, MMA, x.device)
    if tp is None:
        tp = torch.empty((m, 64), dtype=torch.bfloat16, device=x.device)
    _ok(_lib.mxq_quantize_lowrank_noalloc(_ptr(x), _dtype_code(x), m, k, fmt, hadamard_b, _ptr(l1), r,
                                          _ptr(wq.tensor_scale) if wq is not None else None, _ptr(q.codes),
                                          _ptr(q.scales), _ptr(q.tensor_scale), _ptr(tp), _stream(stream)),
        "mxq_quantize_lowrank_noalloc")
    return q, tp


def qlinear(xq: QTensor, wq: QTensor, tp: torch.Tensor = None, l2p: torch.Tensor = None,
            out_dtype=torch.bfloat16, out: torch.Tensor = None, stream=None) -> torch.Tensor:
    """y = deq(xq) . deq(wq)^T (+ t . l2 from the packed operands) on tcgen05 tensor cores."""
    m, n = xq.rows, wq.rows
    y = out if out is not None else torch.empty((m, n), dtype=out_dtype, device=xq.codes.device)
    xc, wc = xq.c(), wq.c()
    _ok(_lib.mxq_qlinear(ctypes.byref(xc), ctypes.byref(wc), _ptr(tp), _ptr(l2p), _ptr(y), _dtype_code(y),
                         _stream(stream)), "mxq_qlinear")
    return y


def qlinear_w4a16_workspace_bytes(m: int, n: int, k: int) -> int:
    return _size(_lib.mxq_qlinear_w4a16_workspace_bytes, m, n, k)


def qlinear_w4a16(x: torch.Tensor, wq: QTensor, out_dtype=torch.bfloat16, out: torch.Tensor = None,
                  workspace: torch.Tensor = None, fused: bool = False, stream=None) -> torch.Tensor:
    """y = bf16(x) . bf16(q s)^T for an INT4-g32/g64 weight in the canonical
    layout.  With a workspace (allocated here when the library asks for one
    and `fused` is false) the weight is unpacked once and multiplied by the
    bf16 GEMM; otherwise the fused kernel converts it in shared memory."""
    _require_cuda(x)
    assert x.dtype == torch.bfloat16
    x = x.contiguous()
    m, k = x.shape
    y = out if out is not None else torch.empty((m, wq.rows), dtype=out_dtype, device=x.device)
    if fused:
        workspace = None
    elif workspace is None:
        wsb = qlinear_w4a16_workspace_bytes(m, wq.rows, k)
        if wsb:
            workspace = torch.empty(wsb, dtype=torch.uint8, device=x.device)
    wc = wq.c()
    _ok(_lib.mxq_qlinear_w4a16(_ptr(x), m, k, ctypes.byref(wc), _ptr(y), _dtype_code(y), _ptr(workspace),
                               workspace.numel() if workspace is not None else 0, _stream(stream)),
        "mxq_qlinear_w4a16")
    return y


def route(table, layer: int, step: int, n_steps: int) -> int:
    """Format id of `layer` at denoising `step` from a host uint8 table [layers][intervals]."""
    import numpy as np
    tab = np.ascontiguousarray(np.asarray(table, dtype=np.uint8))
    n_layers, n_int = tab.shape
    return _lib.mxq_route(tab.ctypes.data_as(ctypes.c_void_p), n_layers, n_int, layer, step, n_steps)


@dataclass
class RoutedLayer:
    """A linear layer prepared for routed execution: its weight quantized (MMA
    layout) in every format its table row names, and the optional low-rank
    branch (l1: K x r bf16, l2p: packed up projection)."""
    weights: dict
    l1: Optional[torch.Tensor] = None
    l2p: Optional[torch.Tensor] = None
    hadamard_b: int = 0

    def c(self) -> _LayerC:
        lay = _LayerC()
        for f, q in self.weights.items():
            lay.w[f] = q.c()
        lay.l1 = _ptr(self.l1)
        lay.l2p = _ptr(self.l2p)
        lay.r = self.l1.shape[1] if self.l1 is not None else 0
        lay.hadamard_b = self.hadamard_b
        return lay


def prepare_routed_layer(w: torch.Tensor, formats: Sequence[int], l1: torch.Tensor = None, l2: torch.Tensor = None,
                         hadamard_b: int = 0, stream=None) -> RoutedLayer:
    """Quantizes the weight w (N x K) once in each of `formats` (MMA layout)
    and packs the low-rank up projection l2 (r x N bf16) when given."""
    ws = {int(f): quantize(w, int(f), hadamard_b, MMA, stream=stream) for f in sorted(set(int(f) for f in formats))}
    l2p = lowrank_pack_l2(l2, stream=stream) if l2 is not None else None
    return RoutedLayer(ws, l1.contiguous() if l1 is not None else None, l2p, hadamard_b)


def qlinear_routed_workspace_bytes(m: int, k: int, r: int = 0) -> int:
    return _size(_lib.mxq_qlinear_routed_workspace_bytes, m, k, r)


def qlinear_routed(x: torch.Tensor, layer_w: RoutedLayer, table, layer: int, step: int, n_steps: int,
                   out_dtype=torch.bfloat16, out: torch.Tensor = None, workspace: torch.Tensor = None,
                   stream=None):
    """The routed linear layer: reads layer's format for `step` from the host
    table [layers][intervals], quantizes x in it and runs the GEMM against the
    weight prepared in that format.  Returns (y, routed format id)."""
    import numpy as np
    _require_cuda(x)
    x = x.contiguous()
    m, k = x.shape
    n = next(iter(layer_w.weights.values())).rows
    y = out if out is not None else torch.empty((m, n), dtype=out_dtype, device=x.device)
    r = layer_w.l1.shape[1] if layer_w.l1 is not None else 0
    wsb = qlinear_routed_workspace_bytes(m, k, r)
    if workspace is None:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=x.device)
    tab = np.ascontiguousarray(np.asarray(table, dtype=np.uint8))
    n_layers, n_int = tab.shape
    used = ctypes.c_int32(-1)
    lay = layer_w.c()
    _ok(_lib.mxq_qlinear_routed(_ptr(x), _dtype_code(x), m, k, ctypes.byref(lay), tab.ctypes.data_as(ctypes.c_void_p),
                                n_layers, n_int, layer, step, n_steps, _ptr(y), _dtype_code(y), ctypes.byref(used),
                                _ptr(workspace), workspace.numel(), _stream(stream)), "mxq_qlinear_routed")
    return y, used.value


@dataclass
class MixedWeight:
    """A weight whose output channels keep their own format among MXFP4,
    INT4-g32 and NVFP4, laid out as three groups of rows (mxq_mixed_weight)."""
    rows: int
    cols: int
    n_group: tuple
    choice: torch.Tensor
    group_index: torch.Tensor
    mx_codes: torch.Tensor
    mx_scales: torch.Tensor
    i4_codes: torch.Tensor
    i4_scales: torch.Tensor
    nv_values: torch.Tensor
    nv_tensor_scale: torch.Tensor

    def c(self) -> _MixedC:
        return _MixedC(self.rows, self.cols, (ctypes.c_int64 * 3)(*self.n_group), _ptr(self.choice),
                       _ptr(self.group_index), _ptr(self.mx_codes), _ptr(self.mx_scales), _ptr(self.i4_codes),
                       _ptr(self.i4_scales), _ptr(self.nv_values), _ptr(self.nv_tensor_scale))


def prepare_mixed_weight(w: torch.Tensor, choice: torch.Tensor, stream=None) -> MixedWeight:
    """Lays out w (N x K) with each output channel in the format `choice`
    (device or host uint8[N] of MXFP4 / INT4_G32 / NVFP4, e.g. from
    select_weight_format) names: the channel grouping from mxq_mixed_plan,
    the whole weight quantized in each format, then mxq_mixed_prepare."""
    import numpy as np
    _require_cuda(w)
    w = w.contiguous()
    n, k = w.shape
    ch = np.ascontiguousarray(choice.cpu().numpy() if isinstance(choice, torch.Tensor) else choice, dtype=np.uint8)
    n_group = (ctypes.c_int64 * 3)()
    gidx = np.zeros(max(n, 1), np.int32)
    _ok(_lib.mxq_mixed_plan(ch.ctypes.data_as(ctypes.c_void_p), n, n_group, gidx.ctypes.data_as(ctypes.c_void_p)),
        "mxq_mixed_plan")
    sizes = (ctypes.c_size_t * 5)()
    _ok(_lib.mxq_mixed_weight_bytes(n_group, k, sizes), "mxq_mixed_weight_bytes")
    dev = w.device
    buf = [torch.empty(max(int(b), 1), dtype=torch.uint8, device=dev) for b in sizes]
    q = {f: quantize(w, f, stream=stream) for f in (MXFP4, INT4_G32, NVFP4)}
    mw = MixedWeight(n, k, tuple(n_group), torch.from_numpy(ch).to(dev), torch.from_numpy(gidx[:n]).to(dev),
                     buf[0], buf[1], buf[2], buf[3].view(torch.float32) if sizes[3] else buf[3], buf[4],
                     q[NVFP4].tensor_scale)
    mc = mw.c()
    qc = [q[f].c() for f in (MXFP4, INT4_G32, NVFP4)]
    _ok(_lib.mxq_mixed_prepare(ctypes.byref(qc[0]), ctypes.byref(qc[1]), ctypes.byref(qc[2]), ctypes.byref(mc),
                               _stream(stream)), "mxq_mixed_prepare")
    mw._keep = q   # the NVFP4 tensor scale lives in the NVFP4 quantization
    return mw


def qlinear_mixed_workspace_bytes(m: int, mw: MixedWeight, out_dtype=torch.bfloat16) -> int:
    mc = mw.c()
    return _size(_lib.mxq_qlinear_mixed_workspace_bytes, m, ctypes.byref(mc), BF16 if out_dtype == torch.bfloat16 else F32)


def qlinear_mixed(xq: QTensor, mw: MixedWeight, out_dtype=torch.bfloat16, out: torch.Tensor = None,
                  workspace: torch.Tensor = None, stream=None) -> torch.Tensor:
    """y = deq(xq) . deq(W)^T for an MXFP8 (MMA layout) activation and a
    weight with per-channel formats."""
    m = xq.rows
    y = out if out is not None else torch.empty((m, mw.rows), dtype=out_dtype, device=xq.codes.device)
    mc, xc = mw.c(), xq.c()
    wsb = _size(_lib.mxq_qlinear_mixed_workspace_bytes, m, ctypes.byref(mc), _dtype_code(y))
    if workspace is None:
        workspace = torch.empty(max(wsb, 1), dtype=torch.uint8, device=xq.codes.device)
    _ok(_lib.mxq_qlinear_mixed(ctypes.byref(xc), ctypes.byref(mc), _ptr(y), _dtype_code(y), _ptr(workspace),
                               workspace.numel(), _stream(stream)), "mxq_qlinear_mixed")
    return y


def check(stream=None) -> int:
    """Synchronizes and returns the status of bounded device waits (0 = ok)."""
    return _lib.mxq_check(_stream(stream))
