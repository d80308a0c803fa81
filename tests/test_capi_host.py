"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/mxq.h declares, sizes and routing agree with the
documented formulas, and bad arguments are rejected before any launch."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def mxq():
    import __graft_entry__
    __graft_entry__.build()   # loads build.py by path, so a stale library cannot get in the way
    import microscaling_bit_quantization_b200 as m
    return m


def _declared():
    src = open(os.path.join(ROOT, "include", "mxq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mxq_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(mxq):
    names = _declared()
    assert len(names) >= 15
    lib = ctypes.CDLL(mxq.LIB_PATH)
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(mxq.EXPORTS)


def test_status_strings(mxq):
    for code in range(6):
        assert mxq.lib().mxq_status_string(code)


def test_sizes(mxq):
    M = mxq
    assert M.codes_bytes(M.NVFP4, 64, 256) == 64 * 128
    assert M.codes_bytes(M.MXFP8, 64, 256) == 64 * 256
    assert M.codes_bytes(M.INT4_G64, 64, 256, M.MMA) == 64 * 256
    assert M.scales_bytes(M.NVFP4, 64, 256) == 64 * 16
    assert M.scales_bytes(M.NVFP4, 64, 256, M.MMA) == 128 * 16
    assert M.scales_bytes(M.MXFP4, 300, 96, M.MMA) == 384 * 16
    assert M.scales_bytes(M.MXFP8, 4096, 3072, M.MMA) == 4096 * 96
    assert M.scales_bytes(M.INT4_G32, 10, 64) == 10 * 2 * 4
    assert M.scales_bytes(M.INT8_ROW, 10, 64) == 40
    assert M.scales_bytes(M.FP8_TENSOR, 10, 64) == 0
    assert M.quantize_workspace_bytes(M.NVFP4) >= 4 and M.quantize_workspace_bytes(M.MXFP8) == 0
    assert M.lowrank_packed_bytes(4096) == 4096 * 128


def test_bad_shapes_rejected_on_host(mxq):
    L, P = mxq.lib(), ctypes.c_void_p
    size = ctypes.c_size_t(0)
    assert L.mxq_codes_bytes(mxq.MXFP8, 4, 48, 0, ctypes.byref(size)) == 1          # 48 % 32
    assert L.mxq_codes_bytes(mxq.INT4_G64, 4, 96, 0, ctypes.byref(size)) == 1       # 96 % 64
    assert L.mxq_codes_bytes(9, 4, 64, 0, ctypes.byref(size)) == 1                  # bad fmt
    dummy = P(256)
    # cols not a multiple of 16, hadamard not a power of two, null pointers
    assert L.mxq_quantize(dummy, 1, 4, 40, mxq.INT8_ROW, 0, 0, dummy, dummy, None, None, 0, None) == 1
    assert L.mxq_quantize(dummy, 1, 4, 64, mxq.MXFP8, 48, 0, dummy, dummy, None, None, 0, None) == 1
    assert L.mxq_quantize(None, 1, 4, 64, mxq.MXFP8, 0, 0, dummy, dummy, None, None, 0, None) == 1
    # NVFP4 needs a tensor-scale pointer and workspace
    assert L.mxq_quantize(dummy, 1, 4, 64, mxq.NVFP4, 0, 0, dummy, dummy, None, dummy, 16, None) == 1
    assert L.mxq_quantize(dummy, 1, 4, 64, mxq.NVFP4, 0, 0, dummy, dummy, dummy, dummy, 2, None) == 5
    assert L.mxq_hadamard_block(dummy, dummy, 1, 4, 64, 3, None) == 1
    assert L.mxq_hadamard_block(dummy, dummy, 1, 4, 64, 512, None) == 1
    assert L.mxq_lowrank_down(dummy, 1, 4, 64, dummy, 33, dummy, None) == 1
    assert L.mxq_cast(dummy, 10, 2, dummy, None) == 1


def test_quantize_mse_argument_checks(mxq):
    L, P = mxq.lib(), ctypes.c_void_p
    size = ctypes.c_size_t(0)
    assert L.mxq_quantize_mse_workspace_bytes(4, 64, ctypes.byref(size)) == 0
    assert size.value == 256 + 4 * 4 * 16 + 4 * 16 + 16
    assert L.mxq_quantize_mse_workspace_bytes(300, 32, ctypes.byref(size)) == 0
    assert size.value == 256 + 600 * 16 + 300 * 16 + 3 * 16
    assert L.mxq_quantize_mse_workspace_bytes(4, 40, ctypes.byref(size)) == 1
    d = P(256)

    def call(fmt=mxq.NVFP4, iters=2, cols=64, ts=d, ws=d, wsb=1 << 20):
        return L.mxq_quantize_mse(d, 1, 4, cols, fmt, iters, 0, d, d, ts, None, ws, wsb, None)

    assert call(fmt=mxq.MXFP4) == 2          # NVFP4 only
    assert call(iters=-1) == 1
    assert call(cols=40) == 1
    assert call(ts=None) == 1
    assert call(ws=None) == 1
    assert call(wsb=64) == 5                 # workspace too small
    assert call(ws=P(256 + 8)) == 1          # workspace not 256-byte aligned


def test_mx_grid_argument_checks(mxq):
    L, P = mxq.lib(), ctypes.c_void_p
    size = ctypes.c_size_t(0)
    assert L.mxq_fit_mx_grid_workspace_bytes(300, 64, 3, ctypes.byref(size)) == 0
    assert size.value == 256 + 8 * 3 * 600 + 8 * 300 + 8 * 3
    assert L.mxq_fit_mx_grid_workspace_bytes(4, 48, 1, ctypes.byref(size)) == 1     # 48 % 32
    assert L.mxq_fit_mx_grid_workspace_bytes(4, 64, 9, ctypes.byref(size)) == 1     # more than 8 candidates
    d = P(256)
    q = L.mxq_quantize_mx_grid
    assert q(d, 1, 4, 64, mxq.NVFP4, 0, ctypes.c_float(1.0), 0, d, d, None) == 2   # MX formats only
    assert q(d, 1, 4, 64, mxq.MXFP4, 0, ctypes.c_float(0.75), 0, d, d, None) == 1  # g outside [1, 2]
    assert q(d, 1, 4, 64, mxq.MXFP4, 0, ctypes.c_float(2.5), 0, d, d, None) == 1
    assert q(d, 1, 4, 64, mxq.MXFP4, 48, ctypes.c_float(1.0), 0, d, d, None) == 1  # bad Hadamard size
    gs = (ctypes.c_float * 2)(1.0, 3.0)
    fit = L.mxq_fit_mx_grid
    assert fit(d, 1, 4, 64, mxq.MXFP4, 0, gs, 2, d, d, 1 << 20, None) == 1         # 3.0 outside [1, 2]
    gs[1] = 1.5
    assert fit(d, 1, 4, 64, mxq.MXFP4, 0, gs, 0, d, d, 1 << 20, None) == 1         # no candidates
    assert fit(d, 1, 4, 64, mxq.MXFP4, 0, gs, 2, d, d, 16, None) == 5              # workspace too small
    assert fit(d, 1, 4, 64, mxq.INT4_G32, 0, gs, 2, d, d, 1 << 20, None) == 2


def test_calibration_argument_checks(mxq):
    L, P = mxq.lib(), ctypes.c_void_p
    size = ctypes.c_size_t(0)
    assert L.mxq_calibrate_workspace_bytes(300, 1152, 3, ctypes.byref(size)) == 0 and size.value > 300 * 3 * 8
    assert L.mxq_calibrate_workspace_bytes(4, 48, 3, ctypes.byref(size)) == 1      # 48 % 64
    d = P(256)
    c3 = (ctypes.c_int32 * 3)(5, 6, 0)
    cal = L.mxq_calibrate_activation
    assert cal(d, 1, 4, 64, c3, 0, d, d, d, 1 << 20, None) == 1                  # no candidates
    assert cal(d, 1, 4, 64, c3, 3, None, d, d, 1 << 20, None) == 1               # no accumulator
    assert cal(d, 1, 4, 64, c3, 3, d, d, d, 16, None) == 5                       # workspace too small
    bad = (ctypes.c_int32 * 1)(9)
    assert cal(d, 1, 4, 64, bad, 1, d, d, d, 1 << 20, None) == 1                 # bad format id
    pick = L.mxq_calibrate_pick
    assert pick(d, c3, 3, 9, d, None) == 1                                       # bad forced format
    assert pick(None, c3, 3, -1, d, None) == 1


def test_w4a16_argument_checks(mxq):
    L = mxq.lib()
    P = ctypes.c_void_p
    d = P(256)

    def qt(fmt, layout, rows, cols):
        return mxq._QTensorC(fmt, layout, rows, cols, 256, 256, None)

    call = lambda q, k=128, yd=1: L.mxq_qlinear_w4a16(d, 4, k, ctypes.byref(q), d, yd, None, 0, None)
    assert call(qt(mxq.NVFP4, 0, 8, 128)) == 2            # INT4 groups only
    assert call(qt(mxq.INT4_G64, 1, 8, 128)) == 1         # canonical layout only
    assert call(qt(mxq.INT4_G64, 0, 8, 96), k=96) == 1    # k % 64
    assert call(qt(mxq.INT4_G64, 0, 8, 192), k=128) == 1  # cols != k
    assert call(qt(mxq.INT4_G32, 0, 8, 128), yd=7) == 1   # bad output dtype
    big = qt(mxq.INT4_G64, 0, (1 << 31) - 1, 1 << 20)
    assert L.mxq_qlinear_w4a16(d, (1 << 31) - 1, 1 << 20, ctypes.byref(big), d, 1, None, 0, None) == 1   # stage count
    # every factor at its largest: the product of tiles and stages (about 2^73) must not wrap around
    kmax = (1 << 31) - 64
    huge = qt(mxq.INT4_G64, 0, (1 << 31) - 1, kmax)
    assert L.mxq_qlinear_w4a16(d, (1 << 31) - 1, kmax, ctypes.byref(huge), d, 1, None, 0, None) == 1
    size = ctypes.c_size_t(0)
    assert L.mxq_qlinear_w4a16_workspace_bytes(4096, 12288, 3072, ctypes.byref(size)) == 0
    assert size.value == 12288 * 3072 * 2   # large m: the unpacked bf16 weight
    assert L.mxq_qlinear_w4a16_workspace_bytes(64, 12288, 3072, ctypes.byref(size)) == 0 and size.value == 0
    assert L.mxq_qlinear_w4a16_workspace_bytes(64, 128, 96, ctypes.byref(size)) == 1   # k % 64


def test_qlinear_argument_checks(mxq):
    L = mxq.lib()
    Q = mxq._QTensorC
    y = ctypes.c_void_p(256)
    a = Q(mxq.NVFP4, mxq.MMA, 64, 256, 256, 256, 256)
    b = Q(mxq.MXFP4, mxq.MMA, 128, 256, 256, 256, 256)
    assert L.mxq_qlinear(ctypes.byref(a), ctypes.byref(b), None, None, y, 0, None) == 2   # format pair
    b = Q(mxq.NVFP4, mxq.CANONICAL, 128, 256, 256, 256, 256)
    assert L.mxq_qlinear(ctypes.byref(a), ctypes.byref(b), None, None, y, 0, None) == 1   # layout
    b = Q(mxq.NVFP4, mxq.MMA, 128, 192, 256, 256, 256)
    assert L.mxq_qlinear(ctypes.byref(a), ctypes.byref(b), None, None, y, 0, None) == 1   # K mismatch
    i4 = Q(mxq.INT4_G64, mxq.MMA, 64, 96, 256, 256, 0)
    assert L.mxq_qlinear(ctypes.byref(i4), ctypes.byref(i4), None, None, y, 0, None) == 1   # K % 64 (group)
    i4 = Q(mxq.INT4_G32, mxq.CANONICAL, 64, 96, 256, 256, 0)
    assert L.mxq_qlinear(ctypes.byref(i4), ctypes.byref(i4), None, None, y, 0, None) == 1   # layout
    a = Q(mxq.NVFP4, mxq.MMA, 64, 96, 256, 256, 256)
    assert L.mxq_qlinear(ctypes.byref(a), ctypes.byref(a), None, None, y, 0, None) == 1   # K % 64
    big_a = Q(mxq.MXFP8, mxq.MMA, 1 << 26, 32, 256, 256, 0)
    big_b = Q(mxq.MXFP8, mxq.MMA, 1 << 26, 32, 256, 256, 0)
    assert L.mxq_qlinear(ctypes.byref(big_a), ctypes.byref(big_b), None, None, y, 0, None) == 1   # tile count
    i8 = Q(mxq.INT8_ROW, mxq.MMA, 64, 256, 256, 256, 0)
    t = ctypes.c_void_p(256)
    assert L.mxq_qlinear(ctypes.byref(i8), ctypes.byref(i8), t, t, y, 0, None) == 2       # branch on INT8
    a = Q(mxq.NVFP4, mxq.MMA, 64, 256, 256, 256, 256)
    assert L.mxq_qlinear(ctypes.byref(a), ctypes.byref(a), t, None, y, 0, None) == 1      # branch without l2p
    assert L.mxq_lowrank_down_packed(t, 1, 4, 64, t, 8, t, None, t, None) == 1             # one tensor scale


def test_noalloc_rejects_arguments_before_any_cuda_call(mxq):
    """The allocation-free entry point checks every argument before it looks
    up its device array: on this GPU-less host a CUDA call would fail, so a
    plain MXQ_EINVAL / MXQ_EUNSUPPORTED shows that none was made."""
    L, P = mxq.lib(), ctypes.c_void_p
    d = P(256)
    call = L.mxq_quantize_lowrank_noalloc
    assert call(d, 1, 64, 256, 9, 0, d, 32, d, d, d, d, d, None) == 1          # bad format
    assert call(d, 1, 64, 256, mxq.NVFP4, 3, d, 32, d, d, d, d, d, None) == 1  # bad rotation size
    assert call(d, 1, 64, 256, mxq.NVFP4, 0, d, 33, d, d, d, d, d, None) == 1  # rank above 32
    assert call(d, 1, 64, 256, mxq.NVFP4, 0, d, 32, None, d, d, d, d, None) == 1   # no weight tensor scale
    assert call(None, 1, 64, 256, mxq.NVFP4, 0, d, 32, d, d, d, d, d, None) == 1   # no input
    assert call(d, 1, 64, 256, mxq.INT8_ROW, 0, d, 32, d, d, d, d, d, None) == 2   # no branch on INT8
    assert call(d, 1, 40000, 512, mxq.NVFP4, 0, d, 32, d, d, d, d, d, None) == 5   # beyond the 4 MiB array


def _routed_layout(m, k, r):
    up = lambda b: (b + 255) // 256 * 256
    rnd = lambda a, b: (a + b - 1) // b * b
    total = up(4096 + 4 * m * r) + up(m * k)
    total += up(max(rnd(m, 128) * rnd(k // 16, 16), m * (k // 32) * 4, 4 * m)) + up(4)
    return total + (up(128 * m) if r else 0)


def test_routed_workspace_and_argument_checks(mxq):
    L, P = mxq.lib(), ctypes.c_void_p
    size = ctypes.c_size_t(0)
    for m, k, r in ((8192, 1152, 0), (8192, 4608, 0), (4096, 3072, 32), (1, 16, 8), (0, 64, 0)):
        assert L.mxq_qlinear_routed_workspace_bytes(m, k, r, ctypes.byref(size)) == 0
        assert size.value == _routed_layout(m, k, r), (m, k, r)
    assert L.mxq_qlinear_routed_workspace_bytes(4, 40, 0, ctypes.byref(size)) == 1      # k % 16
    assert L.mxq_qlinear_routed_workspace_bytes(4, 64, 33, ctypes.byref(size)) == 1     # rank
    Q = mxq._QTensorC
    m, k, n = 64, 256, 128
    lay = mxq._LayerC()
    lay.w[mxq.MXFP8] = Q(mxq.MXFP8, mxq.MMA, n, k, 256, 256, None)
    lay.w[mxq.INT8_ROW] = Q(mxq.INT8_ROW, mxq.MMA, n, k, 256, 256, None)
    table = np.array([[mxq.MXFP8, mxq.INT8_ROW, mxq.NVFP4]], np.uint8)
    tp = table.ctypes.data_as(P)
    d = P(256)
    ws = P(1 << 20)
    used = ctypes.c_int32(-1)

    def call(step=0, n_steps=3, layer=0, lay=lay, ws=ws, wsb=1 << 24, x=d):
        return L.mxq_qlinear_routed(x, 1, m, k, ctypes.byref(lay), tp, 1, 3, layer, step, n_steps, d, 1,
                                    ctypes.byref(used), ws, wsb, None)

    assert call(step=3) == 1                     # step out of range
    assert call(layer=1) == 1                    # layer out of range
    assert call(n_steps=0) == 1
    assert call(step=2) == 1 and used.value == mxq.NVFP4   # routed to a format the layer was not prepared in
    assert call(wsb=1024) == 5                   # workspace too small
    assert call(ws=P((1 << 20) + 16)) == 1       # workspace not 256-byte aligned
    assert call(x=None) == 1                     # the quantizer's own checks apply
    lay.r, lay.l1, lay.l2p = 8, 256, 256
    assert call(step=1) == 2 and used.value == mxq.INT8_ROW   # a branch on an INT8 entry
    lay.w[mxq.MXFP8].cols = 512
    assert call(step=0) == 1                     # weight K differs from x


def test_mixed_plan_and_sizes(mxq):
    L = mxq.lib()
    ch = np.array([1, 2, 3, 2, 1, 1, 3, 2, 2], np.uint8)
    ng = (ctypes.c_int64 * 3)()
    gi = np.zeros(len(ch), np.int32)
    assert L.mxq_mixed_plan(ch.ctypes.data_as(ctypes.c_void_p), len(ch), ng, gi.ctypes.data_as(ctypes.c_void_p)) == 0
    assert list(ng) == [3, 2, 4]
    assert gi.tolist() == [0, 0, 0, 1, 1, 2, 1, 2, 3]
    bad = np.array([1, 0], np.uint8)   # MXFP8 is not a weight candidate
    assert L.mxq_mixed_plan(bad.ctypes.data_as(ctypes.c_void_p), 2, ng, gi.ctypes.data_as(ctypes.c_void_p)) == 1
    sizes = (ctypes.c_size_t * 5)()
    g3 = (ctypes.c_int64 * 3)(3, 2, 4)
    assert L.mxq_mixed_weight_bytes(g3, 256, sizes) == 0
    assert list(sizes) == [3 * 256, 128 * 16, 2 * 256, 2 * 8 * 4, 4 * 256 * 2]
    assert L.mxq_mixed_weight_bytes(g3, 48, sizes) == 1    # k % 32
    mw = mxq._MixedC(9, 256, (ctypes.c_int64 * 3)(3, 2, 4), 256, 256, 256, 256, 256, 256, 256, 256)
    size = ctypes.c_size_t(0)
    assert L.mxq_qlinear_mixed_workspace_bytes(100, ctypes.byref(mw), 1, ctypes.byref(size)) == 0
    up = lambda b: (b + 255) // 256 * 256
    assert size.value == up(100 * 8 * 4) + up(100 * 256 * 2) + up(100 * 3 * 2) + up(100 * 2 * 2) + up(100 * 4 * 2)
    single = mxq._MixedC(9, 256, (ctypes.c_int64 * 3)(0, 0, 9), 256, 256, 256, 256, 256, 256, 256, 256)
    assert L.mxq_qlinear_mixed_workspace_bytes(100, ctypes.byref(single), 1, ctypes.byref(size)) == 0
    assert size.value == up(100 * 256 * 2)          # the bf16 activation only: the GEMM writes y itself
    wrong = mxq._MixedC(9, 256, (ctypes.c_int64 * 3)(3, 2, 3), 256, 256, 256, 256, 256, 256, 256, 256)
    assert L.mxq_qlinear_mixed_workspace_bytes(100, ctypes.byref(wrong), 1, ctypes.byref(size)) == 1   # counts != N
    xq = mxq._QTensorC(mxq.NVFP4, mxq.MMA, 100, 256, 256, 256, 256)
    assert L.mxq_qlinear_mixed(ctypes.byref(xq), ctypes.byref(mw), ctypes.c_void_p(256), 1, ctypes.c_void_p(256),
                               1 << 30, None) == 1        # activation must be MXFP8


def test_route_matches_oracle(mxq, orc):
    rng = np.random.default_rng(3)
    for n_layers, n_int, n_steps in ((112, 10, 20), (7, 3, 11), (1, 1, 1)):
        table = rng.integers(0, 7, size=(n_layers, n_int)).astype(np.uint8)
        for layer in range(n_layers):
            for step in range(-1, n_steps + 1):
                assert mxq.route(table, layer, step, n_steps) == orc.route(table, n_layers, n_int, layer, step, n_steps)


def test_last_cuda_error_string(mxq):
    """Before any CUDA failure the thread's last error reads as no error; the
    Python error for MXQ_ECUDA names the CUDA error through it."""
    s = mxq.lib().mxq_last_cuda_error_string()
    assert isinstance(s, bytes) and len(s) > 0
    assert b"no error" in s.lower()
