"""GPU parity of the HBM-bound kernels against the oracle: quantize (every
format, fp32/bf16 input, both layouts, with and without Hadamard),
dequantize, the Hadamard rotation, the element casts (exhaustively over all
2^32 fp32 bit patterns) and the per-channel format selection.  Codes,
scales and choices must match bit for bit."""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import assert_qtensor_equal, byte_scales_from_mma, dev, host_values, nasty_matrix

pytestmark = pytest.mark.gpu

ALL_FMTS = (0, 1, 2, 3, 4, 5, 6)


@pytest.fixture(scope="module")
def mxq():
    import microscaling_bit_quantization_b200 as m
    assert torch.cuda.is_available() and m.lib().mxq_device_supported(0) == 1
    return m


def _moderate(x):
    x = x.copy()
    x[3, :] = np.clip(x[3, :], -1e4, 1e4)   # keep Hadamard sums finite
    return x


@pytest.mark.parametrize("fmt", ALL_FMTS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("hadamard_b", [0, 2, 32, 128, 256])
def test_quantize_small_ragged(mxq, orc, fmt, dtype, hadamard_b):
    rows, cols = 37, 512
    x = nasty_matrix(100 + fmt, rows, cols)
    if hadamard_b:
        x = _moderate(x)
    xv = host_values(x, dtype)
    ref = orc.quantize(xv, fmt, hadamard_b)
    for layout in (mxq.CANONICAL, mxq.MMA):
        q = mxq.quantize(dev(x, dtype), fmt, hadamard_b, layout)
        torch.cuda.synchronize()
        assert_qtensor_equal(q, ref, layout_mma=layout == mxq.MMA)


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("rows,cols", [(37, 1088), (300, 1152), (128, 1152), (1, 64)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_quantize_mma_scale_padding(mxq, orc, fmt, rows, cols, dtype):
    """The MMA layout pads the byte scales to 16 columns and 128 rows; the
    quantizer writes those padding bytes as zero itself, so a scale buffer
    that held 0xFF (a NaN E8M0 scale) before the call reads as the oracle's
    scales plus zero padding after it."""
    x = nasty_matrix(500 + fmt + rows, rows, cols)
    ref = orc.quantize(host_values(x, dtype), fmt)
    q = mxq.alloc_qtensor(fmt, rows, cols, mxq.MMA)
    for _ in range(2):   # the second call writes over its own output
        q.codes.fill_(0xFF)
        q.scales.fill_(0xFF)
        mxq.quantize(dev(x, dtype), fmt, 0, mxq.MMA, out=q)
        torch.cuda.synchronize()
        assert_qtensor_equal(q, ref, layout_mma=True)


@pytest.mark.parametrize("rows,cols", [(4097, 2064), (5, 5120), (3, 2560), (1, 4096), (1027, 4608), (6, 5136),
                                       (2, 2048)])
def test_quantize_int8_row_long_rows(mxq, orc, rows, cols):
    """INT8 per row over bf16 rows longer than 2048 elements, where rows are
    coded in blocks of 4 staged in shared memory: ragged last blocks, single
    rows, the longest row that path takes (5120) and rows just outside it on
    both sides; every code and scale."""
    x = nasty_matrix(300 + rows % 97 + cols % 89, rows, cols)
    ref = orc.quantize(host_values(x, "bf16"), mxq.INT8_ROW)
    for layout in (mxq.CANONICAL, mxq.MMA):
        q = mxq.quantize(dev(x, "bf16"), mxq.INT8_ROW, 0, layout)
        torch.cuda.synchronize()
        assert_qtensor_equal(q, ref, layout_mma=layout == mxq.MMA)


@pytest.mark.parametrize("fmt", ALL_FMTS)
def test_quantize_edge_shapes(mxq, orc, fmt):
    blk = {0: 32, 1: 32, 2: 16, 3: 32, 4: 64, 5: 16, 6: 16}[fmt]
    for rows, cols in ((0, 64), (1, 64), (129, blk), (3, 1024 + 64)):
        x = nasty_matrix(7, max(rows, 1), cols)[:rows]
        ref = orc.quantize(x, fmt) if rows else None
        for layout in (mxq.CANONICAL, mxq.MMA):
            q = mxq.quantize(dev(x, "f32"), fmt, 0, layout)
            torch.cuda.synchronize()
            if rows:
                assert_qtensor_equal(q, ref, layout_mma=layout == mxq.MMA)
            elif fmt in (2, 6):
                assert q.tensor_scale.item() == 1.0
    # all-zero tensor
    z = np.zeros((8, 128), np.float32)
    q = mxq.quantize(dev(z, "bf16"), fmt)
    assert_qtensor_equal(q, orc.quantize(z, fmt))


def test_quantize_full_size_workloads(mxq, orc):
    """Each workload's activations (and weights) at full size, every element."""
    w2 = workloads.chameleon_selection()
    q = mxq.quantize(dev(w2["x"], "bf16"), mxq.MXFP8, 0, mxq.MMA)
    assert_qtensor_equal(q, orc.quantize(w2["x"], mxq.MXFP8), layout_mma=True)
    del w2
    w3 = workloads.svdquant_mlp_up()
    for fmt in (mxq.NVFP4, mxq.INT4_G64):
        for name in ("x", "w"):
            q = mxq.quantize(dev(w3[name], "bf16"), fmt, 0, mxq.MMA)
            assert_qtensor_equal(q, orc.quantize(w3[name], fmt), layout_mma=True)
    del w3
    w4 = workloads.mxfp4_hadamard_gemm()
    for hb in (0, 128):
        for name in ("x", "w"):   # activations and the weight, with and without the rotation
            q = mxq.quantize(dev(w4[name], "bf16"), mxq.MXFP4, hb, mxq.MMA)
            assert_qtensor_equal(q, orc.quantize(w4[name], mxq.MXFP4, hb), layout_mma=True)
    w1 = workloads.tiny_nvfp4_linear()
    q = mxq.quantize(dev(w1["x"], "f32"), mxq.NVFP4)
    assert_qtensor_equal(q, orc.quantize(w1["x"], mxq.NVFP4))


def test_quantize_dit_activations(mxq, orc):
    """Workload 5 activations at full size (M = 8192, both widths): the tail
    index of the first, middle and last steps, the three routed formats, and a
    forced layer's input with its 163x column spread; every element."""
    seed = 5
    table, forced = workloads.dit_format_table(seed)
    for step in (0, 9, 19):
        for width in (workloads.DIT_HIDDEN, workloads.DIT_MLP):
            x = workloads.dit_activation(seed, step, width)
            xd = dev(x, "bf16")
            for fmt in (mxq.INT8_ROW, mxq.FP8_TENSOR, mxq.MXFP8):
                q = mxq.quantize(xd, fmt, 0, mxq.MMA)
                assert_qtensor_equal(q, orc.quantize(x, fmt), layout_mma=True)
            del xd, q
    for layer in forced[:2]:
        x = workloads.dit_layer_input(seed, 4, int(layer), forced)
        q = mxq.quantize(dev(x, "bf16"), mxq.MXFP8, 0, mxq.MMA)
        assert_qtensor_equal(q, orc.quantize(x, mxq.MXFP8), layout_mma=True)


@pytest.mark.parametrize("fmt", ALL_FMTS)
@pytest.mark.parametrize("layout", [0, 1])
def test_dequantize(mxq, orc, fmt, layout):
    x = nasty_matrix(200 + fmt, 29, 256)
    oq = orc.quantize(x, fmt)
    q = mxq.quantize(dev(x, "f32"), fmt, 0, layout)
    want = orc.dequantize_f32(oq)
    y32 = mxq.dequantize(q, torch.float32).cpu().numpy()
    np.testing.assert_array_equal(y32.view(np.uint32), want.view(np.uint32))
    y16 = mxq.dequantize(q, torch.bfloat16).cpu()
    want16 = torch.from_numpy(want).to(torch.bfloat16)
    assert torch.equal(y16.view(torch.int16), want16.view(torch.int16))


@pytest.mark.parametrize("b", [2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_block(mxq, orc, b):
    x = _moderate(nasty_matrix(300 + b, 45, 512))
    y = mxq.hadamard_block(dev(x, "f32"), b).cpu().numpy()
    np.testing.assert_array_equal(y.view(np.uint32), orc.hadamard(x, b).view(np.uint32))
    xb = host_values(x, "bf16")
    yb = mxq.hadamard_block(dev(x, "bf16"), b).cpu()
    want = torch.from_numpy(orc.hadamard(xb, b)).to(torch.bfloat16)
    assert torch.equal(yb.view(torch.int16), want.view(torch.int16))


def test_hadamard_full_size(mxq, orc):
    w4 = workloads.mxfp4_hadamard_gemm()
    x = w4["w"]
    y = mxq.hadamard_block(dev(x, "f32"), 128).cpu().numpy()
    np.testing.assert_array_equal(y.view(np.uint32), orc.hadamard(x, 128).view(np.uint32))


@pytest.mark.parametrize("elem", ["e4m3", "e2m1"])
def test_cast_exhaustive(mxq, orc, elem):
    """Every fp32 bit pattern (NaN inputs excluded for E2M1, which has no NaN)."""
    chunk = 1 << 27
    bad = 0
    for start in range(0, 1 << 32, chunk):
        bits = torch.arange(start, start + chunk, dtype=torch.int64, device="cuda")
        x = bits.to(torch.int32).view(torch.float32) if start < (1 << 31) else \
            (bits - (1 << 32)).to(torch.int32).view(torch.float32)
        got = mxq.cast(x.contiguous(), elem)
        want = torch.from_numpy(orc.cast_range(start, chunk, elem)).cuda()
        if elem == "e2m1":
            keep = ~torch.isnan(x)
            bad += int((got[keep] != want[keep]).sum())
        else:
            bad += int((got != want).sum())
        del bits, x, got, want
    assert bad == 0


def _near_tie_ok(choice_gpu, choice_ref, sse_ref, cands):
    """Rows may differ only where the oracle's best two errors are within 1e-12 relative."""
    diff = np.nonzero(choice_gpu != choice_ref)[0]
    for r in diff:
        s = np.sort(sse_ref[r])
        assert s[1] - s[0] <= 1e-12 * max(s[0], 1e-300), (r, sse_ref[r])
    return len(diff)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_select_small(mxq, orc, dtype):
    x = nasty_matrix(400, 40, 256)
    x = host_values(_moderate(x), dtype)
    cands = [mxq.INT4_G32, mxq.NVFP4, mxq.MXFP4, mxq.MXFP8, mxq.INT8_ROW, mxq.FP8_TENSOR, mxq.INT4_G64]
    ch, sse = mxq.select_weight_format(dev(x, dtype), cands)
    ref_ch, ref_sse = orc.select_weight_format(x, cands)
    np.testing.assert_allclose(sse.cpu().numpy(), ref_sse, rtol=1e-12, atol=0)
    _near_tie_ok(ch.cpu().numpy(), ref_ch, ref_sse, cands)


def test_select_constructed_rows(mxq, orc):
    """The oracle's constructed rows (exact ties, strict winners) choose identically."""
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    rng = np.random.default_rng(23)
    w = np.zeros((4, 64), np.float32)
    w[0] = rng.choice(grid, 64) * 448
    w[0, ::16] = 2688
    w[1] = rng.choice(grid, 64) * rng.choice([-1, 1], 64)
    w[1, ::16] = 6
    w[2] = w[1] * np.float32(2.0 ** -20)
    w[3] = rng.integers(-7, 8, 64) * np.float32(0.25)
    w[3, 0], w[3, 32] = 1.75, -1.75
    for cands in ([mxq.INT4_G32, mxq.NVFP4, mxq.MXFP4], [mxq.INT4_G32, mxq.MXFP4, mxq.NVFP4]):
        ch, sse = mxq.select_weight_format(dev(w, "f32"), cands)
        ref_ch, ref_sse = orc.select_weight_format(w, cands)
        np.testing.assert_array_equal(ch.cpu().numpy(), ref_ch)
        np.testing.assert_array_equal(sse.cpu().numpy() == 0, ref_sse == 0)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_select_fixed_sets_small(mxq, orc, dtype):
    """The two candidate sets with a specialised kernel ({MXFP4, NVFP4,
    INT4-g32} and {MXFP8, INT8 row, FP8 tensor}), in two orders each, on the
    nasty inputs: errors to 1e-12 relative, choices up to near-ties."""
    x = host_values(_moderate(nasty_matrix(401, 70, 320)), dtype)
    for cands in ([mxq.INT4_G32, mxq.NVFP4, mxq.MXFP4], [mxq.MXFP4, mxq.INT4_G32, mxq.NVFP4],
                  [mxq.INT8_ROW, mxq.FP8_TENSOR, mxq.MXFP8], [mxq.MXFP8, mxq.INT8_ROW, mxq.FP8_TENSOR]):
        ch, sse = mxq.select_weight_format(dev(x, dtype), cands)
        ref_ch, ref_sse = orc.select_weight_format(x, cands)
        np.testing.assert_allclose(sse.cpu().numpy(), ref_sse, rtol=1e-12, atol=0)
        np.testing.assert_array_equal(sse.cpu().numpy() == 0, ref_sse == 0)
        _near_tie_ok(ch.cpu().numpy(), ref_ch, ref_sse, cands)


def test_select_full_size(mxq, orc):
    """Workload 2: W 3072 x 3072 bf16 Student-t, candidates {INT4-g32, NVFP4, MXFP4}."""
    w = workloads.chameleon_selection()["w"]
    cands = [mxq.INT4_G32, mxq.NVFP4, mxq.MXFP4]
    ch, sse = mxq.select_weight_format(dev(w, "bf16"), cands)
    ref_ch, ref_sse = orc.select_weight_format(w, cands)
    np.testing.assert_allclose(sse.cpu().numpy(), ref_sse, rtol=1e-12, atol=0)
    assert _near_tie_ok(ch.cpu().numpy(), ref_ch, ref_sse, cands) <= 3


# ------------------------------------------------------------------ MSE-fitted NVFP4 scales

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("iters", [0, 1, 3])
def test_quantize_mse_small(mxq, orc, dtype, iters):
    rows, cols = 37, 512   # ragged rows (padded MMA scale tiles), 32 blocks per row
    x = nasty_matrix(300 + iters, rows, cols)
    xv = host_values(x, dtype)
    ref, ref_sse = orc.quantize_mse_nvfp4(xv, iters)
    for layout in (mxq.CANONICAL, mxq.MMA):
        q, sse = mxq.quantize_mse(dev(x, dtype), iters, layout)
        torch.cuda.synchronize()
        assert_qtensor_equal(q, ref, layout_mma=layout == mxq.MMA)
        assert sse.item() == ref_sse


def test_quantize_mse_edge_shapes(mxq, orc):
    for rows, cols in ((1, 16), (129, 16), (3, 1024 + 64), (300, 48)):
        x = nasty_matrix(11, rows, cols)
        ref, ref_sse = orc.quantize_mse_nvfp4(x, 2)
        for layout in (mxq.CANONICAL, mxq.MMA):
            q, sse = mxq.quantize_mse(dev(x, "f32"), 2, layout)
            torch.cuda.synchronize()
            assert_qtensor_equal(q, ref, layout_mma=layout == mxq.MMA)
            assert sse.item() == ref_sse
    q, sse = mxq.quantize_mse(torch.empty((0, 64), device="cuda"), 2)
    assert q.tensor_scale.item() == 1.0 and sse.item() == 0.0
    z = np.zeros((8, 128), np.float32)
    q, sse = mxq.quantize_mse(dev(z, "bf16"), 2)
    ref, _ = orc.quantize_mse_nvfp4(z, 2)
    assert_qtensor_equal(q, ref)
    assert sse.item() == 0.0


def test_quantize_mse_full_size(mxq, orc):
    """Workload 3's residual weight R (12288 x 3072 bf16), two rounds, MMA
    layout: sampled rows against the oracle's block step under the device's
    final tensor scale; run-to-run identity; the reported error against the
    dequantized result; lower error than the usual NVFP4 scales."""
    w = workloads.svdquant_mlp_up()["w"]
    n, k = w.shape
    wd = dev(w, "bf16")
    q, sse = mxq.quantize_mse(wd, 2, mxq.MMA)
    q2, sse2 = mxq.quantize_mse(wd, 2, mxq.MMA)
    torch.cuda.synchronize()
    assert torch.equal(q.codes, q2.codes) and torch.equal(q.scales, q2.scales)
    assert q.tensor_scale.item() == q2.tensor_scale.item() and sse.item() == sse2.item()
    s_t = q.tensor_scale.item()
    rows = np.sort(np.random.default_rng(37).choice(n, 48, replace=False))
    ref, _ = orc.mse_nvfp4_blocks(w[rows], s_t)
    codes = q.codes.cpu().numpy().reshape(n, k // 2)
    np.testing.assert_array_equal(codes[rows], ref.codes)
    canon, pad = byte_scales_from_mma(q.scales.cpu().numpy(), n, k // 16)
    np.testing.assert_array_equal(canon[rows], ref.scales)
    assert (pad == 0).all()
    wt = torch.from_numpy(w).cuda().double()
    err = ((mxq.dequantize(q, torch.float32).double() - wt) ** 2).sum().item()
    assert err == pytest.approx(sse.item(), rel=1e-5)
    u = mxq.quantize(wd, mxq.NVFP4)
    usual = ((mxq.dequantize(u, torch.float32).double() - wt) ** 2).sum().item()
    assert sse.item() < usual


# ------------------------------------------------------------------ MX fixed grid scale

GRID = [1.0, 1.0625, 1.125, 1.25, 4.0 / 3.0, 1.5, 1.75, 2.0]


@pytest.mark.parametrize("fmt", [1, 0])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("hadamard_b", [0, 32, 128])
def test_mx_grid_small(mxq, orc, fmt, dtype, hadamard_b):
    rows, cols = 37, 512
    x = nasty_matrix(400 + fmt, rows, cols)
    if hadamard_b:
        x = _moderate(x)
    xv = host_values(x, dtype)
    for g in (1.0, 1.125, 4.0 / 3.0, 2.0):
        ref = orc.quantize_mx_grid(xv, fmt, g, hadamard_b)
        for layout in (mxq.CANONICAL, mxq.MMA):
            q = mxq.quantize_mx_grid(dev(x, dtype), fmt, g, hadamard_b, layout)
            torch.cuda.synchronize()
            assert_qtensor_equal(q, ref, layout_mma=layout == mxq.MMA)
    best, sse = mxq.fit_mx_grid(dev(x, dtype), fmt, GRID, hadamard_b)
    ref_sse = orc.mx_grid_sse(xv, fmt, GRID, hadamard_b)
    np.testing.assert_array_equal(sse.cpu().numpy(), ref_sse)
    assert best == GRID[int(np.argmin(ref_sse))]


def test_mx_grid_fit_ragged_groups(mxq, orc):
    # 300 rows: three row groups, the last one ragged; 1 and 8 candidates
    x = nasty_matrix(12, 300, 96)
    for gs in ([1.125], GRID):
        _, sse = mxq.fit_mx_grid(dev(x, "f32"), mxq.MXFP4, gs, 32)
        np.testing.assert_array_equal(sse.cpu().numpy(), orc.mx_grid_sse(x, mxq.MXFP4, gs, 32))
    _, sse = mxq.fit_mx_grid(torch.empty((0, 64), device="cuda"), mxq.MXFP4, GRID[:2])
    assert sse.cpu().tolist() == [0.0, 0.0]


def test_mx_grid_full_size(mxq, orc):
    """Workload 4's weight W (4096 x 4096 bf16) after the 128-wide rotation:
    run-to-run identity, the g = 1 error against the usual quantizer's
    dequantized result, and a fitted grid scale at least as good as g = 1."""
    w = workloads.mxfp4_hadamard_gemm()["w"]
    wd = dev(w, "bf16")
    best, sse = mxq.fit_mx_grid(wd, mxq.MXFP4, GRID, 128)
    _, sse2 = mxq.fit_mx_grid(wd, mxq.MXFP4, GRID, 128)
    torch.cuda.synchronize()
    assert torch.equal(sse, sse2)
    h = mxq.hadamard_block(wd.float(), 128).double()
    deq = mxq.dequantize(mxq.quantize(wd, mxq.MXFP4, 128), torch.float32).double()
    assert sse[0].item() == pytest.approx(((h - deq) ** 2).sum().item(), rel=1e-9)
    assert sse.min().item() <= sse[0].item() and best == GRID[int(torch.argmin(sse).item())]
    q = mxq.quantize_mx_grid(wd, mxq.MXFP4, best, 128, mxq.MMA)
    u = mxq.quantize(wd, mxq.MXFP4, 128, mxq.MMA)
    assert torch.equal(q.codes, u.codes) == (best == 1.0)


# ------------------------------------------------------------------ activation-format calibration

CALIB = [5, 6, 0]   # INT8 per row, FP8 per tensor, MXFP8 (workload 5's palette)


def _pick_ok(gpu_entry, ref_sse, cands, forced=-1):
    if forced >= 0:
        return gpu_entry == forced
    s = np.sort(ref_sse)
    return gpu_entry == cands[int(np.argmin(ref_sse))] or s[1] - s[0] <= 1e-12 * s[0]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_calibrate_small(mxq, orc, dtype):
    rng = np.random.default_rng(61)
    xs = []
    for nu in (2.2, 20.0):
        x = rng.standard_t(nu, size=(300, 1152)).astype(np.float32)   # three row groups, the last ragged
        x[:, rng.choice(1152, 8, replace=False)] *= 60.0
        xs.append(host_values(x, dtype))
    sse = torch.zeros(3, dtype=torch.float64, device="cuda")
    mom = torch.zeros(2, dtype=torch.float64, device="cuda")
    ref_sse, ref_mom = np.zeros(3), np.zeros(2)
    for x in xs:
        mxq.calibrate_activation(dev(x, dtype), CALIB, sse, mom)
        orc.calibrate_activation(x, CALIB, ref_sse, ref_mom)
    torch.cuda.synchronize()
    np.testing.assert_allclose(sse.cpu().numpy(), ref_sse, rtol=1e-12)   # per-row order differs
    np.testing.assert_array_equal(mom.cpu().numpy(), ref_mom)            # same order: bit-exact
    entry = torch.zeros(1, dtype=torch.uint8, device="cuda")
    mxq.calibrate_pick(sse, CALIB, entry)
    assert _pick_ok(int(entry.item()), ref_sse, CALIB)
    mxq.calibrate_pick(sse, CALIB, entry, forced_fmt=mxq.MXFP8)
    assert entry.item() == mxq.MXFP8


def test_calibrate_table(mxq, orc):
    """A 3-layer x 4-interval table from seeded activations whose tails
    thin out along the trajectory; layer 2 forced to MXFP8; then routed."""
    n_layers, n_int, per = 3, 4, 2
    table = torch.zeros((n_layers, n_int), dtype=torch.uint8, device="cuda")
    ref = np.zeros((n_layers, n_int), np.uint8)
    for layer in range(n_layers):
        for it in range(n_int):
            sse = torch.zeros(3, dtype=torch.float64, device="cuda")
            mom = torch.zeros(2, dtype=torch.float64, device="cuda")
            ref_sse, ref_mom = np.zeros(3), np.zeros(2)
            for s in range(per):
                x = workloads.student_t(70 + layer, "calib.%d.%d" % (it, s), (256, 1152), 2.0 + 10.0 * it)
                if layer == 1:
                    x = x * workloads.dit_forced_column_factors(7, layer, 1152)[None, :]
                x = host_values(x, "bf16")
                mxq.calibrate_activation(dev(x, "bf16"), CALIB, sse, mom)
                orc.calibrate_activation(x, CALIB, ref_sse, ref_mom)
            forced = mxq.MXFP8 if layer == 2 else -1
            mxq.calibrate_pick(sse, CALIB, table[layer, it:it + 1], forced_fmt=forced)
            ref[layer, it] = orc.calibrate_pick(ref_sse, CALIB, forced)
            np.testing.assert_array_equal(mom.cpu().numpy(), ref_mom)
            assert _pick_ok(int(table[layer, it].item()), ref_sse, CALIB, forced)
    tab = table.cpu().numpy()
    assert (tab[2] == mxq.MXFP8).all()
    for layer in range(n_layers):
        for step in range(20):
            assert mxq.route(tab, layer, step, 20) == orc.route(tab, n_layers, n_int, layer, step, 20)


def test_calibrate_full_size(mxq, orc):
    """Workload 5's fc1 input at step 0 (8192 x 1152 bf16), the benchmark's call."""
    x = workloads.dit_activation(5, 0, 1152)
    sse = torch.zeros(3, dtype=torch.float64, device="cuda")
    mom = torch.zeros(2, dtype=torch.float64, device="cuda")
    mxq.calibrate_activation(dev(x, "bf16"), CALIB, sse, mom)
    ref_sse, ref_mom = np.zeros(3), np.zeros(2)
    orc.calibrate_activation(x, CALIB, ref_sse, ref_mom)
    torch.cuda.synchronize()
    np.testing.assert_allclose(sse.cpu().numpy(), ref_sse, rtol=1e-12)
    np.testing.assert_array_equal(mom.cpu().numpy(), ref_mom)


# ------------------------------------------------------------------ error path

def test_bounded_wait_reports_timeout(mxq, orc):
    """A bounded device wait that runs out is latched in the error word and
    reported by mxq_check (MXQ_ETIMEOUT = 4), which clears it; the context
    stays usable (no trap, fault or unbounded loop is involved)."""
    assert mxq.check() == 0
    assert mxq.lib().mxq_selftest_wait_timeout(20000, None) == 0   # 20 ms
    assert mxq.check() == 4
    assert mxq.check() == 0
    x = nasty_matrix(71, 37, 512)
    q = mxq.quantize(dev(x, "f32"), mxq.NVFP4)
    torch.cuda.synchronize()
    assert_qtensor_equal(q, orc.quantize(x, mxq.NVFP4))
    assert mxq.lib().mxq_selftest_wait_timeout(0, None) == 1        # bound outside 1 us .. 1 s
