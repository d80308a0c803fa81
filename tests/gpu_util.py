"""Helpers shared by the GPU parity tests: moving the seeded numpy inputs to
the device, comparing quantized tensors with the oracle's, and undoing the
MMA scale layout with the formula include/mxq.h documents."""
import numpy as np
import torch

import workloads


def dev(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.cuda()


def host_values(a: np.ndarray, dtype: str) -> np.ndarray:
    """The exact values the device sees for `a` stored as `dtype`."""
    return workloads.to_bf16_values(a) if dtype == "bf16" else np.ascontiguousarray(a, np.float32)


def nasty_matrix(seed: int, rows: int, cols: int) -> np.ndarray:
    """Small matrix mixing the cases the quantizers must get right: heavy
    tails, outlier columns, all-zero blocks, signed zeros, fp32 subnormals,
    values near fp32 max, and exact rounding midpoints of the E2M1/E4M3
    grids."""
    rng = np.random.default_rng(seed)
    x = (rng.standard_t(3, size=(rows, cols)) * np.exp(rng.uniform(-4, 4, size=(rows, 1)))).astype(np.float32)
    x[:, rng.choice(cols, max(1, cols // 50), replace=False)] *= 80.0
    if rows > 2:
        x[1, :] = 0.0
        x[1, 1::3] = -0.0
        x[2, :min(64, cols)] = (rng.standard_normal(min(64, cols)) * 1e-39).astype(np.float32)   # subnormal block
    if rows > 4:
        h = min(32, cols)
        x[3, :h] = np.float32(3e38) * rng.uniform(-1, 1, h).astype(np.float32)
        mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 1.0625, 1.1875, 17, 19, 6.5], np.float32)
        x[4, :] = rng.choice(mids, cols) * rng.choice([-1, 1], cols)
        x[4, ::16] = 6.0
    return x


def unpack4(codes: np.ndarray, rows: int) -> np.ndarray:
    c = codes.reshape(rows, -1)
    return np.stack([c & 0xF, c >> 4], -1).reshape(rows, -1)


def mma_offset(r, s, s_pad):
    r = np.asarray(r, np.int64)
    s = np.asarray(s, np.int64)
    return ((r // 128) * (s_pad // 4) + s // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + s % 4


def byte_scales_from_mma(buf: np.ndarray, rows: int, nscale: int):
    """(canonical rows x nscale array, padding bytes) of an MMA-layout byte-scale buffer."""
    s_pad = (nscale + 15) // 16 * 16
    r, s = np.meshgrid(np.arange(rows), np.arange(nscale), indexing="ij")
    off = mma_offset(r, s, s_pad)
    used = np.zeros(buf.size, bool)
    used[off.ravel()] = True
    return buf[off], buf[~used]


def assert_qtensor_equal(gq, oq, layout_mma=False):
    """Bit-exact comparison of a device QTensor with an oracle QTensor."""
    from microscaling_bit_quantization_b200 import INT4_G32, INT4_G64, MXFP4, MXFP8, NVFP4, FP8_TENSOR, INT8_ROW
    fmt, rows, cols = oq.fmt, oq.rows, oq.cols
    codes = gq.codes.cpu().numpy()
    if layout_mma and fmt in (INT4_G32, INT4_G64):
        # MMA layout: the E4M3 byte of each integer code (exact for |q| <= 7, zero as +0)
        q = unpack4(oq.codes, rows).astype(np.int32)
        q = np.where(q & 8, q - 16, q).astype(np.float32)
        want = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        want = np.where(q == 0, 0, want).astype(np.uint8)
        np.testing.assert_array_equal(codes.reshape(rows, cols), want)
    else:
        np.testing.assert_array_equal(codes.reshape(oq.codes.shape), oq.codes)
    if fmt in (MXFP8, MXFP4, NVFP4):
        sb = gq.scales.cpu().numpy()
        if layout_mma:
            canon, pad = byte_scales_from_mma(sb, rows, oq.scales.shape[1])
            np.testing.assert_array_equal(canon, oq.scales)
            assert (pad == 0).all()
        else:
            np.testing.assert_array_equal(sb.reshape(oq.scales.shape), oq.scales)
    elif fmt in (INT4_G32, INT4_G64):
        s = gq.scales.cpu().view(torch.float32).numpy()
        s = s.reshape(oq.scales.shape[1], rows).T if layout_mma else s.reshape(oq.scales.shape)
        np.testing.assert_array_equal(s.view(np.uint32), oq.scales.view(np.uint32))
    elif fmt == INT8_ROW:
        np.testing.assert_array_equal(gq.scales.cpu().view(torch.float32).numpy().view(np.uint32),
                                      oq.scales.view(np.uint32))
    if fmt in (NVFP4, FP8_TENSOR):
        assert np.float32(gq.tensor_scale.item()) == np.float32(oq.tensor_scale)


def gemm_close(y, ref, bf16_out=False):
    """Tolerance for fp32 output: relative Frobenius error <= 1e-4
    and max abs error <= 1e-4 * max|Y_ref|.  bf16 output additionally allows
    the final rounding to bf16: 2^-8 |Y_ref| per element (half a bf16 ulp is
    at most 2^-9 |Y|; the factor 2 covers the fp32 error under it)."""
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.abs(ref).max()
    err = np.abs(y - ref)
    if bf16_out:
        ok = err <= 1e-4 * scale + 2.0 ** -8 * np.abs(ref)
        assert ok.all(), "max excess %g" % (err - 1e-4 * scale - 2.0 ** -8 * np.abs(ref)).max()
    else:
        rel = np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-300)
        assert rel <= 1e-4, "relative Frobenius error %g" % rel
        assert err.max() <= 1e-4 * scale, "max abs error %g vs %g" % (err.max(), 1e-4 * scale)
