"""Pins of the CPU oracle against facts fixed outside it (CPU only).

Each test checks the oracle against something it does not compute itself:
hand-worked values from the published format definitions (tests/golden/),
closed forms, torch's independent fp8 / bf16 casts, scipy's Sylvester
Hadamard matrix, invariants, and brute force over every code.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_pairs(name):
    rows = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#")[0].strip()
        if line:
            a, b = line.split()
            rows.append((a, b))
    return rows


def _nan_eq(a, b):
    return (math.isnan(a) and math.isnan(b)) or (a == b and math.copysign(1, a) == math.copysign(1, b))


# ------------------------------------------------------------------ codec tables

def test_e2m1_table_closed_form(orc):
    mags = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    for c in range(16):
        v = orc.e2m1_value(c)
        assert abs(v) == mags[c & 7]
        assert math.copysign(1, v) == (-1 if c & 8 else 1)


def test_e4m3_golden_values(orc):
    for code, val in _read_pairs("e4m3_codes.txt"):
        assert _nan_eq(orc.e4m3_value(int(code, 16)), float(val)), code


def test_e4m3_table_against_torch(orc):
    # torch's float8_e4m3fn decode is an independent implementation of the same table.
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        assert _nan_eq(orc.e4m3_value(c), float(ref[c])), hex(c)


def test_e4m3_extremes(orc):
    finite = [orc.e4m3_value(c) for c in range(256) if not math.isnan(orc.e4m3_value(c))]
    assert len(finite) == 254
    assert max(finite) == 448.0 and min(finite) == -448.0
    assert min(v for v in finite if v > 0) == 2.0 ** -9


def test_e8m0_closed_form(orc):
    for b in range(255):
        assert orc.e8m0_value(b) == 2.0 ** (b - 127)
    assert math.isnan(orc.e8m0_value(255))


# ------------------------------------------------------------------ rounding

def test_e2m1_golden_rounding(orc):
    for v, code in _read_pairs("e2m1_rne.txt"):
        assert orc.to_e2m1(float(v)) == int(code, 16), v


def test_e4m3_golden_rounding(orc):
    for v, code in _read_pairs("e4m3_rne.txt"):
        assert orc.to_e4m3(float(v)) == int(code, 16), v


def test_every_code_round_trips(orc):
    for c in range(16):
        assert orc.to_e2m1(orc.e2m1_value(c)) == c
    for c in range(256):
        v = orc.e4m3_value(c)
        if not math.isnan(v):
            assert orc.to_e4m3(v) == c, hex(c)


def _brute_nearest(v, table):
    """Nearest code by exhaustive search; ties to the even code; no sign handling."""
    a = abs(v)
    best = None
    for c, m in enumerate(table):
        d = abs(a - m)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return best[1]


def test_e2m1_brute_force(orc):
    table = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    rng = np.random.default_rng(11)
    vals = np.concatenate([rng.uniform(-8, 8, 4000), np.arange(-700, 701) / 100.0]).astype(np.float32)
    for v in vals:
        v = float(v)
        c = _brute_nearest(min(abs(v), 6.0), table) | (8 if math.copysign(1, v) < 0 else 0)
        assert orc.to_e2m1(v) == c, v


def test_e4m3_against_torch_cast(orc):
    # torch's RNE fp32 -> float8_e4m3fn cast agrees with ours wherever it does
    # not overflow to NaN (|v| <= 464, the midpoint above 448).
    rng = np.random.default_rng(12)
    bits = rng.integers(0, 2 ** 32, size=20000, dtype=np.uint64).astype(np.uint32)
    hi = (np.arange(2 ** 16, dtype=np.uint32) << 16)
    vals = np.concatenate([bits, hi, hi | 0x8000, hi | 0x7FFF]).view(np.float32)
    vals = vals[np.isfinite(vals) & (np.abs(vals) <= 464.0)]
    ref = torch.from_numpy(vals.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([orc.to_e4m3(float(v)) for v in vals], np.uint8)
    assert np.array_equal(ours, ref)


def test_bulk_cast_range_against_torch(orc):
    # The bulk path used by the exhaustive GPU test, on contiguous bit-pattern
    # ranges: [2^-12, ...) upwards, and the negative range below -1.
    for first in (0x39800000, 0xBF800000, 0x43C00000):
        got = orc.cast_range(first, 1 << 20, "e4m3")
        v = (np.uint32(first) + np.arange(1 << 20, dtype=np.uint32)).view(np.float32)
        ok = np.abs(v) <= 464.0
        ref = torch.from_numpy(v.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(got[ok], ref[ok])
        assert (got[~ok] & 0x7F == 0x7E).all()
    got = orc.cast_range(0x3E000000, 1 << 16, "e2m1")
    v = (np.uint32(0x3E000000) + np.arange(1 << 16, dtype=np.uint32)).view(np.float32)
    assert all(got[i] == orc.to_e2m1(float(v[i])) for i in range(0, 1 << 16, 97))


def test_e4m3_saturates(orc):
    for v in (465.0, 480.0, 1e30, float("inf")):
        assert orc.to_e4m3(v) == 0x7E
        assert orc.to_e4m3(-v) == 0xFE
    assert orc.to_e4m3(float("nan")) == 0x7F


def test_round_bf16_against_torch(orc):
    rng = np.random.default_rng(13)
    x = np.concatenate([rng.standard_normal(20000) * 10 ** rng.uniform(-30, 30, 20000),
                        (np.arange(1, 4000) * (1 + 2 ** -8))]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    got = orc.round_bf16_array(x)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


# ------------------------------------------------------------------ quantizers

def _blocks():
    return json.load(open(os.path.join(GOLDEN, "quant_blocks.json")))


def _unpack4(codes):
    lo, hi = codes & 0xF, codes >> 4
    return np.stack([lo, hi], -1).reshape(codes.shape[0], -1)


def test_mxfp4_golden_block(orc):
    for key in ("mxfp4", "mxfp4_saturating"):
        g = _blocks()[key]
        x = np.zeros((1, 32), np.float32)
        x[0, :len(g["x_head"])] = g["x_head"]
        q = orc.quantize(x, orc.MXFP4)
        assert q.scales[0, 0] == g["scale_byte"]
        codes = _unpack4(q.codes)[0]
        assert list(codes[:len(g["codes_head"])]) == g["codes_head"]
        assert (codes[len(g["codes_head"]):] == 0).all()


def test_nvfp4_golden_blocks(orc):
    g = _blocks()["nvfp4"]
    x = np.zeros((1, 32), np.float32)
    x[0, :4] = g["x_head_block0"]
    x[0, 16:19] = g["x_head_block1"]
    q = orc.quantize(x, orc.NVFP4)
    assert q.tensor_scale == g["tensor_scale"]
    assert list(q.scales[0]) == g["scale_bytes"]
    codes = _unpack4(q.codes)[0]
    assert list(codes[:4]) == g["codes_head_block0"]
    assert list(codes[16:19]) == g["codes_head_block1"]


def test_int4_golden_group(orc):
    g = _blocks()["int4_g32"]
    x = np.zeros((1, 32), np.float32)
    x[0, :5] = g["x_head"]
    q = orc.quantize(x, orc.INT4_G32)
    assert q.scales[0, 0] == np.float32(g["scale"])
    assert list(_unpack4(q.codes)[0][:5]) == g["codes_head"]


def test_mx_scale_rule_closed_form(orc):
    # OCP MX: X = 2^(floor(log2 amax) - emax_elem); check the scale byte for
    # amax spanning many binades (incl. subnormal fp32) and the clamp at -127.
    for emax, fmt in ((8, orc.MXFP8), (2, orc.MXFP4)):
        for p in list(range(-149, 128, 7)) + [-149, -126, 127]:
            for frac in (1.0, 1.5, 1.9999):
                amax = np.float32(frac * 2.0 ** p)
                if not np.isfinite(amax) or amax == 0:
                    continue
                x = np.zeros((1, 32), np.float32)
                x[0, 3] = amax
                q = orc.quantize(x, fmt)
                e = max(-127, min(127, math.floor(math.log2(float(amax))) - emax))
                assert q.scales[0, 0] == e + 127, (fmt, amax)


def test_all_zero_blocks(orc):
    x = np.zeros((2, 64), np.float32)
    for fmt in range(7):
        q = orc.quantize(x, fmt)
        assert (q.codes == 0).all(), fmt
        if fmt in (orc.MXFP8, orc.MXFP4):
            assert (q.scales == 127).all()
        if fmt in (orc.NVFP4, orc.FP8_TENSOR):
            assert q.tensor_scale == 1.0
        assert (q.dequantize() == 0).all()


def test_representable_blocks_are_lossless(orc):
    rng = np.random.default_rng(14)
    # MXFP4: E2M1 grid values times one power of two per block, each block containing 6*2^e.
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    x = rng.choice(grid, size=(8, 64)) * rng.choice([-1, 1], size=(8, 64))
    x[:, 0] = 6
    x[:, 32] = -6
    x = (x * (2.0 ** rng.integers(-20, 20, size=(8, 1)))).astype(np.float32)
    assert np.array_equal(orc.quantize(x, orc.MXFP4).dequantize(), x.astype(np.float64))
    # MXFP8: E4M3 values times a power of two.
    e4 = np.array([orc.e4m3_value(c) for c in range(127)], np.float32)
    x = rng.choice(e4, size=(8, 64)) * rng.choice([-1, 1], size=(8, 64))
    x[:, 1] = 448
    x[:, 40] = 448
    x = (x * (2.0 ** rng.integers(-10, 10, size=(8, 1)))).astype(np.float32)
    assert np.array_equal(orc.quantize(x, orc.MXFP8).dequantize(), x.astype(np.float64))
    # INT4: integers in [-7,7] times s with 7*s exactly representable.
    q = rng.integers(-7, 8, size=(4, 64)).astype(np.float32)
    q[:, 0] = 7
    q[:, 32] = -7
    x = (q * np.float32(0.25)).astype(np.float32)
    assert np.array_equal(orc.quantize(x, orc.INT4_G32).dequantize(), x.astype(np.float64))


def _nearest_grid_error(v, grid_vals):
    return np.min(np.abs(v[..., None] - grid_vals[None, :]), axis=-1)


def test_mx_elements_are_nearest_grid_points(orc):
    # Brute force: each MX element's dequantized value is a nearest point of
    # the block's scaled grid (within saturation).
    rng = np.random.default_rng(15)
    x = (rng.standard_t(3, size=(16, 128)) * 10.0 ** rng.uniform(-3, 3, size=(16, 1))).astype(np.float32)
    for fmt, mags in ((orc.MXFP4, [orc.e2m1_value(c) for c in range(8)]),
                      (orc.MXFP8, [orc.e4m3_value(c) for c in range(127)])):
        q = orc.quantize(x, fmt)
        d = q.dequantize()
        for r in range(x.shape[0]):
            for b in range(x.shape[1] // 32):
                X = orc.e8m0_value(int(q.scales[r, b]))
                grid = np.array(sorted(set([m * X for m in mags] + [-m * X for m in mags])))
                v = x[r, b * 32:(b + 1) * 32].astype(np.float64)
                err = np.abs(v - d[r, b * 32:(b + 1) * 32])
                np.testing.assert_array_equal(err, _nearest_grid_error(v, grid))


def test_nvfp4_error_bound_and_scale_range(orc):
    rng = np.random.default_rng(16)
    x = (rng.standard_normal((32, 256)) * np.exp(rng.uniform(-3, 3, (32, 1)))).astype(np.float32)
    q = orc.quantize(x, orc.NVFP4)
    amax_t = float(np.abs(x).max())
    assert q.tensor_scale == np.float32(np.float32(amax_t) / np.float32(2688.0))
    d = q.dequantize()
    e4 = np.array([[orc.e4m3_value(int(b)) for b in row] for row in q.scales])
    assert (e4 >= 0).all() and (e4 <= 448).all()
    # within each block the error is at most half the largest grid gap (2 units of d)
    # plus the saturation excess; d ~ amax_b / 6 up to E4M3 rounding (< 1/16 relative).
    blk = x.reshape(32, 16, 16).astype(np.float64)
    dd = (e4 * q.tensor_scale)[..., None]
    assert (np.abs(blk - d.reshape(32, 16, 16)) <= 1.0 * dd + np.maximum(np.abs(blk) - 6 * dd, 0) + 1e-30).all()


def test_quantize_dequantize_idempotent(orc):
    rng = np.random.default_rng(17)
    x = (rng.standard_t(3, size=(16, 256)) * 0.7).astype(np.float32)
    for fmt in (orc.MXFP8, orc.MXFP4, orc.INT4_G32, orc.INT4_G64, orc.INT8_ROW, orc.NVFP4, orc.FP8_TENSOR):
        q1 = orc.quantize(x, fmt)
        q2 = orc.quantize(orc.dequantize_f32(q1), fmt)
        assert np.array_equal(q1.codes, q2.codes), fmt
        if fmt in (orc.MXFP8, orc.MXFP4):
            assert np.array_equal(q1.scales, q2.scales)


def test_int8_row_and_fp8_tensor_closed_forms(orc):
    rng = np.random.default_rng(18)
    x = rng.standard_normal((8, 96)).astype(np.float32)
    q = orc.quantize(x, orc.INT8_ROW)
    s = (np.abs(x).max(1) / np.float32(127)).astype(np.float32)
    assert np.array_equal(q.scales, s)
    codes = q.codes.view(np.int8).astype(np.int32)
    t = (x / s[:, None]).astype(np.float32)
    assert np.array_equal(codes, np.clip(np.rint(t), -127, 127).astype(np.int32))  # rint = RNE
    q = orc.quantize(x, orc.FP8_TENSOR)
    s = np.float32(np.abs(x).max()) / np.float32(448)
    assert q.tensor_scale == np.float32(s)
    ref = torch.from_numpy((x / np.float32(s)).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q.codes, ref)


def test_int4_codes_match_rint(orc):
    rng = np.random.default_rng(19)
    x = rng.standard_normal((8, 128)).astype(np.float32)
    for fmt, g in ((orc.INT4_G32, 32), (orc.INT4_G64, 64)):
        q = orc.quantize(x, fmt)
        s = (np.abs(x.reshape(8, -1, g)).max(-1) / np.float32(7)).astype(np.float32)
        assert np.array_equal(q.scales, s)
        t = (x.reshape(8, -1, g) / s[..., None]).astype(np.float32)
        ref = np.clip(np.rint(t), -7, 7).astype(np.int64).reshape(8, -1) & 0xF
        assert np.array_equal(_unpack4(q.codes), ref)


def test_nonfinite_input_rejected(orc):
    x = np.zeros((1, 32), np.float32)
    x[0, 5] = np.inf
    with pytest.raises(orc.OracleError):
        orc.quantize(x, orc.MXFP8)


# ------------------------------------------------------------------ Hadamard

def test_hadamard_norm_constants(orc):
    inv_sqrt2 = np.array([0x3F3504F3], np.uint32).view(np.float32)[0]   # RN_f32(1/sqrt 2)
    for lg in range(1, 9):
        b = 1 << lg
        want = np.float32(2.0 ** -(lg // 2)) * (inv_sqrt2 if lg & 1 else np.float32(1))
        assert np.float32(orc.hadamard_norm(b)) == want, b
    # and it is the correctly rounded value of 1/sqrt(b)
    for lg in range(1, 9):
        b = 1 << lg
        ref = np.float32(1.0 / math.sqrt(b))
        assert abs(float(np.float32(orc.hadamard_norm(b))) - 1 / math.sqrt(b)) <= abs(float(ref) - 1 / math.sqrt(b))


def test_hadamard_matches_sylvester_matrix(orc):
    import scipy.linalg
    rng = np.random.default_rng(20)
    for b in (2, 4, 16, 128, 256):
        x = rng.standard_normal((5, 2 * b)).astype(np.float32)
        H = scipy.linalg.hadamard(b).astype(np.float64) / math.sqrt(b)
        ref = np.concatenate([x[:, :b].astype(np.float64) @ H, x[:, b:].astype(np.float64) @ H], 1)
        got = orc.hadamard(x, b).astype(np.float64)
        tol = (math.log2(b) + 2) * 2 ** -23 * np.abs(x).sum(1, keepdims=True)
        assert (np.abs(got - ref) <= tol).all(), b


def test_hadamard_b2_exact_and_orthogonal(orc):
    x = np.array([[3.0, 1.0, -2.5, 0.5]], np.float32)
    n = np.float32(orc.hadamard_norm(2))
    want = np.array([[(3 + 1) * n, (3 - 1) * n, (-2.5 + 0.5) * n, (-2.5 - 0.5) * n]], np.float32)
    assert np.array_equal(orc.hadamard(x, 2), want)
    for b in (4, 32, 128):
        y = orc.hadamard(np.eye(b, dtype=np.float32), b).astype(np.float64)
        np.testing.assert_allclose(y @ y.T, np.eye(b), atol=1e-6)


def test_hadamard_preserves_gemm(orc):
    rng = np.random.default_rng(21)
    x = rng.standard_normal((6, 256)).astype(np.float32)
    w = rng.standard_normal((5, 256)).astype(np.float32)
    y = orc.hadamard(x, 128).astype(np.float64) @ orc.hadamard(w, 128).astype(np.float64).T
    np.testing.assert_allclose(y, x.astype(np.float64) @ w.astype(np.float64).T, rtol=0, atol=1e-4)


def test_hadamard_lowers_error_on_heavy_tails(orc):
    # Qualitative claim of "Bridging the Gap ...", item 3 (not a parity pin).
    rng = np.random.default_rng(22)
    x = rng.laplace(0, 1, (64, 1024)).astype(np.float32)
    x[:, rng.choice(1024, 8, replace=False)] *= 30
    plain = orc.quantize(x, orc.MXFP4).dequantize()
    err_plain = ((plain - x) ** 2).sum()
    xr = orc.hadamard(x, 128)
    rot = orc.quantize(x, orc.MXFP4, hadamard_b=128).dequantize()
    err_rot = ((rot - xr) ** 2).sum()
    assert err_rot < err_plain


# ------------------------------------------------------------------ selection

def test_selection_constructed_rows(orc):
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    rng = np.random.default_rng(23)
    k = 64
    w = np.zeros((4, k), np.float32)
    # row 0: carries the tensor max 2688 -> s_t = 1; the E2M1 grid x 448 in every block
    w[0] = rng.choice(grid, k) * 448
    w[0, ::16] = 2688
    # row 1: E2M1 grid values with 6 in every 16-block: NVFP4 and MXFP4 both exact
    w[1] = rng.choice(grid, k) * rng.choice([-1, 1], k)
    w[1, ::16] = 6
    # row 2: the same grid scaled by 2^-20: NVFP4 block scale underflows, MXFP4 exact
    w[2] = w[1] * np.float32(2.0 ** -20)
    # row 3: integers times 1/4 with +-7 in every 32-group: INT4 exact
    w[3] = rng.integers(-7, 8, k) * np.float32(0.25)
    w[3, 0], w[3, 32] = 1.75, -1.75
    INT4, NV, MX = orc.INT4_G32, orc.NVFP4, orc.MXFP4
    choice, sse = orc.select_weight_format(w, [INT4, NV, MX])
    assert sse[1, 1] == 0 and sse[1, 2] == 0 and choice[1] == NV      # tie -> lower index
    assert sse[2, 2] == 0 and sse[2, 1] > 0 and choice[2] == MX
    assert sse[3, 0] == 0 and choice[3] == INT4
    choice2, _ = orc.select_weight_format(w, [INT4, MX, NV])
    assert choice2[1] == MX


def test_selection_minimality_recomputed(orc):
    rng = np.random.default_rng(24)
    w = (rng.standard_t(4, size=(48, 256)) * 0.0141).astype(np.float32)
    cands = [orc.INT4_G32, orc.NVFP4, orc.MXFP4, orc.MXFP8, orc.INT8_ROW]
    choice, sse = orc.select_weight_format(w, cands)
    # independent recomputation of each error from quantize + dequantize
    ref = np.stack([((orc.quantize(w, f).dequantize() - w.astype(np.float64)) ** 2).sum(1) for f in cands], 1)
    np.testing.assert_allclose(sse, ref, rtol=1e-12, atol=0)
    for r in range(w.shape[0]):
        assert sse[r, cands.index(choice[r])] == sse[r].min()
        assert cands.index(choice[r]) == int(np.argmin(sse[r]))


def test_fp_grid_wins_on_heavy_tails(orc):
    # Qualitative claim ("Bridging the Gap ...": FP grids suit heavy tails,
    # INT grids suit uniform data) -- a sanity check, not parity.
    rng = np.random.default_rng(25)
    heavy = (rng.standard_t(2, size=(64, 256))).astype(np.float32)
    flat = rng.uniform(-1, 1, size=(64, 256)).astype(np.float32)
    c_heavy, _ = orc.select_weight_format(heavy, [orc.INT4_G32, orc.MXFP4])
    c_flat, _ = orc.select_weight_format(flat, [orc.INT4_G32, orc.MXFP4])
    assert (c_heavy == orc.MXFP4).mean() > (c_flat == orc.MXFP4).mean()


# ------------------------------------------------------------------ MSE-fitted NVFP4 scales

_E2M1_GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _e2m1_nearest(t: float) -> float:
    """E2M1 value nearest to t (ties to the even grid index), saturating at 6;
    written here from the grid, independently of the oracle's rounding."""
    a = abs(t)
    best = 0
    for i, g in enumerate(_E2M1_GRID):
        da, db = abs(a - g), abs(a - _E2M1_GRID[best])
        if da < db or (da == db and i % 2 == 0 and best % 2 == 1):
            best = i
    return math.copysign(_E2M1_GRID[best], t)


def _block_values_under(orc, v, e, s_t):
    """Decoded element values of block v coded under block code e: the
    quotient RN32(v / RN32(value(e) s_t)) by torch's IEEE fp32 division."""
    if e == 0:
        return [0.0] * len(v)
    d = torch.tensor(orc.e4m3_value(e), dtype=torch.float32) * torch.tensor(s_t, dtype=torch.float32)
    t = torch.tensor(v, dtype=torch.float32) / d
    return [_e2m1_nearest(float(z)) for z in t]


def _exact_block_error(v, vals, e_value, s_t):
    from fractions import Fraction
    s = Fraction(s_t) * Fraction(e_value)
    return sum((Fraction(float(a)) - Fraction(b) * s) ** 2 for a, b in zip(v, vals))


def _window(e0):
    if e0 == 0:
        return [0, 1]
    return [e0] + ([e0 + 1] if e0 + 1 <= 126 else []) + [e0 - j for j in range(1, 7) if e0 - j >= 1]


def test_mse_nvfp4_block_choice_brute_force(orc):
    # every block's chosen code has the least exact (rational) error over its
    # candidate window, the first one in scoring order on exact ties, and its
    # element codes are those the scale gives
    rng = np.random.default_rng(31)
    x = (rng.standard_t(3, size=(6, 64)) * 0.02).astype(np.float32)
    q_usual = orc.quantize(x, orc.NVFP4)
    q, _ = orc.quantize_mse_nvfp4(x, 0)
    assert q.tensor_scale == q_usual.tensor_scale
    s_t = q.tensor_scale
    deq = q.dequantize()
    for r in range(x.shape[0]):
        for b in range(x.shape[1] // 16):
            v = [float(z) for z in x[r, 16 * b:16 * b + 16]]
            e0 = int(q_usual.scales[r, b])
            errs = []
            for e in _window(e0):
                vals = _block_values_under(orc, v, e, s_t)
                errs.append((_exact_block_error(v, vals, orc.e4m3_value(e) if e else 0.0, s_t), e, vals))
            best = min(t[0] for t in errs)
            first = next(t for t in errs if t[0] == best)
            chosen = int(q.scales[r, b])
            err_chosen = next(t[0] for t in errs if t[1] == chosen)
            # binary64 scoring may only differ from exact rationals at rounding level
            assert float(err_chosen) <= float(best) * (1 + 1e-12)
            if chosen != first[1]:
                assert float(err_chosen - best) <= float(best) * 1e-12
            vals = next(t[2] for t in errs if t[1] == chosen)
            e_val = orc.e4m3_value(chosen) if chosen else 0.0
            assert list(deq[r, 16 * b:16 * b + 16]) == [a * e_val * s_t for a in vals]


def test_mse_nvfp4_never_worse_per_block(orc):
    rng = np.random.default_rng(32)
    x = (rng.standard_t(2.5, size=(16, 128)) * 0.05).astype(np.float32)
    xd = x.astype(np.float64)
    e_usual = ((orc.quantize(x, orc.NVFP4).dequantize() - xd) ** 2).reshape(16, 8, 16).sum(-1)
    q, sse = orc.quantize_mse_nvfp4(x, 0)
    e_mse = ((q.dequantize() - xd) ** 2).reshape(16, 8, 16).sum(-1)
    assert np.all(e_mse <= e_usual * (1 + 1e-12))
    assert e_mse.sum() < e_usual.sum()
    assert sse == pytest.approx(e_mse.sum(), rel=1e-12)


def test_mse_nvfp4_tensor_step_is_least_squares(orc):
    # one round = block step under the usual s_t (exactly the iters=0 result),
    # then s_t = RN32 of the least-squares factor sum(v u) / sum(u^2) for those
    # codes; recomputed here in exact rationals
    from fractions import Fraction
    rng = np.random.default_rng(33)
    x = (rng.standard_t(3, size=(8, 96)) * 0.03).astype(np.float32)
    q0, _ = orc.quantize_mse_nvfp4(x, 0)
    codes = _unpack4(q0.codes)
    num = den = Fraction(0)
    for r in range(x.shape[0]):
        for c in range(x.shape[1]):
            u = Fraction(orc.e2m1_value(int(codes[r, c]))) * Fraction(orc.e4m3_value(int(q0.scales[r, c // 16])))
            num += Fraction(float(x[r, c])) * u
            den += u * u
    exact = float(np.float32(num / den))   # RN to fp32 via the nearest binary64 first
    q1, _ = orc.quantize_mse_nvfp4(x, 1)
    assert abs(q1.tensor_scale - exact) <= np.spacing(np.float32(exact))
    assert q1.tensor_scale != q0.tensor_scale


def test_mse_nvfp4_power_of_two_equivariance(orc):
    rng = np.random.default_rng(34)
    x = (rng.standard_t(3, size=(8, 64)) * 0.02).astype(np.float32)
    for iters in (0, 2):
        q, sse = orc.quantize_mse_nvfp4(x, iters)
        for j in (6, -5):
            xs = (x * np.float32(2.0 ** j)).astype(np.float32)
            qs, sses = orc.quantize_mse_nvfp4(xs, iters)
            assert np.array_equal(qs.codes, q.codes) and np.array_equal(qs.scales, q.scales)
            assert qs.tensor_scale == q.tensor_scale * 2.0 ** j
            assert sses == sse * 4.0 ** j


def test_mse_nvfp4_degenerate_cases(orc):
    z = np.zeros((3, 32), np.float32)
    q, sse = orc.quantize_mse_nvfp4(z, 2)
    assert q.tensor_scale == 1.0 and sse == 0.0
    assert not q.codes.any() and not q.scales.any()
    # E2M1 grid values with 6 and the tensor max 2688 in every block: the
    # usual code reproduces them exactly, is scored first and kept
    grid = np.array(_E2M1_GRID, np.float32)
    rng = np.random.default_rng(35)
    w = (rng.choice(grid, (2, 64)) * 448).astype(np.float32)
    w[:, ::16] = 2688
    q, sse = orc.quantize_mse_nvfp4(w, 0)
    u = orc.quantize(w, orc.NVFP4)
    assert sse == 0.0 and np.array_equal(q.codes, u.codes) and np.array_equal(q.scales, u.scales)


def test_mse_nvfp4_rounds_lower_the_error(orc):
    # the page's claim for NVFP4 without rotations, on heavy-tailed weights:
    # a sanity check, not parity
    rng = np.random.default_rng(36)
    w = (rng.standard_t(4, size=(64, 256)) * 0.0141).astype(np.float32)
    usual = ((orc.quantize(w, orc.NVFP4).dequantize() - w.astype(np.float64)) ** 2).sum()
    errs = [orc.quantize_mse_nvfp4(w, it)[1] for it in (0, 1, 3)]
    assert errs[0] < usual and errs[2] <= errs[0]


# ------------------------------------------------------------------ MX fixed grid scale

@pytest.mark.parametrize("fmt_name", ["MXFP4", "MXFP8"])
@pytest.mark.parametrize("hadamard_b", [0, 128])
def test_mx_grid_one_is_the_ocp_rule(orc, fmt_name, hadamard_b):
    fmt = getattr(orc, fmt_name)
    rng = np.random.default_rng(41)
    x = (rng.standard_t(3, size=(12, 256)) * 0.03).astype(np.float32)
    q = orc.quantize_mx_grid(x, fmt, 1.0, hadamard_b)
    u = orc.quantize(x, fmt, hadamard_b)
    assert np.array_equal(q.codes, u.codes) and np.array_equal(q.scales, u.scales)


def test_mx_grid_exponent_closed_form(orc):
    # one nonzero element per 32-block with significand m and exponent k:
    # e = k + [g m >= 2] - 2 (E2M1's largest exponent), scale byte e + 127
    ms = [1.0, 1.25, 1.4999999, 1.5, 1.75, 1.9999999]
    ks = [-3, 0, 5]
    x = np.zeros((len(ks), 32 * len(ms)), np.float32)
    for i, k in enumerate(ks):
        for j, m in enumerate(ms):
            x[i, 32 * j + 7] = np.float32(m) * np.float32(2.0 ** k)
    for g in (1.0, 4.0 / 3.0, 1.125, 2.0):
        q = orc.quantize_mx_grid(x, orc.MXFP4, g)
        for i, k in enumerate(ks):
            for j, m in enumerate(ms):
                raise_ = float(np.float32(g)) * float(np.float32(m)) >= 2.0
                assert q.scales[i, j] == k + int(raise_) - 2 + 127


def test_mx_grid_four_thirds_never_clips(orc):
    # g = 4/3: the scale is the least power of two with amax / 2^e < 6
    rng = np.random.default_rng(42)
    x = (rng.standard_t(2, size=(16, 512)) * 0.05).astype(np.float32)
    q = orc.quantize_mx_grid(x, orc.MXFP4, 4.0 / 3.0)
    amax = np.abs(x.astype(np.float64)).reshape(16, 16, 32).max(-1)
    e = q.scales.astype(np.int64) - 127
    assert np.all(amax / 2.0 ** e < 6) and np.all(amax / 2.0 ** (e - 1) >= 6)


def test_mx_grid_sse_recomputed(orc):
    rng = np.random.default_rng(43)
    x = (rng.standard_t(4, size=(140, 256)) * 0.02).astype(np.float32)   # two 128-row groups
    gs = [1.0, 1.125, 1.25, 1.5, 2.0]
    for fmt, had in ((orc.MXFP4, 128), (orc.MXFP4, 0), (orc.MXFP8, 32)):
        sse = orc.mx_grid_sse(x, fmt, gs, had)
        h = orc.hadamard(x, had).astype(np.float64) if had else x.astype(np.float64)
        for j, g in enumerate(gs):
            deq = orc.quantize_mx_grid(x, fmt, g, had).dequantize()
            assert sse[j] == pytest.approx(((h - deq) ** 2).sum(), rel=1e-12)


def test_mx_grid_power_of_two_equivariance(orc):
    rng = np.random.default_rng(44)
    x = (rng.standard_t(3, size=(8, 128)) * 0.02).astype(np.float32)
    gs = [1.0, 1.125, 4.0 / 3.0]
    base = orc.mx_grid_sse(x, orc.MXFP4, gs, 32)
    q = orc.quantize_mx_grid(x, orc.MXFP4, 1.125, 32)
    for j in (4, -6):
        xs = (x * np.float32(2.0 ** j)).astype(np.float32)
        assert np.array_equal(orc.mx_grid_sse(xs, orc.MXFP4, gs, 32), base * 4.0 ** j)
        qs = orc.quantize_mx_grid(xs, orc.MXFP4, 1.125, 32)
        assert np.array_equal(qs.codes, q.codes)
        assert np.array_equal(qs.scales.astype(np.int64), q.scales.astype(np.int64) + j)


def test_mx_grid_fit_beats_ocp_after_rotation(orc):
    # the page's claim (one fixed grid scale for rotated MXFP4) on heavy-tailed
    # weights: some g > 1 lowers the error below the OCP rule -- a sanity check
    rng = np.random.default_rng(45)
    w = (rng.standard_t(4, size=(64, 512)) * 0.02).astype(np.float32)
    sse = orc.mx_grid_sse(w, orc.MXFP4, [1.0, 1.0625, 1.125, 1.1875, 1.25], 128)
    assert sse[1:].min() < sse[0]


# ------------------------------------------------------------------ activation-format calibration

def test_calibration_errors_are_selection_row_sums(orc):
    rng = np.random.default_rng(51)
    cands = [orc.INT8_ROW, orc.FP8_TENSOR, orc.MXFP8]
    xs = [(rng.standard_t(nu, size=(150, 128))).astype(np.float32) for nu in (2.5, 30.0)]
    sse = np.zeros(3)
    mom = np.zeros(2)
    totals = []
    for x in xs:
        _, rows = orc.select_weight_format(x, cands)
        totals.append(rows.sum(0))
        before = sse.copy()
        orc.calibrate_activation(x, cands, sse, mom)
        np.testing.assert_allclose(sse - before, totals[-1], rtol=1e-12)
    np.testing.assert_allclose(sse, totals[0] + totals[1], rtol=1e-12)


def test_calibration_moments_exact(orc):
    # dyadic values k/4 (|k| <= 40): every partial sum is exact, so the
    # accumulated moments equal the integer sums
    rng = np.random.default_rng(52)
    k = rng.integers(-40, 41, size=(260, 64))
    x = (k / 4.0).astype(np.float32)
    mom = np.zeros(2)
    orc.calibrate_activation(x, [orc.MXFP8], np.zeros(1), mom)
    k2 = int((k.astype(object) ** 2).sum())
    k4 = int((k.astype(object) ** 4).sum())
    assert mom[0] == k2 / 16.0 and mom[1] == k4 / 256.0


def test_calibration_pick_is_least_recomputed_error(orc):
    # heavy tails vs near-Gaussian activations: the entry is the candidate
    # whose quantize/dequantize error is least (recomputed independently)
    rng = np.random.default_rng(53)
    cands = [orc.INT8_ROW, orc.FP8_TENSOR, orc.MXFP8, orc.MXFP4]
    for nu in (1.5, 3.0, 50.0):
        x = rng.standard_t(nu, size=(96, 256)).astype(np.float32)
        x[:, :4] *= 40.0   # outlier channels
        sse = np.zeros(len(cands))
        orc.calibrate_activation(x, cands, sse, np.zeros(2))
        ref = [((orc.quantize(x, f).dequantize() - x.astype(np.float64)) ** 2).sum() for f in cands]
        assert orc.calibrate_pick(sse, cands) == cands[int(np.argmin(ref))]
        assert orc.calibrate_pick(sse, cands, orc.MXFP8) == orc.MXFP8


# ------------------------------------------------------------------ W4A16

def test_w4a16_weights_against_torch(orc):
    # every INT4 code against many scales: bf16(RN32(q s)) by torch's own
    # fp32 multiply and bf16 cast
    rng = np.random.default_rng(81)
    k, g = 64, 32
    q = np.tile(np.arange(-7, 8), 30)[: 7 * k].reshape(7, k)
    s = (np.exp(rng.uniform(-30, 30, size=(7, k // g))) * rng.choice([1, 1.0 + 2 ** -20], (7, k // g))).astype(np.float32)
    s[0, 0] = np.float32(1.0 / 3.0)
    nib = (q & 0xF).astype(np.uint8)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    wq = orc.QTensor(orc.INT4_G32, 7, k, codes, s, 0.0)
    w = orc.w4a16_weights(wq)
    ref = (torch.from_numpy(q.astype(np.float32)) * torch.from_numpy(np.repeat(s, g, axis=1))).to(torch.bfloat16)
    assert np.array_equal(w.view(np.uint32), ref.float().numpy().view(np.uint32))


def test_w4a16_brute_force_tiny(orc):
    rng = np.random.default_rng(82)
    x = rng.standard_normal((3, 128)).astype(np.float32)
    w = (rng.standard_normal((5, 128)) * 0.05).astype(np.float32)
    for fmt in (orc.INT4_G32, orc.INT4_G64):
        wq = orc.quantize(w, fmt)
        y = orc.w4a16(x, wq)
        w16 = orc.w4a16_weights(wq)
        for i in range(3):
            for j in range(5):
                acc = math.fsum(float(orc.round_bf16(float(x[i, c]))) * float(w16[j, c]) for c in range(128))
                assert y[i, j] == pytest.approx(acc, rel=1e-14, abs=1e-300)
        # the bf16 weights stay within half a bf16 ulp (plus the fp32 step) of the exact dequantization
        exact = wq.dequantize()
        assert np.all(np.abs(w16 - exact) <= np.abs(exact) * (2.0 ** -8 + 2.0 ** -24) + 1e-45)   # 8-bit significand


# ------------------------------------------------------------------ low rank + GEMM

def test_lowrank_down_brute_force(orc):
    rng = np.random.default_rng(26)
    x = (rng.standard_normal((3, 40)) * 3).astype(np.float32)
    l1 = torch.from_numpy(rng.standard_normal((40, 5)).astype(np.float32)).to(torch.bfloat16).float().numpy()
    t = orc.lowrank_down(x, l1)
    xb = torch.from_numpy(x).to(torch.bfloat16).double().numpy()   # torch's independent bf16 rounding
    for i in range(3):
        for j in range(5):
            ref = math.fsum(float(xb[i, k]) * float(l1[k, j]) for k in range(40))
            assert abs(t[i, j] - ref) <= 1e-12 * max(1.0, abs(ref))


def test_qlinear_brute_force_tiny(orc):
    rng = np.random.default_rng(27)
    x = rng.standard_normal((4, 64)).astype(np.float32)
    w = (rng.standard_normal((3, 64)) * 0.02).astype(np.float32)
    l1 = rng.standard_normal((64, 2)).astype(np.float32)
    l2 = rng.standard_normal((2, 3)).astype(np.float32)
    for fmt in range(7):
        xq, wq = orc.quantize(x, fmt), orc.quantize(w, fmt)
        t = orc.lowrank_down(x, l1)
        y = orc.qlinear(xq, wq, t, l2)
        xd, wd = xq.dequantize(), wq.dequantize()
        for i in range(4):
            for j in range(3):
                ref = math.fsum(xd[i, k] * wd[j, k] for k in range(64)) + math.fsum(t[i, r] * l2[r, j] for r in range(2))
                assert abs(y[i, j] - ref) <= 1e-12 * (1 + abs(ref))
        # row sampling gives the same rows
        ys = orc.qlinear(xq, wq, t[[1, 3]], l2, rows=[1, 3])
        np.testing.assert_array_equal(ys, y[[1, 3]])


def test_nvfp4_dequant_uses_exact_products(orc):
    rng = np.random.default_rng(28)
    x = (rng.standard_normal((4, 64)) * 100).astype(np.float32)
    q = orc.quantize(x, orc.NVFP4)
    d = q.dequantize()
    codes = _unpack4(q.codes)
    for r in range(4):
        for c in range(64):
            ref = orc.e2m1_value(int(codes[r, c])) * orc.e4m3_value(int(q.scales[r, c // 16])) * q.tensor_scale
            assert d[r, c] == ref


# ------------------------------------------------------------------ routing

def test_route_table_read(orc):
    n_layers, n_int, n_steps = 112, 10, 20
    table = (np.arange(n_layers * n_int) % 7).astype(np.uint8).reshape(n_layers, n_int)
    for layer in (0, 5, 111):
        for step in range(n_steps):
            assert orc.route(table, n_layers, n_int, layer, step, n_steps) == table[layer, step // 2]
    assert orc.route(table, n_layers, n_int, 112, 0, n_steps) == -1
    assert orc.route(table, n_layers, n_int, 0, 20, n_steps) == -1
    assert orc.route(table, n_layers, n_int, 0, -1, n_steps) == -1
    # uneven split: 7 intervals over 20 steps -> floor(step * 7 / 20)
    t7 = np.arange(7, dtype=np.uint8)[None, :]
    assert [orc.route(t7, 1, 7, 0, s, 20) for s in range(20)] == [s * 7 // 20 for s in range(20)]


# ------------------------------------------------------------------ per-channel mixed weight formats

def _e2m1_grid(rng, shape, scale):
    """Values of the E2M1 grid times `scale` (exact in binary32)."""
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    return (mags[rng.integers(0, 8, size=shape)] * rng.choice([-1.0, 1.0], size=shape) * scale)


def test_qlinear_mixed_exact_operands(orc):
    """Operands built to be exactly representable -- X in MXFP8, each weight row
    in the format it is given (MXFP4: E2M1 values times a power of two per
    32-block with the block maximum 6 times it; INT4-g32: integers in [-7, 7]
    times a power of two with a 7 in every block; NVFP4: E2M1 values times an
    E4M3 block scale per 16-block whose maximum is 6 times it, and one element
    2688 = 6 * 448 so the tensor scale is exactly 1) -- make the mixed product
    equal the plain product of the unquantized operands, which math.fsum gives
    independently of the oracle.  Routing a row to another format breaks the
    equality."""
    rng = np.random.default_rng(41)
    m, k = 5, 64
    x = np.zeros((m, k), np.float64)
    e4m3_vals = np.array([orc.e4m3_value(c) for c in range(0x7F)], np.float64)   # non-negative codes
    for i in range(m):
        for b in range(k // 32):
            e = int(rng.integers(-6, 6))
            blk = e4m3_vals[rng.integers(0, 0x7F, size=32)] * rng.choice([-1.0, 1.0], size=32)
            blk[int(rng.integers(0, 32))] = 448.0 * rng.choice([-1.0, 1.0])   # floor(log2 amax) - 8 = 0
            x[i, b * 32:(b + 1) * 32] = blk * 2.0 ** e
    choice = np.array([1, 3, 2, 2, 3, 1, 2], np.uint8)   # MXFP4, INT4-g32, NVFP4
    n = len(choice)
    w = np.zeros((n, k), np.float64)
    for r, f in enumerate(choice):
        if f == 1:
            for b in range(k // 32):
                j = int(rng.integers(-8, 0))
                blk = _e2m1_grid(rng, 32, 2.0 ** j)
                blk[int(rng.integers(0, 32))] = 6.0 * 2.0 ** j
                w[r, b * 32:(b + 1) * 32] = blk
        elif f == 3:
            for b in range(k // 32):
                j = int(rng.integers(-8, 0))
                blk = rng.integers(-7, 8, size=32).astype(np.float64) * 2.0 ** j
                blk[int(rng.integers(0, 32))] = -7.0 * 2.0 ** j
                w[r, b * 32:(b + 1) * 32] = blk
        else:
            for b in range(k // 16):
                e4 = float(e4m3_vals[int(rng.integers(8, 0x60))])   # normal E4M3 scales up to 448 / 2
                blk = _e2m1_grid(rng, 16, e4)
                blk[int(rng.integers(0, 16))] = 6.0 * e4
                w[r, b * 16:(b + 1) * 16] = blk
    w[2, 0:16] = _e2m1_grid(rng, 16, 448.0)
    w[2, 5] = 2688.0                                        # tensor amax: s_t = 2688 / 2688 = 1
    x32, w32 = x.astype(np.float32), w.astype(np.float32)
    assert np.array_equal(x32.astype(np.float64), x) and np.array_equal(w32.astype(np.float64), w)
    y = orc.qlinear_mixed(x32, w32, choice)
    for i in range(m):
        for j in range(n):
            ref = math.fsum(x[i, c] * w[j, c] for c in range(k))
            assert abs(y[i, j] - ref) <= 1e-13 * (1.0 + math.fsum(abs(x[i, c] * w[j, c]) for c in range(k)))
    # an NVFP4 row read as MXFP4 loses exactness somewhere
    wrong = choice.copy()
    wrong[2] = 1
    y2 = orc.qlinear_mixed(x32, w32, wrong)
    assert not np.allclose(y2[:, 2], y[:, 2], rtol=1e-9, atol=0)


def test_qlinear_mixed_permutation_and_tensor_scale(orc):
    """Permuting the output channels (weight rows with their formats) permutes
    the columns of Y; and an NVFP4 channel uses the tensor scale of the whole
    weight, not of the NVFP4 channels alone."""
    rng = np.random.default_rng(42)
    x = rng.standard_t(3, size=(6, 128)).astype(np.float32)
    w = (rng.standard_normal((9, 128)) * 0.02).astype(np.float32)
    w[4] *= 50.0                                             # the tensor maximum sits in an MXFP4 row
    choice = np.array([2, 3, 1, 2, 1, 3, 2, 1, 2], np.uint8)
    y = orc.qlinear_mixed(x, w, choice)
    perm = rng.permutation(9)
    yp = orc.qlinear_mixed(x, w[perm], choice[perm])
    np.testing.assert_array_equal(yp, y[:, perm])
    # column 0 (NVFP4) recomputed by brute force from the whole weight's NVFP4 quantization
    xd = orc.quantize(x, orc.MXFP8).dequantize()
    wq = orc.quantize(w, orc.NVFP4)
    assert wq.tensor_scale == orc.quantize(w[[4]], orc.NVFP4).tensor_scale   # set by the MXFP4 row
    wd = wq.dequantize()
    for i in range(6):
        ref = math.fsum(xd[i, c] * wd[0, c] for c in range(128))
        assert abs(y[i, 0] - ref) <= 1e-12 * (1 + abs(ref))
    # the NVFP4 rows alone would have had a different tensor scale
    alone = orc.quantize(w[choice == 2], orc.NVFP4)
    assert alone.tensor_scale != wq.tensor_scale
