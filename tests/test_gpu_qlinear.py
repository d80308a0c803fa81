"""GPU parity of the low-rank branch and the tcgen05 block-scaled GEMM
against the oracle's binary64 GEMM over exactly dequantized operands.

Tolerance for fp32 output: relative Frobenius error
<= 1e-4 and max abs error <= 1e-4 * max|Y_ref|; bf16 output also allows the
final bf16 rounding (see gpu_util.gemm_close).  Quantized operands are
produced by the library and checked bit-exact against the oracle's in
test_gpu_quantize; here the oracle re-derives every operand (codes, scales,
T = bf16(X) . L1) from the same seeded inputs itself."""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import assert_qtensor_equal, dev, gemm_close, host_values

pytestmark = pytest.mark.gpu

GEMM_FMTS = (2, 1, 0, 6, 5, 4, 3)   # NVFP4, MXFP4, MXFP8, FP8_TENSOR, INT8_ROW, INT4_G64, INT4_G32
LOWRANK_FMTS = (2, 1, 0, 6, 4, 3)


@pytest.fixture(scope="module")
def mxq():
    import microscaling_bit_quantization_b200 as m
    assert torch.cuda.is_available() and m.lib().mxq_device_supported(0) == 1
    return m


def _inputs(seed, m, n, k, r=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_t(4, size=(m, k)).astype(np.float32)
    x[:, rng.choice(k, max(1, k // 64), replace=False)] *= 30
    w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    out = {"x": workloads.to_bf16_values(x), "w": workloads.to_bf16_values(w)}
    if r:
        out["l1"] = workloads.to_bf16_values((rng.standard_normal((k, r)) * 0.05).astype(np.float32))
        out["l2"] = workloads.to_bf16_values((rng.standard_normal((r, n)) * 0.05).astype(np.float32))
    return out


def _run(mxq, fmt, d, r, out_dtype, hadamard_b=0, x_dtype="bf16"):
    xq = mxq.quantize(dev(d["x"], x_dtype), fmt, hadamard_b, mxq.MMA)
    wq = mxq.quantize(dev(d["w"], "bf16"), fmt, hadamard_b, mxq.MMA)
    tp = l2p = None
    if r:
        tp = mxq.lowrank_down_packed(dev(d["x"], x_dtype), dev(d["l1"], "bf16"), xq, wq)
        l2p = mxq.lowrank_pack_l2(dev(d["l2"], "bf16"))
    y = mxq.qlinear(xq, wq, tp, l2p, out_dtype=out_dtype)
    assert mxq.check() == 0
    return y, xq, wq


def _ref(orc, fmt, d, r, rows=None, hadamard_b=0):
    oxq = orc.quantize(d["x"], fmt, hadamard_b)
    owq = orc.quantize(d["w"], fmt, hadamard_b)
    t = None
    if r:
        t = orc.lowrank_down(d["x"], d["l1"]) if rows is None else orc.lowrank_down_rows(d["x"], d["l1"], rows)
    return orc.qlinear(oxq, owq, t, d.get("l2"), rows=rows), oxq, owq


@pytest.mark.parametrize("fmt", GEMM_FMTS)
@pytest.mark.parametrize("shape", [(200, 384, 512), (64, 128, 256), (130, 520, 320), (257, 256, 1024)])
def test_qlinear_shapes(mxq, orc, fmt, shape):
    m, n, k = shape
    if k % 64 and fmt in (1, 2, 4):
        pytest.skip("K must be a multiple of 64")
    d = _inputs(10 + fmt, m, n, k)
    ref, oxq, owq = _ref(orc, fmt, d, 0)
    for out_dtype in (torch.float32, torch.bfloat16):
        y, xq, wq = _run(mxq, fmt, d, 0, out_dtype)
        gemm_close(y.float().cpu().numpy(), ref, bf16_out=out_dtype == torch.bfloat16)
    assert_qtensor_equal(xq, oxq, layout_mma=True)
    assert_qtensor_equal(wq, owq, layout_mma=True)


@pytest.mark.parametrize("fmt", GEMM_FMTS)
def test_qlinear_short_k(mxq, orc, fmt):
    k = 64 if fmt in (1, 2, 4) else 96
    d = _inputs(20 + fmt, 70, 300, k)
    ref, _, _ = _ref(orc, fmt, d, 0)
    y, _, _ = _run(mxq, fmt, d, 0, torch.float32)
    gemm_close(y.cpu().numpy(), ref)


@pytest.mark.parametrize("fmt", GEMM_FMTS)
@pytest.mark.parametrize("shape", [(2200, 2200, 512), (2560, 1000, 512)])
def test_qlinear_partial_last_round(mxq, orc, fmt, shape):
    """Rounds of the persistent walk over 74 clusters, with ragged edges and
    the low-rank branch where the format takes it; every output element
    checked.  2200 x 2200: 81 tiles of 256 x 256, a partly filled second
    round (the last tiles are 152 rows and 152 columns).  2560 x 1000: 40
    tiles in one round, the last column tile 232 wide."""
    m, n, k = shape
    r = 32 if fmt in LOWRANK_FMTS else 0
    d = _inputs(60 + fmt + (m % 7), m, n, k, r)
    ref, _, _ = _ref(orc, fmt, d, r)
    for out_dtype in (torch.float32, torch.bfloat16):
        y, _, _ = _run(mxq, fmt, d, r, out_dtype)
        gemm_close(y.float().cpu().numpy(), ref, bf16_out=out_dtype == torch.bfloat16)


@pytest.mark.parametrize("fmt", LOWRANK_FMTS)
@pytest.mark.parametrize("r", [8, 32])
def test_qlinear_lowrank(mxq, orc, fmt, r):
    d = _inputs(30 + fmt, 150, 384, 512, r)
    ref, _, _ = _ref(orc, fmt, d, r)
    for out_dtype in (torch.float32, torch.bfloat16):
        y, _, _ = _run(mxq, fmt, d, r, out_dtype)
        gemm_close(y.float().cpu().numpy(), ref, bf16_out=out_dtype == torch.bfloat16)


def test_lowrank_down(mxq, orc):
    d = workloads.svdquant_mlp_up(draw_weights=False)
    t = mxq.lowrank_down(dev(d["x"], "bf16"), dev(d["l1"], "bf16")).cpu().numpy().astype(np.float64)
    ref = orc.lowrank_down(d["x"], d["l1"])
    err = np.abs(t - ref)
    assert err.max() <= 1e-5 * np.abs(ref).max()
    w1 = workloads.tiny_nvfp4_linear()
    t = mxq.lowrank_down(dev(w1["x"], "f32"), dev(w1["l1"], "bf16")).cpu().numpy()
    ref = orc.lowrank_down(w1["x"], w1["l1"])
    assert np.abs(t - ref).max() <= 1e-5 * np.abs(ref).max()


@pytest.mark.parametrize("m,k,r", [(300, 208, 32), (129, 80, 32), (257, 1104, 32), (300, 208, 24), (64, 16, 32)])
def test_lowrank_down_ragged(mxq, orc, m, k, r):
    """T = bf16(X) . L1 with K not a multiple of the 64-column k-block (the
    rank-32 path loads L1's rows by TMA and the rows past K read as zeros; the
    other ranks build the tiles in the kernel) and M not a multiple of 128;
    every element against the oracle's binary64 T."""
    rng = np.random.default_rng(70 + k + r)
    x = workloads.to_bf16_values(rng.standard_t(4, size=(m, k)).astype(np.float32))
    l1 = workloads.to_bf16_values((rng.standard_normal((k, r)) * 0.05).astype(np.float32))
    t = mxq.lowrank_down(dev(x, "bf16"), dev(l1, "bf16")).cpu().numpy().astype(np.float64)
    ref = orc.lowrank_down(x, l1)
    assert t.shape == ref.shape
    assert np.abs(t - ref).max() <= 1e-5 * max(np.abs(ref).max(), 1e-30)


def test_tiny_nvfp4_linear_full(mxq, orc):
    """Workload 1 end to end, every output: fp32 X, NVFP4, rank-8 branch."""
    w1 = workloads.tiny_nvfp4_linear()
    d = {"x": w1["x"], "w": w1["w"], "l1": w1["l1"], "l2": w1["l2"]}
    ref, oxq, owq = _ref(orc, 2, d, 8)
    xq = mxq.quantize(dev(d["x"], "f32"), 2, 0, mxq.MMA)
    wq = mxq.quantize(dev(d["w"], "f32"), 2, 0, mxq.MMA)
    assert_qtensor_equal(xq, oxq, layout_mma=True)
    assert_qtensor_equal(wq, owq, layout_mma=True)
    l2p = mxq.lowrank_pack_l2(dev(d["l2"], "bf16"))
    # both routes to the packed branch operand: fused, and fp32 t then pack
    tp_fused = mxq.lowrank_down_packed(dev(d["x"], "f32"), dev(d["l1"], "bf16"), xq, wq)
    t = mxq.lowrank_down(dev(d["x"], "f32"), dev(d["l1"], "bf16"))
    tp_split = mxq.lowrank_pack_t(t, xq, wq)
    assert torch.equal(tp_fused.view(torch.int16), tp_split.view(torch.int16))
    y = mxq.qlinear(xq, wq, tp_fused, l2p, out_dtype=torch.float32)
    assert mxq.check() == 0
    gemm_close(y.cpu().numpy(), ref)


def _sample_rows(m, seed, count=256):
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(m, size=count, replace=False))
    rows[-1] = m - 1
    return rows


@pytest.mark.parametrize("fmt", [2, 1, 4])
def test_svdquant_mlp_up_full_size(mxq, orc, fmt):
    """Workload 3 at full size (4096 x 12288 x 3072, rank 32) in the launch
    configuration the benchmark times (NVFP4 and the INT4-g64 variant, plus
    MXFP4); 256 sampled rows x all columns."""
    d = workloads.svdquant_mlp_up()
    rows = _sample_rows(4096, 3)
    ref, _, _ = _ref(orc, fmt, d, 32, rows=rows)
    for out_dtype in (torch.bfloat16, torch.float32):
        y, _, _ = _run(mxq, fmt, d, 32, out_dtype)
        gemm_close(y[torch.from_numpy(rows).cuda()].float().cpu().numpy(), ref,
                   bf16_out=out_dtype == torch.bfloat16)
        del y


@pytest.mark.parametrize("hadamard_b", [0, 128])
def test_mxfp4_hadamard_full_size(mxq, orc, hadamard_b):
    """Workload 4: 8192 x 4096 x 4096 MXFP4, with and without the b=128 rotation."""
    d = workloads.mxfp4_hadamard_gemm()
    rows = _sample_rows(8192, 4)
    ref, _, _ = _ref(orc, 1, d, 0, rows=rows, hadamard_b=hadamard_b)
    y, _, _ = _run(mxq, 1, d, 0, torch.float32, hadamard_b=hadamard_b)
    gemm_close(y[torch.from_numpy(rows).cuda()].cpu().numpy(), ref)


@pytest.mark.parametrize("fmt", [5, 6, 0])
def test_dit_layers_full_size(mxq, orc, fmt):
    """Workload 5 linears at M = 8192 in each routed format."""
    seed = 5
    for (name, kin, nout), step in zip(workloads.DIT_LINEARS, (0, 7, 13, 19)):
        x = workloads.dit_activation(seed, step, kin)
        w = workloads.dit_weight(seed, 0, kin, nout)
        d = {"x": x, "w": w}
        rows = _sample_rows(workloads.DIT_TOKENS, step, 128)
        ref, _, _ = _ref(orc, fmt, d, 0, rows=rows)
        y, _, _ = _run(mxq, fmt, d, 0, torch.float32)
        gemm_close(y[torch.from_numpy(rows).cuda()].cpu().numpy(), ref)


@pytest.mark.parametrize("fmt", LOWRANK_FMTS)
@pytest.mark.parametrize("hadamard_b", [0, 64])
@pytest.mark.parametrize("x_dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [(77, 300, 512, 24), (16448, 64, 64, 16)], ids=["small", "tall"])
def test_quantize_lowrank_fused(mxq, orc, fmt, hadamard_b, x_dtype, shape):
    """The fused activation path equals quantize + lowrank_down_packed bit for
    bit, and its codes/scales equal the oracle's.  The tall shape takes, for
    the tensor-scaled formats, the route that folds every CTA's maximum into
    a cleared word (more 16-row CTAs than amax slots); the small one the
    per-CTA slots."""
    m, n, k, r = shape
    d = _inputs(40 + fmt, m, n, k, r)
    x = dev(d["x"], x_dtype)
    wq = mxq.quantize(dev(d["w"], "bf16"), fmt, hadamard_b, mxq.MMA)
    l1 = dev(d["l1"], "bf16")
    xq, tp = mxq.quantize_lowrank(x, fmt, l1, wq, hadamard_b)
    xq2 = mxq.quantize(x, fmt, hadamard_b, mxq.MMA)
    tp2 = mxq.lowrank_down_packed(x, l1, xq2, wq)
    torch.cuda.synchronize()
    assert torch.equal(xq.codes, xq2.codes)
    if xq.scales is not None:
        assert torch.equal(xq.scales, xq2.scales)
    assert torch.equal(tp.view(torch.int16), tp2.view(torch.int16))
    assert_qtensor_equal(xq, orc.quantize(host_values(d["x"], x_dtype), fmt, hadamard_b), layout_mma=True)


def test_svdquant_fused_path_full_size(mxq, orc):
    """Workload 3 through the fused activation path, as the benchmark runs it."""
    d = workloads.svdquant_mlp_up()
    rows = _sample_rows(4096, 33)
    ref, _, _ = _ref(orc, 2, d, 32, rows=rows)
    wq = mxq.quantize(dev(d["w"], "bf16"), 2, 0, mxq.MMA)
    xq, tp = mxq.quantize_lowrank(dev(d["x"], "bf16"), 2, dev(d["l1"], "bf16"), wq)
    l2p = mxq.lowrank_pack_l2(dev(d["l2"], "bf16"))
    y = mxq.qlinear(xq, wq, tp, l2p, out_dtype=torch.bfloat16)
    assert mxq.check() == 0
    gemm_close(y[torch.from_numpy(rows).cuda()].float().cpu().numpy(), ref, bf16_out=True)


@pytest.mark.parametrize("fmt", [4, 3])
def test_igroup_ragged_and_degenerate(mxq, orc, fmt):
    """INT4 group GEMM: ragged M and N (not multiples of the 128 x 128 tile),
    a K that leaves half a pipeline stage, all-zero activation rows and weight
    rows (group scale 0), and more tiles than SMs."""
    g = 64 if fmt == 4 else 32
    for m, n, k in ((1, 8, g), (129, 136, 3 * g), (300, 1000, 5 * g)):
        d = _inputs(50 + fmt, m, n, k, 16)
        d["x"][m // 2] = 0.0
        d["w"][n // 3] = 0.0
        ref, _, _ = _ref(orc, fmt, d, 16)
        y, _, _ = _run(mxq, fmt, d, 16, torch.float32)
        gemm_close(y.cpu().numpy(), ref)
    d = _inputs(60 + fmt, 1100, 2400, 256)   # 9 x 19 tiles > 148 SMs: persistent CTAs take several
    ref, _, _ = _ref(orc, fmt, d, 0, rows=_sample_rows(1100, 7))
    y, _, _ = _run(mxq, fmt, d, 0, torch.float32)
    gemm_close(y[torch.from_numpy(_sample_rows(1100, 7)).cuda()].cpu().numpy(), ref)


def test_launch_chain_reused_buffers(mxq):
    """Workload 3's step twice per round, both steps sharing the quantized
    activation, packed T and workspace, with no synchronization between them:
    the kernels overlap their setup with the previous kernel but must not read
    or write global memory before it completes, so every output equals the
    same step run alone."""
    d = workloads.svdquant_mlp_up()
    wq = mxq.quantize(dev(d["w"], "bf16"), 2, 0, mxq.MMA)
    l1 = dev(d["l1"], "bf16")
    l2p = mxq.lowrank_pack_l2(dev(d["l2"], "bf16"))
    m, k = d["x"].shape
    xs = [dev(d["x"], "bf16"), dev(workloads.svdquant_mlp_up(seed=9, draw_weights=False)["x"], "bf16")]
    xq = mxq.alloc_qtensor(2, m, k, mxq.MMA)
    tp = torch.empty((m, 64), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(mxq.quantize_lowrank_workspace_bytes(m, 32), dtype=torch.uint8, device="cuda")

    def step(x, y):
        mxq.quantize_lowrank(x, 2, l1, wq, 0, out=xq, tp=tp, workspace=ws)
        mxq.qlinear(xq, wq, tp, l2p, out=y)

    alone = []
    for x in xs:
        y = torch.empty((m, wq.rows), dtype=torch.bfloat16, device="cuda")
        step(x, y)
        torch.cuda.synchronize()
        alone.append(y)
    outs = [torch.empty_like(alone[0]) for _ in range(6)]
    for i, y in enumerate(outs):
        step(xs[i % 2], y)
    torch.cuda.synchronize()
    assert mxq.check() == 0
    for i, y in enumerate(outs):
        assert torch.equal(y, alone[i % 2]), i


# ------------------------------------------------------------------ W4A16

@pytest.mark.parametrize("fmt", [4, 3])
@pytest.mark.parametrize("shape", [(37, 200, 512), (300, 260, 192), (129, 128, 64), (1, 8, 128)])
def test_w4a16_small(mxq, orc, fmt, shape):
    """bf16 activations x INT4-g64 / g32 weights (canonical layout), ragged M
    and N, one K stage up to eight; every element against the oracle."""
    m, n, k = shape
    d = _inputs(90 + fmt, m, n, k)
    xv = host_values(d["x"], "bf16")
    wq = mxq.quantize(dev(d["w"], "bf16"), fmt)
    owq = orc.quantize(host_values(d["w"], "bf16"), fmt)
    assert_qtensor_equal(wq, owq)
    ref = orc.w4a16(xv, owq)
    for out_dtype in (torch.float32, torch.bfloat16):
        y = mxq.qlinear_w4a16(dev(d["x"], "bf16"), wq, out_dtype=out_dtype)
        assert mxq.check() == 0
        gemm_close(y.float().cpu().numpy(), ref, bf16_out=out_dtype == torch.bfloat16)


@pytest.mark.parametrize("fmt", [4, 3])
def test_w4a16_both_routes(mxq, orc, fmt):
    """m = 600 (above the size where the library asks for a workspace): the
    unpacked-weight route and the fused kernel, every element against the
    oracle, fp32 and bf16 out."""
    m, n, k = 600, 392, 320
    d = _inputs(95 + fmt, m, n, k)
    assert mxq.qlinear_w4a16_workspace_bytes(m, n, k) == n * k * 2
    wq = mxq.quantize(dev(d["w"], "bf16"), fmt)
    ref = orc.w4a16(host_values(d["x"], "bf16"), orc.quantize(host_values(d["w"], "bf16"), fmt))
    for fused in (False, True):
        for out_dtype in (torch.float32, torch.bfloat16):
            y = mxq.qlinear_w4a16(dev(d["x"], "bf16"), wq, out_dtype=out_dtype, fused=fused)
            assert mxq.check() == 0
            gemm_close(y.float().cpu().numpy(), ref, bf16_out=out_dtype == torch.bfloat16)


def test_w4a16_full_size(mxq, orc):
    """Workload 3's shape with its residual weight as INT4-g64: 256 sampled
    rows (all 12288 columns) against the oracle."""
    d = workloads.svdquant_mlp_up()
    wq = mxq.quantize(dev(d["w"], "bf16"), 4)
    owq = orc.quantize(d["w"], 4)
    rows = _sample_rows(4096, 91)
    ref = orc.w4a16(d["x"], owq, rows=rows)
    y = mxq.qlinear_w4a16(dev(d["x"], "bf16"), wq)
    assert mxq.check() == 0
    gemm_close(y[torch.from_numpy(rows).cuda()].float().cpu().numpy(), ref, bf16_out=True)


def test_launch_chain_in_cuda_graph(mxq):
    """The fused activation path and the GEMM captured in a CUDA graph (the
    programmatic launches become programmatic graph edges) give, on replay,
    exactly the outputs of the same calls run eagerly."""
    d = workloads.svdquant_mlp_up(m=1024, n=2048)
    wq = mxq.quantize(dev(d["w"], "bf16"), 2, 0, mxq.MMA)
    l1 = dev(d["l1"], "bf16")
    l2p = mxq.lowrank_pack_l2(dev(d["l2"], "bf16"))
    x = dev(d["x"], "bf16")
    m, k = x.shape
    xq = mxq.alloc_qtensor(2, m, k, mxq.MMA)
    tp = torch.empty((m, 64), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(mxq.quantize_lowrank_workspace_bytes(m, 32), dtype=torch.uint8, device="cuda")
    y_eager = torch.empty((m, wq.rows), dtype=torch.bfloat16, device="cuda")
    y_graph = torch.empty_like(y_eager)

    def step(y):
        mxq.quantize_lowrank(x, 2, l1, wq, 0, out=xq, tp=tp, workspace=ws)
        mxq.qlinear(xq, wq, tp, l2p, out=y)

    step(y_eager)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(y_graph)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(3):
            step(y_graph)
    y_graph.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert mxq.check() == 0
    assert torch.equal(y_graph, y_eager)
