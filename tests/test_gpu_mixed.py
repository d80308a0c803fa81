"""GPU parity of the linear layer whose weight keeps a format per output
channel (Chameleon article: each output channel takes the format with the
least reconstruction error among INT4-g32, NVFP4 and MXFP4), against MXFP8
activations: mxq_mixed_prepare + mxq_qlinear_mixed against the oracle's
binary64 product of exactly dequantized operands (oracle.qlinear_mixed).
Tolerance as the other GEMM tests (gpu_util.gemm_close)."""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import dev, gemm_close

pytestmark = pytest.mark.gpu

MXFP4, NVFP4, INT4_G32, MXFP8 = 1, 2, 3, 0
CANDS = (INT4_G32, NVFP4, MXFP4)


@pytest.fixture(scope="module")
def mxq():
    import microscaling_bit_quantization_b200 as m
    assert torch.cuda.is_available() and m.lib().mxq_device_supported(0) == 1
    return m


def _inputs(seed, m, n, k):
    rng = np.random.default_rng(seed)
    x = rng.standard_t(3, size=(m, k)).astype(np.float32)
    x[:, rng.choice(k, max(1, k // 64), replace=False)] *= 30
    w = (rng.standard_t(4, size=(n, k)) * 0.014).astype(np.float32)
    return workloads.to_bf16_values(x), workloads.to_bf16_values(w), rng


@pytest.mark.parametrize("shape", [(200, 300, 256), (64, 129, 128), (257, 520, 512), (1, 8, 64)])
def test_mixed_small(mxq, orc, shape):
    m, n, k = shape
    x, w, rng = _inputs(70 + n, m, n, k)
    choice = rng.choice(np.array(CANDS, np.uint8), size=n)
    xq = mxq.quantize(dev(x, "bf16"), MXFP8, 0, mxq.MMA)
    mw = mxq.prepare_mixed_weight(dev(w, "bf16"), choice)
    assert mw.n_group == tuple(int((choice == f).sum()) for f in (MXFP4, INT4_G32, NVFP4))
    ref = orc.qlinear_mixed(x, w, choice)
    for out_dtype in (torch.float32, torch.bfloat16):
        y = mxq.qlinear_mixed(xq, mw, out_dtype=out_dtype)
        assert mxq.check() == 0
        gemm_close(y.float().cpu().numpy(), ref, bf16_out=out_dtype == torch.bfloat16)


@pytest.mark.parametrize("only", [MXFP4, INT4_G32, NVFP4])
def test_mixed_single_group(mxq, orc, only):
    """Every channel in one format (the other groups empty) equals the oracle,
    and the chosen rows of an otherwise mixed weight keep their values when
    the grouping changes."""
    m, n, k = 150, 260, 384
    x, w, _ = _inputs(80 + only, m, n, k)
    choice = np.full(n, only, np.uint8)
    xq = mxq.quantize(dev(x, "bf16"), MXFP8, 0, mxq.MMA)
    y = mxq.qlinear_mixed(xq, mxq.prepare_mixed_weight(dev(w, "bf16"), choice), out_dtype=torch.float32)
    assert mxq.check() == 0
    gemm_close(y.cpu().numpy(), orc.qlinear_mixed(x, w, choice))


def test_mixed_selection_workload_full_size(mxq, orc):
    """Workload 2 at full size: W 3072 x 3072 (Student-t 4) with the formats
    the library's selection chose per channel, X 4096 x 3072 (Student-t 3)
    in MXFP8; 256 sampled rows x all columns, fp32 and bf16 output."""
    d = workloads.chameleon_selection()
    wd = dev(d["w"], "bf16")
    choice, _ = mxq.select_weight_format(wd, CANDS, want_sse=False)
    choice = choice.cpu().numpy()
    assert set(choice.tolist()) <= set(CANDS)
    xq = mxq.quantize(dev(d["x"], "bf16"), MXFP8, 0, mxq.MMA)
    mw = mxq.prepare_mixed_weight(wd, choice)
    rows = np.sort(np.random.default_rng(2).choice(4096, 256, replace=False))
    rows[-1] = 4095
    ref = orc.qlinear_mixed(d["x"], d["w"], choice, rows=rows)
    for out_dtype in (torch.float32, torch.bfloat16):
        y = mxq.qlinear_mixed(xq, mw, out_dtype=out_dtype)
        assert mxq.check() == 0
        gemm_close(y[torch.from_numpy(rows).cuda()].float().cpu().numpy(), ref,
                   bf16_out=out_dtype == torch.bfloat16)
