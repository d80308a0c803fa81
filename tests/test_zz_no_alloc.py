"""The allocation-free entry point, mxq_quantize_lowrank_noalloc, against the
workspace entry point mxq_quantize_lowrank.

Some callers cannot allocate device memory themselves: a host application
that owns every device buffer and passes the library only inputs and
outputs, or a latency-bound caller that cannot afford a cudaMalloc (which
may synchronize the device).  For them the library keeps its scratch in a
4 MiB device array of its own.  This file is named so that pytest collects
it last; it also passes when run alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mxq():
    import microscaling_bit_quantization_b200 as m
    assert torch.cuda.is_available() and m.lib().mxq_device_supported(0) == 1
    return m


def _inputs(seed, m, k, n, r):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(m, k, generator=g)
    x[:, torch.randperm(k, generator=g)[: k // 64]] *= 40.0
    w = torch.randn(n, k, generator=g) * 0.02
    l1 = torch.randn(k, r, generator=g) * 0.05
    l2 = torch.randn(r, n, generator=g) * 0.05
    bf = torch.bfloat16
    return x.to(bf).cuda(), w.to(bf).cuda(), l1.to(bf).cuda(), l2.to(bf).cuda()


def _noalloc_call(mxq, x, fmt, l1, wq, hadamard_b=0):
    """Direct call through the C ABI (no workspace argument)."""
    m, k = x.shape
    q = mxq.alloc_qtensor(fmt, m, k, mxq.MMA, x.device)
    tp = torch.empty((m, 64), dtype=torch.bfloat16, device=x.device)
    P = ctypes.c_void_p
    xdt = mxq.BF16 if x.dtype == torch.bfloat16 else mxq.F32
    st = mxq.lib().mxq_quantize_lowrank_noalloc(
        P(x.data_ptr()), xdt, m, k, fmt, hadamard_b, P(l1.data_ptr()), l1.shape[1],
        P(wq.tensor_scale.data_ptr()) if wq.tensor_scale is not None else None,
        P(q.codes.data_ptr()), P(q.scales.data_ptr()) if q.scales is not None else None,
        P(q.tensor_scale.data_ptr()) if q.tensor_scale is not None else None, P(tp.data_ptr()),
        P(torch.cuda.current_stream().cuda_stream))
    return st, q, tp


@pytest.mark.parametrize("fmt", [2, 1])   # NVFP4, MXFP4
def test_noalloc_matches_workspace_entry_point(mxq, fmt):
    for call, seed in enumerate((11, 12)):   # two calls in a row share the device array
        x, w, l1, l2 = _inputs(seed + 10 * fmt, 300 + 64 * call, 512, 384, 32)
        wq = mxq.quantize(w, fmt, 0, mxq.MMA)
        ref_q, ref_tp = mxq.quantize_lowrank(x, fmt, l1, wq)
        st, q, tp = _noalloc_call(mxq, x, fmt, l1, wq)
        assert st == 0
        torch.cuda.synchronize()
        assert torch.equal(q.codes, ref_q.codes)
        assert torch.equal(q.scales, ref_q.scales)
        if fmt == 2:
            assert torch.equal(q.tensor_scale, ref_q.tensor_scale)
        assert torch.equal(tp.view(torch.int16), ref_tp.view(torch.int16))
        # and the layer output built on it, within the GEMM tolerance
        l2p = mxq.lowrank_pack_l2(l2)
        y = mxq.qlinear(q, wq, tp, l2p, out_dtype=torch.float32).double().cpu().numpy()
        y_ref = mxq.qlinear(ref_q, wq, ref_tp, l2p, out_dtype=torch.float32).double().cpu().numpy()
        assert mxq.check() == 0
        err = np.abs(y - y_ref)
        assert np.linalg.norm(y - y_ref) <= 1e-4 * np.linalg.norm(y_ref)
        assert err.max() <= 1e-4 * np.abs(y_ref).max()


@pytest.mark.parametrize("x_fp32,hadamard_b,m0,k", [(True, 0, 260, 512), (False, 128, 260, 512),
                                                    (True, 128, 260, 512), (True, 0, 16384, 64)])
def test_noalloc_amax_routes(mxq, x_fp32, hadamard_b, m0, k):
    """NVFP4 through the other amax routes in the shared array: per-CTA
    maxima of the mma.sync low-rank kernel (fp32 input), of the amax pass
    (with the rotation), and, past 960 16-row CTAs, the amax word cleared and
    folded into: two calls in a row (the second on a different input, so a
    stale maximum would show) equal the workspace entry point bit for bit."""
    fmt = 2
    for call, seed in enumerate((21, 22)):
        x, w, l1, _ = _inputs(seed + 7 * hadamard_b, m0 + 64 * call, k, 384, 32)
        if x_fp32:
            x = x.float()
        if call == 1:
            x = x * 0.25   # a smaller tensor amax than the first call's
        wq = mxq.quantize(w, fmt, hadamard_b, mxq.MMA)
        ref_q, ref_tp = mxq.quantize_lowrank(x, fmt, l1, wq, hadamard_b)
        st, q, tp = _noalloc_call(mxq, x, fmt, l1, wq, hadamard_b)
        assert st == 0
        torch.cuda.synchronize()
        assert mxq.check() == 0
        assert torch.equal(q.codes, ref_q.codes)
        assert torch.equal(q.scales, ref_q.scales)
        assert torch.equal(q.tensor_scale, ref_q.tensor_scale)
        assert torch.equal(tp.view(torch.int16), ref_tp.view(torch.int16))


def test_noalloc_rejects_sizes_beyond_the_array(mxq):
    x, w, l1, _ = _inputs(13, 64, 512, 128, 32)
    wq = mxq.quantize(w, 2, 0, mxq.MMA)
    P = ctypes.c_void_p
    dummy = P(x.data_ptr())
    # 4096 + 4 * m * r bytes must fit in 4 MiB: m = 40000 rows at rank 32 does not
    st = mxq.lib().mxq_quantize_lowrank_noalloc(dummy, mxq.BF16, 40000, 512, 2, 0, P(l1.data_ptr()), 32,
                                                P(wq.tensor_scale.data_ptr()), dummy, dummy, dummy, dummy, None)
    assert st == 5   # MXQ_ENOSPACE, nothing launched
