"""The routed linear layer, mxq_qlinear_routed: the format-table read, the
activation quantized in the routed format and the GEMM against the weight
prepared in that format, in one library call (Chameleon article: each layer
reads its activation format for the current timestep interval from a table
at generation time).

Workload 5 (28 DiT blocks x 4 linears, M = 8192, 20 steps in 10 intervals,
a seeded table over INT8 per token, FP8 per tensor and MXFP8, 4 layers forced
to MXFP8 whose inputs carry channel ranges up to 163x): sampled (layer,
step) pairs covering every format, every linear shape and a forced layer,
128 sampled rows x all columns against the oracle's route -> quantize ->
binary64 GEMM.  Tolerance as the other GEMM tests (gpu_util.gemm_close)."""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import dev, gemm_close

pytestmark = pytest.mark.gpu

SEED = 5
N_STEPS = workloads.DIT_STEPS


@pytest.fixture(scope="module")
def mxq():
    import microscaling_bit_quantization_b200 as m
    assert torch.cuda.is_available() and m.lib().mxq_device_supported(0) == 1
    return m


def _pairs(table, forced):
    """(layer, step) pairs: per chosen step one forced layer and, for each of
    the three formats, a layer routed to it at that step, rotating through the
    four linear shapes."""
    pairs = []
    n_layers = table.shape[0]
    forced_set = set(int(f) for f in forced)
    for si, step in enumerate((0, 7, 12, 19)):
        pairs.append((int(forced[si % len(forced)]), step))
        interval = step * table.shape[1] // N_STEPS
        for fi, fmt in enumerate((5, 6, 0)):
            kind = (si + fi) % 4
            for layer in range(kind, n_layers, 4):
                if layer not in forced_set and table[layer, interval] == fmt:
                    pairs.append((layer, step))
                    break
    return pairs


def test_pairs_cover_the_stack():
    table, forced = workloads.dit_format_table(SEED)
    pairs = _pairs(table, forced)
    fmts = {int(table[layer, step * 10 // N_STEPS]) for layer, step in pairs}
    assert fmts == {5, 6, 0}
    assert {layer % 4 for layer, _ in pairs} == {0, 1, 2, 3}
    assert any(layer in set(forced.tolist()) for layer, _ in pairs)


def test_routed_stack_against_oracle(mxq, orc):
    table, forced = workloads.dit_format_table(SEED)
    n_layers = table.shape[0]
    ws = torch.empty(mxq.qlinear_routed_workspace_bytes(workloads.DIT_TOKENS, workloads.DIT_MLP, 0),
                     dtype=torch.uint8, device="cuda")
    for i, (layer, step) in enumerate(_pairs(table, forced)):
        kin, nout = workloads.dit_layer_shape(layer)
        x = workloads.dit_layer_input(SEED, step, layer, forced)
        w = workloads.dit_weight(SEED, layer, kin, nout)
        lw = mxq.prepare_routed_layer(dev(w, "bf16"), set(table[layer].tolist()))
        out_dtype = torch.bfloat16 if i % 3 == 2 else torch.float32
        y, used = mxq.qlinear_routed(dev(x, "bf16"), lw, table, layer, step, N_STEPS, out_dtype=out_dtype,
                                     workspace=ws)
        assert mxq.check() == 0
        fmt = orc.route(table, n_layers, table.shape[1], layer, step, N_STEPS)
        assert used == fmt
        rows = np.sort(np.random.default_rng(1000 + i).choice(workloads.DIT_TOKENS, 128, replace=False))
        rows[-1] = workloads.DIT_TOKENS - 1
        ref = orc.qlinear(orc.quantize(x, fmt), orc.quantize(w, fmt), rows=rows)
        got = y[torch.from_numpy(rows).cuda()].float().cpu().numpy()
        gemm_close(got, ref, bf16_out=out_dtype == torch.bfloat16)
        del y, lw


def test_routed_equals_composed_calls(mxq):
    """The routed call runs exactly the kernels of the separate calls: its
    output equals quantize (or quantize_lowrank) + qlinear bit for bit, with
    and without the low-rank branch and the rotation."""
    rng = np.random.default_rng(7)
    m, k, n, r = 300, 512, 640, 16
    x = dev(workloads.to_bf16_values(rng.standard_t(3, size=(m, k)).astype(np.float32)), "bf16")
    w = dev(workloads.to_bf16_values((rng.standard_normal((n, k)) * 0.02).astype(np.float32)), "bf16")
    l1 = dev(workloads.to_bf16_values((rng.standard_normal((k, r)) * 0.05).astype(np.float32)), "bf16")
    l2 = dev(workloads.to_bf16_values((rng.standard_normal((r, n)) * 0.05).astype(np.float32)), "bf16")
    table = np.array([[2, 1, 0, 6], [4, 3, 5, 2]], np.uint8)   # 2 layers x 4 intervals, 8 steps
    for layer, branch, had in ((0, False, 0), (0, True, 0), (1, True, 0), (0, False, 64), (1, False, 0)):
        fmts = set(table[layer].tolist())
        if had:
            fmts = {f for f in fmts if f != 5 and f != 6}
        lw = mxq.prepare_routed_layer(w, fmts, l1 if branch else None, l2 if branch else None, hadamard_b=had)
        for step in range(8):
            fmt = int(table[layer, step // 2])
            if fmt not in fmts or (branch and fmt == 5):
                continue
            y, used = mxq.qlinear_routed(x, lw, table, layer, step, 8, out_dtype=torch.float32)
            assert used == fmt
            wq = lw.weights[fmt]
            if branch:
                xq, tp = mxq.quantize_lowrank(x, fmt, l1, wq, had)
                y2 = mxq.qlinear(xq, wq, tp, lw.l2p, out_dtype=torch.float32)
            else:
                xq = mxq.quantize(x, fmt, had, mxq.MMA)
                y2 = mxq.qlinear(xq, wq, out_dtype=torch.float32)
            assert mxq.check() == 0
            assert torch.equal(y, y2), (layer, branch, had, step, fmt)


def test_routed_lowrank_against_oracle(mxq, orc):
    """Workload 1 (fp32 activations, NVFP4, rank-8 branch) through the routed
    call: every output element against the oracle."""
    d = workloads.tiny_nvfp4_linear()
    table = np.full((1, 10), 2, np.uint8)
    lw = mxq.prepare_routed_layer(dev(d["w"], "f32"), [2], dev(d["l1"], "bf16"), dev(d["l2"], "bf16"))
    y, used = mxq.qlinear_routed(dev(d["x"], "f32"), lw, table, 0, 3, N_STEPS, out_dtype=torch.float32)
    assert mxq.check() == 0 and used == 2
    ref = orc.qlinear(orc.quantize(d["x"], 2), orc.quantize(d["w"], 2), orc.lowrank_down(d["x"], d["l1"]), d["l2"])
    gemm_close(y.cpu().numpy(), ref)
