"""Seeded synthetic inputs for the five workloads.

This module holds random draws and dtype rounding only -- none of the
quantization method's arithmetic -- so that the oracle and the CUDA library
are fed byte-identical inputs.  Every tensor comes from numpy's
``default_rng`` on a ``SeedSequence`` sub-stream named by the tensor, is
drawn in binary64, cast to fp32 and, for bf16 tensors, rounded once to
bf16 (round-to-nearest-even, through torch's CPU cast).  Arrays are returned
as fp32 numpy arrays holding the exact (bf16-representable where stated)
values.

The distributions follow what the pages say about diffusion-model tensors:
heavy tails and a few outlier channels (Chameleon article: early denoising
steps carry more outliers; the SDXL skip-concat convolutions see channel
ranges up to 163x; MixDiT article section 1: a small share of outliers
carries much of the activation energy), and the sizes of a DiT/UNet linear
layer.  The exact recipes are in the workload docstrings.
"""
from __future__ import annotations

import numpy as np

try:
    import torch
except ImportError:  # pragma: no cover - torch is part of the image
    torch = None


def _rng(seed: int, name: str) -> np.random.Generator:
    key = [ord(c) for c in name]
    return np.random.default_rng(np.random.SeedSequence([seed] + key))


def to_bf16_values(a: np.ndarray) -> np.ndarray:
    """Round an fp32 array to bf16 (RNE) and return the values as fp32."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def normal(seed, name, shape, std=1.0, bf16=True):
    a = (_rng(seed, name).standard_normal(shape) * std).astype(np.float32)
    return to_bf16_values(a) if bf16 else a


def student_t(seed, name, shape, nu, scale=1.0, bf16=True):
    a = (_rng(seed, name).standard_t(nu, size=shape) * scale).astype(np.float32)
    return to_bf16_values(a) if bf16 else a


def laplace(seed, name, shape, b=1.0, bf16=True):
    a = _rng(seed, name).laplace(0.0, b, size=shape).astype(np.float32)
    return to_bf16_values(a) if bf16 else a


def outlier_columns(seed, name, k, count, lo, hi, pin_max=None):
    """`count` distinct column indices of [0, k) and log-uniform factors in
    [lo, hi]; with pin_max, the first chosen column gets exactly pin_max."""
    g = _rng(seed, name)
    cols = np.sort(g.choice(k, size=count, replace=False))
    f = np.exp(g.uniform(np.log(lo), np.log(hi), size=count))
    if pin_max is not None:
        f[0] = pin_max
    return cols, f.astype(np.float32)


# --------------------------------------------------------------------------
# Workload 1: tiny NVFP4 W4A4 linear with a rank-8 low-rank branch.
# --------------------------------------------------------------------------
def tiny_nvfp4_linear(seed: int = 1):
    """X 64x256 fp32 N(0,1) with 4 seeded outlier columns x50; W 128x256 fp32
    N(0, 0.02^2); L1 256x8 and L2 8x128 bf16 N(0, 0.01^2)."""
    x = normal(seed, "x", (64, 256), bf16=False)
    cols = np.sort(_rng(seed, "x.outliers").choice(256, size=4, replace=False))
    x[:, cols] *= np.float32(50.0)
    return {
        "x": x, "x_dtype": "f32",
        "w": normal(seed, "w", (128, 256), 0.02, bf16=False), "w_dtype": "f32",
        "l1": normal(seed, "l1", (256, 8), 0.01), "l2": normal(seed, "l2", (8, 128), 0.01),
        "outlier_cols": cols,
    }


# --------------------------------------------------------------------------
# Workload 2: per-channel weight-format choice + MXFP8 activations.
# --------------------------------------------------------------------------
def chameleon_selection(seed: int = 2, n: int = 3072, k: int = 3072, m: int = 4096):
    """W n x k bf16 Student-t(nu=4) scaled to std 0.02 (t4 has std sqrt(2));
    X m x k bf16 Student-t(nu=3), unscaled."""
    return {
        "w": student_t(seed, "w", (n, k), 4.0, 0.02 / np.sqrt(2.0)), "w_dtype": "bf16",
        "x": student_t(seed, "x", (m, k), 3.0), "x_dtype": "bf16",
    }


# --------------------------------------------------------------------------
# Workload 3: SVDQuant W4A4 DiT MLP up-projection (NVFP4 and INT4-g64).
# --------------------------------------------------------------------------
def svdquant_mlp_up(seed: int = 3, m: int = 4096, k: int = 3072, n: int = 12288, rank: int = 32,
                    draw_weights: bool = True):
    """X m x k bf16 N(0,1) with 1% of the columns scaled by log-uniform
    [20, 100]; residual weight R n x k bf16 N(0, 0.02^2); L1 k x rank and
    L2 rank x n bf16 N(0, 0.05^2)."""
    x = normal(seed, "x", (m, k), bf16=False)
    cols, f = outlier_columns(seed, "x.outliers", k, max(1, k // 100), 20.0, 100.0)
    x[:, cols] *= f[None, :]
    out = {"x": to_bf16_values(x), "x_dtype": "bf16", "outlier_cols": cols,
           "l1": normal(seed, "l1", (k, rank), 0.05), "l2": normal(seed, "l2", (rank, n), 0.05)}
    if draw_weights:
        out["w"] = normal(seed, "w", (n, k), 0.02)
        out["w_dtype"] = "bf16"
    return out


# --------------------------------------------------------------------------
# Workload 4: MXFP4 GEMM with block-diagonal Hadamard rotation (b = 128).
# --------------------------------------------------------------------------
def mxfp4_hadamard_gemm(seed: int = 4, m: int = 8192, k: int = 4096, n: int = 4096):
    """X m x k bf16 Laplace(0, 1); W n x k bf16 N(0, 0.02^2)."""
    return {
        "x": laplace(seed, "x", (m, k)), "x_dtype": "bf16",
        "w": normal(seed, "w", (n, k), 0.02), "w_dtype": "bf16",
    }


# --------------------------------------------------------------------------
# Workload 5: timestep-routed mixed-format DiT stack.
# --------------------------------------------------------------------------
DIT_HIDDEN, DIT_MLP, DIT_BLOCKS, DIT_TOKENS = 1152, 4608, 28, 8192
DIT_STEPS, DIT_INTERVALS = 20, 10
# (name, in_features, out_features) of the four linears of one block.
DIT_LINEARS = (("qkv", DIT_HIDDEN, 3 * DIT_HIDDEN), ("proj", DIT_HIDDEN, DIT_HIDDEN),
               ("fc1", DIT_HIDDEN, DIT_MLP), ("fc2", DIT_MLP, DIT_HIDDEN))


def dit_tail_nu(step: int, n_steps: int = DIT_STEPS) -> float:
    """Student-t tail index: 2 at step 0 rising linearly to 30 at the last step."""
    return 2.0 + 28.0 * step / (n_steps - 1)


def dit_format_table(seed: int = 5, formats=(5, 6, 0), forced_value: int = 0, n_forced: int = 4):
    """Seeded table[layer][interval] over `formats` (default INT8 per-token,
    FP8 per-tensor, MXFP8 by id), with `n_forced` seeded layers pinned to
    `forced_value` (MXFP8) in every interval.  Returns (table, forced_layers)."""
    n_layers = DIT_BLOCKS * len(DIT_LINEARS)
    g = _rng(seed, "table")
    table = np.asarray(formats, dtype=np.uint8)[g.integers(0, len(formats), size=(n_layers, DIT_INTERVALS))]
    forced = np.sort(g.choice(n_layers, size=n_forced, replace=False))
    table[forced, :] = forced_value
    return np.ascontiguousarray(table), forced


def dit_activation(seed: int, step: int, in_features: int, m: int = DIT_TOKENS):
    """Fresh bf16 activation for one step (shared by the 28 blocks)."""
    return student_t(seed, "act.%d.%d" % (step, in_features), (m, in_features), dit_tail_nu(step))


def dit_forced_column_factors(seed: int, layer: int, in_features: int):
    """Per-column factors log-uniform in [1, 163], the largest pinned at 163."""
    g = _rng(seed, "forced.%d" % layer)
    f = np.exp(g.uniform(0.0, np.log(163.0), size=in_features))
    f[g.integers(0, in_features)] = 163.0
    return f.astype(np.float32)


def dit_weight(seed: int, layer: int, in_features: int, out_features: int):
    return normal(seed, "w.%d" % layer, (out_features, in_features), 0.02)


def dit_layer_shape(layer: int):
    """(in_features, out_features) of stack layer `layer` (4 linears per block)."""
    _, kin, nout = DIT_LINEARS[layer % len(DIT_LINEARS)]
    return kin, nout


def dit_layer_input(seed: int, step: int, layer: int, forced, m: int = DIT_TOKENS):
    """Input of stack layer `layer` at `step`: the step's shared activation of
    that width, and for a forced layer its columns times the layer's factors
    (log-uniform in [1, 163]), rounded once more to bf16."""
    kin, _ = dit_layer_shape(layer)
    x = dit_activation(seed, step, kin, m)
    if layer in set(int(f) for f in forced):
        x = to_bf16_values(x * dit_forced_column_factors(seed, layer, kin)[None, :])
    return x
