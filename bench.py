#!/usr/bin/env python
"""Benchmark of the W4A4 quantized linear layer (SVDQuant MLP up-projection,
NVFP4, rank-32 low-rank branch): X 4096 x 3072 bf16, residual weight
12288 x 3072, L1 3072 x 32, L2 32 x 12288, output bf16.

One step is one inference pass of the layer's hot path on one batch:
  tensor amax of X -> NVFP4 quantization of X (MMA layout) -> low-rank down
  projection T = bf16(X) . L1 -> packing of T for the GEMM -> tcgen05
  block-scaled GEMM with the fused epilogue and low-rank up projection.
The weight (quantized to NVFP4, L2 packed) is prepared once, before timing,
as a deployed layer's weights are.

Contract: `python bench.py --gpus N --steps K --warmup W` prints one JSON line
on rank 0.  N > 1 runs under torchrun, one process per GPU; each rank runs the
same layer on its own batch (data parallel over tokens, no collective on the
data path: weak scaling); the timed region is bracketed by a barrier and a
device synchronize, and the time is the max over ranks.  Inputs and outputs
rotate over 4 device-resident sets (about 620 MB > 126 MB L2), so every step
reads its operands from HBM.  The timed steps replay CUDA graphs of 20
consecutive steps (and of the K mod 20 left), captured before timing: the
host issues one launch per 20 steps instead of two Python API calls per step,
whose cost (~40-90 us per step through ctypes) would otherwise pace the
device, and the programmatic edges between kernels hold across steps.  The
same steps launched eagerly are timed after (`ms_per_step_eager`), and the
end-to-end leg stays eager.

After the timed steps the same process measures, on the same stream: the
dominant kernel (the GEMM) and the activation side by CUDA-graph replay of
100 launches each; every bandwidth-bound row with a 256 MiB read of another
buffer before each launch (L2 holds nothing of its inputs) and CUDA events
around the launch; the other workloads' GEMMs (MXFP4 with and without the
128-wide rotation, the timestep-routed W8A8 stack, the tiny NVFP4 layer's
latency) and the remaining kernels; the oracle on the host cores.

`--impl reference` times the CPU oracle (oracle/, plain C + numpy binary64
GEMM) on the host cores on a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

M, K, N, RANK = 4096, 3072, 12288, 32
FLOP_MAIN = 2 * M * N * K                       # 309,237,645,312
FLOP_LR_UP = 2 * M * N * RANK                   # inside the GEMM kernel
FLOP_LR_DOWN = 2 * M * K * RANK
FLOP_STEP = FLOP_MAIN + FLOP_LR_UP + FLOP_LR_DOWN
N_SETS = 4
WORKLOAD = "svdquant_mlp_up_nvfp4_w4a4_lowrank32"
FLUSH_BYTES = 256 << 20                         # > 2 x the 126 MB L2


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "src": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except Exception:
            self.proc = None

    def wait_ready(self, samples=3, limit_s=20.0):
        """Returns once the sampler has produced a few lines (nvidia-smi start-up
        is kept out of the timed region)."""
        t0 = time.time()
        while self.proc is not None and len(self.lines) < samples and time.time() - t0 < limit_s:
            time.sleep(0.05)
        self.skip = len(self.lines)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.08)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in self.lines[getattr(self, "skip", 0):]:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def _dist_init():
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def _max_over_ranks(value, world):
    """Max of a per-rank scalar over all ranks (the job's time is its slowest rank)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(ms_local, world, flop_per_rank):
    """(max ms over ranks, whole-job TFLOP/s): every rank runs the same layer on
    its own batch, so the job does world * flop_per_rank per step."""
    ms = _max_over_ranks(ms_local, world)
    return ms, world * flop_per_rank / (ms * 1e-3) / 1e12


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ oracle

class OracleSample:
    """The oracle as it stands, on a bounded sample of the workload per step:
    `rows` token rows of X against the first `cols` output channels of the
    weight -- NVFP4 quantization (C), low-rank down projection (C), binary64
    GEMM over exactly dequantized operands (numpy matmul), which dequantizes
    its weight slice on every call."""

    def __init__(self, rows=64, cols=N):
        import oracle
        import workloads
        d = workloads.svdquant_mlp_up()
        self.rows, self.cols = rows, cols
        self.x = d["x"][:rows].copy()
        self.l1, self.l2 = d["l1"], d["l2"][:, :cols].copy()
        self.wq = oracle.quantize(d["w"][:cols].copy(), oracle.NVFP4)
        self.flops = 2 * rows * cols * K + 2 * rows * cols * RANK + 2 * rows * K * RANK
        self.desc = ("%d of %d token rows x %d of %d output channels per step: NVFP4 quantize, low-rank down "
                     "projection, binary64 GEMM over exactly dequantized operands (incl. dequantizing the "
                     "%d x %d weight slice)" % (rows, M, cols, N, cols, K))

    def step(self):
        import oracle
        xq = oracle.quantize(self.x, oracle.NVFP4)
        t = oracle.lowrank_down(self.x, self.l1)
        return oracle.qlinear(xq, self.wq, t, self.l2)

    def timed(self, steps, threads=1):
        from threadpoolctl import threadpool_limits
        with threadpool_limits(threads):
            t0 = time.perf_counter()
            for _ in range(steps):
                self.step()
            return (time.perf_counter() - t0) / steps


def host_cores():
    return len(os.sched_getaffinity(0))


def oracle_bandwidth_rows():
    """The oracle's quantize and selection at workload 2's full sizes, in GB/s
    of the same algorithmic bytes as the GPU rows: MXFP8 quantization of X
    (4096 x 3072) on one thread and on all host cores (row ranges on threads;
    MX blocks are independent, so the codes are the same), and the per-channel
    selection of W (3072 x 3072) over INT4-g32, NVFP4, MXFP4 on one thread
    (its NVFP4 candidate needs the tensor scale of the whole W)."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    import workloads
    d = workloads.chameleon_selection()
    x, w = d["x"], d["w"]
    n = host_cores()
    qbytes = x.size * 2 + x.size + x.size // 32

    def q_rows(i, parts):
        r0, r1 = i * x.shape[0] // parts, (i + 1) * x.shape[0] // parts
        return oracle.quantize(x[r0:r1], oracle.MXFP8)

    t0 = time.perf_counter()
    oracle.quantize(x, oracle.MXFP8)
    t_one = time.perf_counter() - t0
    with ThreadPoolExecutor(n) as ex:
        list(ex.map(lambda i: q_rows(i, n), range(n)))      # warm the pool
        t0 = time.perf_counter()
        list(ex.map(lambda i: q_rows(i, n), range(n)))
        t_all = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.select_weight_format(w, [oracle.INT4_G32, oracle.NVFP4, oracle.MXFP4])
    t_sel = time.perf_counter() - t0
    sbytes = w.size * 2 + w.shape[0]
    return {
        "quantize_mxfp8_x_4096x3072": {"single_thread_GB/s": qbytes / t_one / 1e9, "all_cores_GB/s": qbytes / t_all / 1e9,
                                       "cores": n, "seconds_single": t_one, "seconds_all": t_all},
        "select_w_3072x3072": {"single_thread_GB/s": sbytes / t_sel / 1e9, "seconds_single": t_sel, "cores": 1},
    }


def run_reference(args, world, rank):
    if rank != 0:
        return
    o = OracleSample(rows=8, cols=512)   # ~40 ms per step: --steps in the thousands still ends in minutes
    o.timed(args.warmup)
    sec = o.timed(args.steps)
    value = o.flops / sec / 1e12
    line = {"impl": "reference", "metric": "qlinear TFLOPS (NVFP4 W4A4 + rank-32 low-rank), whole step",
            "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sec, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "m": M, "k": K, "n": N, "rank": RANK, "sample_rows": o.rows,
                       "sample_cols": o.cols},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                             "sample": o.desc + "; 1 thread"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm

class Timer:
    """Device timing on the launching stream.

    graph_ms: CUDA-graph replay of `n` calls (rotating their own inputs),
      `reps` replays; mean time per call -- the steady state of back-to-back
      launches, whose setup overlaps the previous kernel as in the step.
    flushed_ms: CUDA events around each call, after a 256 MiB read of another
      buffer (so L2 holds none of the call's inputs); median of `n` calls."""

    def __init__(self, torch, dev, stream):
        self.torch, self.dev, self.stream = torch, dev, stream
        self.flush_buf = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.flush_buf.fill_(1.0)
        self.flush_out = torch.empty((), dtype=torch.float32, device=dev)

    def flush(self):
        self.torch.sum(self.flush_buf, dim=0, dtype=self.torch.float32, out=self.flush_out)

    def graph_ms(self, fn, n=20, reps=5):
        torch = self.torch
        side = torch.cuda.Stream(device=self.dev)
        side.wait_stream(self.stream)
        with torch.cuda.stream(side):
            fn(0)
        self.stream.wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            for i in range(n):
                fn(i)
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(self.stream)
        for _ in range(reps):
            g.replay()
        b.record(self.stream)
        torch.cuda.synchronize()
        del g
        return a.elapsed_time(b) / (reps * n)

    def flushed_ms(self, fn, n=20, warm=3):
        torch = self.torch
        for i in range(warm):
            self.flush()
            fn(i)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for i, (a, b) in enumerate(evs):
            self.flush()
            a.record(self.stream)
            fn(i)
            b.record(self.stream)
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in evs)


def _hbm_row(kernel, ms, nbytes, peaks, **extra):
    gbs = nbytes / (ms * 1e-3) / 1e9
    row = {"kernel": kernel, "us": 1e3 * ms, "bytes": nbytes, "GB/s": gbs, "frac": gbs / peaks["hbm_gbs"]}
    row.update(extra)
    return row


def quantize_rows(mxq, torch, dev, timer, peaks, inputs):
    """Every quantize format alone on each named input (MMA layout), L2 flushed
    before each launch.  Bytes: read 2 B per element + canonical codes and
    scales written."""
    out = {}
    qws = torch.empty(mxq.quantize_workspace_bytes(mxq.NVFP4), dtype=torch.uint8, device=dev)
    for label, x in inputs:
        rows, cols = x.shape
        for name, fmt, had in (("NVFP4", mxq.NVFP4, 0), ("MXFP4", mxq.MXFP4, 0), ("MXFP4+hadamard128", mxq.MXFP4, 128),
                               ("MXFP8", mxq.MXFP8, 0), ("INT4_G64", mxq.INT4_G64, 0), ("INT8_ROW", mxq.INT8_ROW, 0),
                               ("FP8_TENSOR", mxq.FP8_TENSOR, 0)):
            q = mxq.alloc_qtensor(fmt, rows, cols, mxq.MMA, dev)
            t_ms = timer.flushed_ms(lambda i: mxq.quantize(x, fmt, had, mxq.MMA, out=q, workspace=qws))
            nbytes = (rows * cols * 2 + mxq.codes_bytes(fmt, rows, cols, mxq.CANONICAL)
                      + mxq.scales_bytes(fmt, rows, cols, mxq.CANONICAL))
            launches = 2 if fmt in (mxq.NVFP4, mxq.FP8_TENSOR) else 1
            out["%s %s" % (label, name)] = _hbm_row("k_quantize (%d launch%s)" % (launches, "es" if launches > 1 else ""),
                                                    t_ms, nbytes, peaks)
            del q
    return out


def routed_stack_row(mxq, torch, dev, timer, peaks):
    """Workload 5: 28 DiT blocks x 4 linears (qkv 1152->3456, proj 1152->1152,
    fc1 1152->4608, fc2 4608->1152), M = 8192 tokens, 20 denoising steps in 10
    intervals, the seeded format table over INT8 per token, FP8 per tensor and
    MXFP8 with 4 layers forced to MXFP8.  Each layer call is one
    mxq_qlinear_routed (table read, activation quantized in the routed format,
    GEMM against the weight prepared in that format).  Every step's calls are
    captured in a CUDA graph (the table is read at capture); the 20 graphs are
    replayed in order.  Inputs: per step fresh Student-t(nu(step)) activations
    of widths 1152 and 4608 shared by the blocks, forced layers' columns times
    log-uniform [1, 163] factors, weights N(0, 0.02^2) -- drawn on the device
    with torch's seeded generator (the parity tests use the workloads module's
    host draws of the same distributions)."""
    import workloads
    table, forced = workloads.dit_format_table(5)
    n_layers = table.shape[0]
    steps = workloads.DIT_STEPS
    Mt = workloads.DIT_TOKENS
    g = torch.Generator(device=dev)
    g.manual_seed(5)
    bf = torch.bfloat16

    def student_t(nu, shape):
        # t = z / sqrt(chi2_nu / nu), chi2_nu = 2 * Gamma(nu / 2, 1)
        z = torch.randn(shape, generator=g, device=dev)
        gam = torch._standard_gamma(torch.full(shape, nu / 2.0, device=dev), generator=g)
        return z / torch.sqrt(2.0 * gam / nu)

    layers = []
    for layer in range(n_layers):
        kin, nout = workloads.dit_layer_shape(layer)
        w = (torch.randn((nout, kin), generator=g, device=dev) * 0.02).to(bf)
        layers.append(mxq.prepare_routed_layer(w, set(table[layer].tolist())))
        del w
    forced_f = {}
    for layer in forced.tolist():
        kin, _ = workloads.dit_layer_shape(layer)
        f = torch.exp(torch.rand(kin, generator=g, device=dev) * float(torch.log(torch.tensor(163.0))))
        f[int(torch.randint(0, kin, (1,), generator=g, device=dev))] = 163.0
        forced_f[layer] = f
    inputs = []
    for step in range(steps):
        nu = workloads.dit_tail_nu(step)
        xs = {kin: student_t(nu, (Mt, kin)).to(bf) for kin in (workloads.DIT_HIDDEN, workloads.DIT_MLP)}
        for layer, f in forced_f.items():
            kin, _ = workloads.dit_layer_shape(layer)
            xs[("forced", layer)] = (xs[kin].float() * f[None, :]).to(bf)
        inputs.append(xs)
    ys = {nout: torch.empty((Mt, nout), dtype=bf, device=dev) for nout in {3456, 1152, 4608}}
    ws = torch.empty(mxq.qlinear_routed_workspace_bytes(Mt, workloads.DIT_MLP, 0), dtype=torch.uint8, device=dev)

    def call(layer, step):
        kin, nout = workloads.dit_layer_shape(layer)
        xs = inputs[step]
        x = xs[("forced", layer)] if ("forced", layer) in xs else xs[kin]
        mxq.qlinear_routed(x, layers[layer], table, layer, step, steps, out=ys[nout], workspace=ws)

    flops = {0: 0, 5: 0, 6: 0}
    calls = {0: [], 5: [], 6: []}
    for step in range(steps):
        for layer in range(n_layers):
            kin, nout = workloads.dit_layer_shape(layer)
            fmt = int(table[layer, step * table.shape[1] // steps])
            flops[fmt] += 2 * Mt * nout * kin
            calls[fmt].append((layer, step))

    def capture(pairs):
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(timer.stream)
        with torch.cuda.stream(side):
            for layer, step in pairs[:2]:
                call(layer, step)
        timer.stream.wait_stream(side)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, capture_error_mode="thread_local"):
            for layer, step in pairs:
                call(layer, step)
        return gr

    def time_graphs(graphs, reps=3):
        for gr in graphs:
            gr.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(timer.stream)
        for _ in range(reps):
            for gr in graphs:
                gr.replay()
        b.record(timer.stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    step_graphs = [capture([(layer, step) for layer in range(n_layers)]) for step in range(steps)]
    pass_ms = time_graphs(step_graphs)
    del step_graphs
    fp8_peak = 2.0 * peaks["bf16_tflops"]
    split = {}
    names = {5: "INT8_ROW", 6: "FP8_TENSOR", 0: "MXFP8"}
    for fmt, pairs in calls.items():
        gr = capture(pairs)
        f_ms = time_graphs([gr])
        del gr
        tf = flops[fmt] / (f_ms * 1e-3) / 1e12
        split[names[fmt]] = {"layer_calls": len(pairs), "ms": f_ms, "flop": flops[fmt], "TFLOP/s": tf,
                             "frac_of_fp8_int8_peak": tf / fp8_peak}
    total_flop = sum(flops.values())
    assert mxq.check() == 0
    return {"workload": "routed W8A8 DiT stack: 28 blocks x 4 linears, M 8192, hidden 1152, MLP 4608, 20 steps, "
                        "10 intervals, formats {INT8 per token, FP8 per tensor, MXFP8}, 4 forced MXFP8 layers",
            "pass_ms_20_steps": pass_ms, "ms_per_step": pass_ms / steps, "flop_per_pass": total_flop,
            "TFLOP/s": total_flop / (pass_ms * 1e-3) / 1e12,
            "frac_of_fp8_int8_peak": total_flop / (pass_ms * 1e-3) / 1e12 / fp8_peak, "fp8_int8_peak": fp8_peak,
            "per_format": split,
            "launches_per_layer_call": "2 (k_quantize or k_quantize_int8_row, k_gemm) + 1 for FP8 per tensor "
                                       "(amax pass)"}


def run_ours(args, world, rank, local):
    import numpy as np  # noqa: F401
    import torch

    import microscaling_bit_quantization_b200 as mxq
    import workloads
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if mxq.lib().mxq_device_supported(local) != 1:
        raise RuntimeError("this benchmark needs an sm_100 GPU")
    stream = torch.cuda.current_stream()

    d = workloads.svdquant_mlp_up()
    x_host = torch.from_numpy(d["x"]).to(torch.bfloat16)
    w = torch.from_numpy(d["w"]).to(torch.bfloat16).to(dev)
    l1 = torch.from_numpy(d["l1"]).to(torch.bfloat16).to(dev)
    l2 = torch.from_numpy(d["l2"]).to(torch.bfloat16).to(dev)
    del d

    # Offline weight preparation (once): NVFP4 codes + scales, packed L2.
    wq0 = mxq.quantize(w, mxq.NVFP4, 0, mxq.MMA)
    l2p = mxq.lowrank_pack_l2(l2)
    sets = []
    for i in range(N_SETS):
        wq = mxq.alloc_qtensor(mxq.NVFP4, N, K, mxq.MMA, dev)
        wq.codes.copy_(wq0.codes)
        wq.scales.copy_(wq0.scales)
        wq.tensor_scale.copy_(wq0.tensor_scale)
        s = {"x": x_host.to(dev), "wq": wq, "l2p": l2p.clone(),
             "xq": mxq.alloc_qtensor(mxq.NVFP4, M, K, mxq.MMA, dev),
             "tp": torch.empty((M, 64), dtype=torch.bfloat16, device=dev),
             "qws": torch.empty(mxq.quantize_lowrank_workspace_bytes(M, RANK), dtype=torch.uint8, device=dev),
             "y": torch.empty((M, N), dtype=torch.bfloat16, device=dev)}
        sets.append(s)
    del wq0

    def quant(i):
        s = sets[i % N_SETS]
        mxq.quantize_lowrank(s["x"], mxq.NVFP4, l1, s["wq"], 0, out=s["xq"], tp=s["tp"], workspace=s["qws"])

    def gemm(i):
        s = sets[i % N_SETS]
        mxq.qlinear(s["xq"], s["wq"], s["tp"], s["l2p"], out=s["y"])

    def step(i):
        quant(i)
        gemm(i)

    launches_per_step = 3      # k_lowrank_tc (T + tensor amax), k_quantize (codes, scales, packed T), k_gemm

    for i in range(max(args.warmup, N_SETS)):   # every input set has been through the path once
        step(i)
    torch.cuda.synchronize()
    assert mxq.check() == 0

    # Consecutive steps are captured once as CUDA graphs (each step's three kernels and the
    # programmatic edges between all of them, across steps too): a graph of G = 20 steps (five
    # rounds of the rotating sets) and one of the K mod G left over; the timed region replays the
    # first K // G times and the second once -- exactly K steps, one host launch per 20, so the
    # number is the device's, not the Python submission's.  The same steps launched eagerly are
    # timed after, for reference (ms_per_step_eager).
    G = 20 if args.steps >= 20 else max(args.steps, 1)
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for i in range(N_SETS):
            step(i)
    stream.wait_stream(side)
    torch.cuda.synchronize()

    def capture(n):   # thread_local: under torchrun the NCCL watchdog thread may query events meanwhile
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            for i in range(n):
                step(i)
        return g

    g_full = capture(G)
    rem = args.steps % G
    g_rem = capture(rem) if rem else None
    g_full.replay()
    if g_rem is not None:
        g_rem.replay()
    torch.cuda.synchronize()
    assert mxq.check() == 0

    # ---- timed region: exactly K steps between a pair of events on the launching stream
    sampler = ClockSampler(local)
    sampler.start()
    sampler.wait_ready()
    _barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(args.steps // G):
        g_full.replay()   # steps i .. i + G - 1 use the sets in the same rotation (G % N_SETS == 0)
    if g_rem is not None:
        g_rem.replay()
    end.record(stream)
    torch.cuda.synchronize()
    _barrier(world)
    clocks = sampler.stop()
    ms_local = start.elapsed_time(end) / args.steps
    ms, value = job_throughput(ms_local, world, FLOP_STEP)
    assert mxq.check() == 0
    del g_full, g_rem

    # the same K steps launched eagerly through the Python API (two calls per step)
    _barrier(world)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(args.steps):
        step(i)
    end.record(stream)
    torch.cuda.synchronize()
    args.ms_eager = _max_over_ranks(start.elapsed_time(end) / args.steps, world)
    assert mxq.check() == 0

    peaks = _peaks()
    fp4_peak = peaks["bf16_tflops"] * 4.0          # nominal dense FP4 : BF16 ratio 9 : 2.25
    int8_peak = peaks["bf16_tflops"] * 2.0         # nominal dense INT8/FP8 : BF16 ratio 4.5 : 2.25
    timer = Timer(torch, dev, stream)

    # ---- the dominant kernel and the activation side, right after the timed region, on the same
    # stream: CUDA-graph replay of 20 launches over the rotating sets, 5 replays (100 launches each)
    gemm_ms = timer.graph_ms(gemm, n=20, reps=5)
    quant_ms = timer.graph_ms(quant, n=20, reps=5)
    gemm_flops = FLOP_MAIN + FLOP_LR_UP
    gemm_tflops = gemm_flops / (gemm_ms * 1e-3) / 1e12
    # algorithmic bytes of the activation side: read bf16 X once, write codes, scales, packed T
    quant_bytes = M * K * 2 + M * K // 2 + (M * K // 16) + M * 64 * 2
    quant_gbs = quant_bytes / (quant_ms * 1e-3) / 1e9
    profiles_traffic = None
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            profiles_traffic = json.load(f).get("k_gemm_nvfp4")
    except Exception:
        pass

    rows = {}
    if args.rows == "none":   # the contract line only (e.g. under a profiler)
        return finish(args, world, rank, ms, value, clocks, gemm_tflops, fp4_peak, peaks, profiles_traffic, gemm_ms,
                      gemm_flops, rows, stream, sets, step, x_host, launches_per_step, torch, mxq)
    rows["activation_side"] = {"kernel": "k_lowrank_tc (T + tensor amax) + k_quantize<NVFP4> (codes, scales, "
                                         "packed T), X 4096 x 3072 bf16, graph replay of 100 launches",
                               "us": 1e3 * quant_ms, "bytes": quant_bytes, "GB/s": quant_gbs,
                               "frac": quant_gbs / peaks["hbm_gbs"]}
    rows["activation_side_flushed"] = _hbm_row("the same two kernels, L2 flushed before each call",
                                               timer.flushed_ms(quant), quant_bytes, peaks)

    # ---- quantize alone: workload 3's X (25 MB) and workload 4's X (67 MB), L2 flushed
    w4 = workloads.mxfp4_hadamard_gemm()
    x4 = torch.from_numpy(w4["x"]).to(torch.bfloat16).to(dev)
    w4d = torch.from_numpy(w4["w"]).to(torch.bfloat16).to(dev)
    del w4
    rows["quantize"] = quantize_rows(mxq, torch, dev, timer, peaks,
                                     (("X 4096x3072", sets[0]["x"]), ("X 8192x4096", x4)))

    # ---- workload 2: per-channel selection of W and MXFP8 quantization of X (Student-t), L2 flushed
    w2 = workloads.chameleon_selection()
    wsel = torch.from_numpy(w2["w"]).to(torch.bfloat16).to(dev)
    x2 = torch.from_numpy(w2["x"]).to(torch.bfloat16).to(dev)
    del w2
    cands = (mxq.INT4_G32, mxq.NVFP4, mxq.MXFP4)
    sel_ms = timer.flushed_ms(lambda i: mxq.select_weight_format(wsel, cands, want_sse=False))
    rows["select_weight_format"] = _hbm_row("k_quantize amax pass + k_select over INT4-g32, NVFP4, MXFP4, "
                                            "W 3072 x 3072 bf16", sel_ms, wsel.numel() * 2 + wsel.shape[0], peaks)
    q2 = mxq.alloc_qtensor(mxq.MXFP8, *x2.shape, mxq.MMA, dev)
    x2_ms = timer.flushed_ms(lambda i: mxq.quantize(x2, mxq.MXFP8, 0, mxq.MMA, out=q2))
    rows["quantize_mxfp8_workload2_x"] = _hbm_row("k_quantize<MXFP8>, X 4096 x 3072 bf16 Student-t(3)", x2_ms,
                                                  x2.numel() * (2 + 1) + x2.numel() // 32, peaks)
    # the per-channel mixed-format linear layer on the selection's choices: X (MXFP8) . W^T
    choice, _ = mxq.select_weight_format(wsel, cands, want_sse=False)
    mw = mxq.prepare_mixed_weight(wsel, choice)
    y2 = torch.empty((x2.shape[0], wsel.shape[0]), dtype=torch.bfloat16, device=dev)
    ws2 = torch.empty(mxq.qlinear_mixed_workspace_bytes(x2.shape[0], mw), dtype=torch.uint8, device=dev)
    mix_ms = timer.graph_ms(lambda i: mxq.qlinear_mixed(q2, mw, out=y2, workspace=ws2), n=10, reps=5)
    mix_step_ms = timer.graph_ms(lambda i: (mxq.quantize(x2, mxq.MXFP8, 0, mxq.MMA, out=q2),
                                            mxq.qlinear_mixed(q2, mw, out=y2, workspace=ws2)), n=10, reps=5)
    f2 = 2 * x2.shape[0] * wsel.shape[0] * wsel.shape[1]
    rows["mixed_format_linear_workload2"] = {
        "kernels": "k_gemm<MXFP8> on the MXFP4 rows (E4M3 bytes), k_gemm_igroup<32> on the INT4-g32 rows, "
                   "k_gemm<bf16> on the NVFP4 rows (x dequantized to bf16), scale conversion, dequantize, scatter",
        "channels_mxfp4_int4g32_nvfp4": list(mw.n_group), "us": 1e3 * mix_ms,
        "TFLOP/s": f2 / (mix_ms * 1e-3) / 1e12, "frac_of_fp8_peak": f2 / (mix_ms * 1e-3) / 1e12 / int8_peak,
        "with_mxfp8_quantize_us": 1e3 * mix_step_ms}
    del q2, x2, mw, y2, ws2

    # ---- workload 4: MXFP4 GEMM 8192 x 4096 x 4096, without and with the 128-wide rotation
    f4 = 2 * 8192 * 4096 * 4096
    for had in (0, 128):
        wq4 = mxq.quantize(w4d, mxq.MXFP4, had, mxq.MMA)
        xq4 = [mxq.alloc_qtensor(mxq.MXFP4, 8192, 4096, mxq.MMA, dev) for _ in range(2)]
        y4 = torch.empty((8192, 4096), dtype=torch.bfloat16, device=dev)
        for q in xq4:
            mxq.quantize(x4, mxq.MXFP4, had, mxq.MMA, out=q)
        g_ms = timer.graph_ms(lambda i: mxq.qlinear(xq4[i % 2], wq4, out=y4), n=20, reps=5)
        s_ms = timer.graph_ms(lambda i: (mxq.quantize(x4, mxq.MXFP4, had, mxq.MMA, out=xq4[i % 2]),
                                         mxq.qlinear(xq4[i % 2], wq4, out=y4)), n=10, reps=5)
        rows["mxfp4_gemm_8192x4096x4096_h%d" % had] = {
            "kernel": "k_gemm<MXFP4> (bf16 out)", "gemm_us": 1e3 * g_ms, "TFLOP/s": f4 / (g_ms * 1e-3) / 1e12,
            "frac_of_fp4_peak": f4 / (g_ms * 1e-3) / 1e12 / fp4_peak,
            "step_us (quantize X%s + GEMM)" % (" with the rotation" if had else ""): 1e3 * s_ms,
            "step_TFLOP/s": f4 / (s_ms * 1e-3) / 1e12}
        del wq4, xq4, y4
    del x4

    # ---- workload 5: the routed W8A8 stack
    rows["routed_stack"] = routed_stack_row(mxq, torch, dev, timer, peaks)
    torch.cuda.empty_cache()

    # ---- workload 1: latency of the tiny NVFP4 W4A4 + rank-8 layer (fp32 X 64 x 256, W 128 x 256)
    d1 = workloads.tiny_nvfp4_linear()
    x1 = torch.from_numpy(d1["x"]).to(dev)
    wq1 = mxq.quantize(torch.from_numpy(d1["w"]).to(dev), mxq.NVFP4, 0, mxq.MMA)
    l1_1 = torch.from_numpy(d1["l1"]).to(torch.bfloat16).to(dev)
    l2p1 = mxq.lowrank_pack_l2(torch.from_numpy(d1["l2"]).to(torch.bfloat16).to(dev))
    xq1 = mxq.alloc_qtensor(mxq.NVFP4, 64, 256, mxq.MMA, dev)
    tp1 = torch.empty((64, 64), dtype=torch.bfloat16, device=dev)
    ws1 = torch.empty(mxq.quantize_lowrank_workspace_bytes(64, 8), dtype=torch.uint8, device=dev)
    y1 = torch.empty((64, 128), dtype=torch.float32, device=dev)

    def tiny(i):
        mxq.quantize_lowrank(x1, mxq.NVFP4, l1_1, wq1, 0, out=xq1, tp=tp1, workspace=ws1)
        mxq.qlinear(xq1, wq1, tp1, l2p1, out=y1)

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(50)]
    for i in range(5):
        tiny(i)
    torch.cuda.synchronize()
    for a, b in evs:
        a.record(stream)
        tiny(0)
        b.record(stream)
        torch.cuda.synchronize()
    rows["tiny_nvfp4_latency"] = {
        "workload": "X 64 x 256 fp32, W 128 x 256, NVFP4, rank 8, fp32 out: k_lowrank (fp32 X, per-CTA amax "
                    "slots) + k_quantize + k_gemm",
        "eager_us_median_of_50": 1e3 * statistics.median(a.elapsed_time(b) for a, b in evs),
        "graph_replay_us": 1e3 * timer.graph_ms(tiny, n=20, reps=5)}
    del x1, wq1, xq1, tp1, ws1, y1

    # ---- the other kernels of the library, alone (graph replay; the two fits and calibration are ALU-bound)
    t_buf = torch.empty((M, RANK), dtype=torch.float32, device=dev)
    lr_ms = timer.flushed_ms(lambda i: mxq.lowrank_down(sets[i % N_SETS]["x"], l1, out=t_buf))
    rows["lowrank_down"] = _hbm_row("k_lowrank_tc (T = bf16(X) L1 alone), X 4096 x 3072 bf16, rank 32, L2 flushed",
                                    lr_ms, M * K * 2 + M * RANK * 4, peaks)
    del t_buf
    mse_ws = torch.empty(mxq.quantize_mse_workspace_bytes(N, K), dtype=torch.uint8, device=dev)
    mse_q = mxq.alloc_qtensor(mxq.NVFP4, N, K, mxq.MMA, dev)
    mse_ms = timer.graph_ms(lambda i: mxq.quantize_mse(w, 2, mxq.MMA, out=mse_q, workspace=mse_ws, want_sse=False),
                            n=2, reps=3)
    _, mse_sse = mxq.quantize_mse(w, 2, mxq.MMA, out=mse_q, workspace=mse_ws)
    usual_sse = ((mxq.dequantize(mxq.quantize(w, mxq.NVFP4), torch.float32).double() - w.double()) ** 2).sum().item()
    rows["quantize_mse_nvfp4"] = _hbm_row("k_mse_block (8 scale candidates per block, binary64 errors) x 3 passes + "
                                          "amax and ordered sums, R 12288 x 3072 bf16, 2 rounds", mse_ms,
                                          N * K * 2 + N * K // 2 + N * K // 16, peaks,
                                          sse_vs_usual_nvfp4=mse_sse.item() / usual_sse)
    del mse_ws, mse_q
    grid = [1.0, 1.0625, 1.125, 1.25, 4.0 / 3.0, 1.5, 1.75, 2.0]
    g_ws = torch.empty(mxq.fit_mx_grid_workspace_bytes(*w4d.shape, len(grid)), dtype=torch.uint8, device=dev)
    g_sse = torch.empty(len(grid), dtype=torch.float64, device=dev)
    fit_ms = timer.graph_ms(lambda i: mxq.fit_mx_grid(w4d, mxq.MXFP4, grid, 128, workspace=g_ws, sse=g_sse), n=2,
                            reps=3)
    g_best, g_sse = mxq.fit_mx_grid(w4d, mxq.MXFP4, grid, 128, workspace=g_ws, sse=g_sse)
    rows["fit_mx_grid"] = _hbm_row("k_mx_grid_err (MXFP4, 8 grid scales, Hadamard 128, binary64 errors) + ordered "
                                   "sums, W 4096 x 4096 bf16", fit_ms, w4d.numel() * 2, peaks, best_grid_scale=g_best,
                                   sse_best_vs_ocp=g_sse.min().item() / g_sse[0].item())
    del g_ws, w4d
    xc = torch.from_numpy(workloads.dit_activation(5, 0, 1152)).to(torch.bfloat16).to(dev)
    calib = [mxq.INT8_ROW, mxq.FP8_TENSOR, mxq.MXFP8]
    c_ws = torch.empty(mxq.calibrate_workspace_bytes(*xc.shape, len(calib)), dtype=torch.uint8, device=dev)
    c_sse = torch.zeros(len(calib), dtype=torch.float64, device=dev)
    c_mom = torch.zeros(2, dtype=torch.float64, device=dev)
    cal_ms = timer.graph_ms(lambda i: mxq.calibrate_activation(xc, calib, c_sse, c_mom, workspace=c_ws), n=4, reps=3)
    rows["calibrate_activation"] = _hbm_row("k_select (3 candidates, per-row binary64 errors) + k_moments + ordered "
                                            "sums, X 8192 x 1152 bf16", cal_ms, xc.numel() * 2, peaks)
    del xc, c_ws
    wq16 = mxq.quantize(w, mxq.INT4_G64)
    y16 = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    w16_ws = torch.empty(mxq.qlinear_w4a16_workspace_bytes(M, N, K), dtype=torch.uint8, device=dev)
    w16_ms = timer.graph_ms(lambda i: mxq.qlinear_w4a16(sets[i % N_SETS]["x"], wq16, out=y16, workspace=w16_ws),
                            n=4, reps=3)
    w16_fused_ms = timer.graph_ms(lambda i: mxq.qlinear_w4a16(sets[i % N_SETS]["x"], wq16, out=y16, fused=True),
                                  n=4, reps=3)
    w16_tf = FLOP_MAIN / (w16_ms * 1e-3) / 1e12
    rows["w4a16_qlinear"] = {"kernel": "INT4-g64 weight unpacked once to bf16 (k_dequantize) + k_gemm<bf16> "
                                       "(kind::f16), X 4096 x 3072 bf16, W 12288 x 3072",
                             "us": 1e3 * w16_ms, "TFLOP/s": w16_tf, "frac_of_bf16_peak": w16_tf / peaks["bf16_tflops"],
                             "bf16_peak": peaks["bf16_tflops"],
                             "fused_kernel_us": 1e3 * w16_fused_ms,
                             "fused_kernel": "k_w4a16 (weights converted to bf16 in shared memory, never written)"}
    del wq16, y16, w16_ws
    wq4 = mxq.quantize(w, mxq.INT4_G64, 0, mxq.MMA)
    xq4 = mxq.quantize(sets[0]["x"], mxq.INT4_G64, 0, mxq.MMA)
    tp4 = mxq.lowrank_down_packed(sets[0]["x"], l1, xq4, wq4)
    i4_ms = timer.graph_ms(lambda i: mxq.qlinear(xq4, wq4, tp4, sets[0]["l2p"], out=sets[i % N_SETS]["y"]), n=4, reps=3)
    i4_tf = gemm_flops / (i4_ms * 1e-3) / 1e12
    rows["int4_g64_qlinear"] = {"kernel": "k_gemm_igroup<64> (E4M3-coded INT4 groups on kind::f8f6f4, fp32 group "
                                          "rescale in the epilogue)",
                                "us": 1e3 * i4_ms, "TFLOP/s": i4_tf, "frac_of_int8_peak": i4_tf / int8_peak,
                                "int8_peak": int8_peak}
    del wq4, xq4, tp4, w
    assert mxq.check() == 0
    return finish(args, world, rank, ms, value, clocks, gemm_tflops, fp4_peak, peaks, profiles_traffic, gemm_ms,
                  gemm_flops, rows, stream, sets, step, x_host, launches_per_step, torch, mxq)


def finish(args, world, rank, ms, value, clocks, gemm_tflops, fp4_peak, peaks, profiles_traffic, gemm_ms, gemm_flops,
           rows, stream, sets, step, x_host, launches_per_step, torch, mxq):
    """End-to-end measurement, the oracle on the host cores, and the JSON line."""
    dev = sets[0]["x"].device

    # ---- end to end through the public API with host buffers: each step copies its X in from
    # pinned memory and its Y out; the copies run on their own streams, overlapping the previous /
    # next step's kernels (inputs and outputs are double-buffered through the rotating sets)
    x_pin = x_host.pin_memory()
    y_pin = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d, d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    e_steps = max(4, min(args.steps, 20))

    def e2e_run(n):
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        ev_done = [torch.cuda.Event() for _ in range(n)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        h2d.wait_stream(stream)
        d2h.wait_stream(stream)
        for i in range(n):
            s = sets[i % N_SETS]
            if i >= N_SETS:   # set i's X was last read by step i - N_SETS, its Y last copied out by it
                h2d.wait_event(ev_out[i - N_SETS])
            with torch.cuda.stream(h2d):
                s["x"].copy_(x_pin, non_blocking=True)
                ev_in[i].record(h2d)
            stream.wait_event(ev_in[i])
            if i >= N_SETS:
                stream.wait_event(ev_done[i - N_SETS])
            step(i)
            ev_out[i].record(stream)
            d2h.wait_event(ev_out[i])
            if i >= 2:
                d2h.wait_event(ev_done[i - 2])
            with torch.cuda.stream(d2h):
                y_pin[i % 2].copy_(s["y"], non_blocking=True)
                ev_done[i].record(d2h)
        stream.wait_event(ev_done[n - 1])
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    e2e_run(4)
    _barrier(world)
    e2e_ms = _max_over_ranks(e2e_run(e_steps), world)
    _barrier(world)
    assert mxq.check() == 0

    cpu = None
    if rank == 0:
        o = OracleSample()
        o.timed(1)
        sec = o.timed(6)
        n_cores = host_cores()
        sec_all = o.timed(6, threads=n_cores)
        cpu = {"value": o.flops / sec / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
               "sample": o.desc + "; 6 steps on 1 thread",
               "extrapolated_full_step_s": sec * M / o.rows,
               "extrapolation": "the sample's time per step x %d / %d token rows (linear in M)" % (M, o.rows),
               "all_cores": {"value": o.flops / sec_all / 1e12, "unit": "TFLOP/s", "cores": n_cores,
                             "sample": "the same sample with numpy's BLAS on all host cores (the C steps stay on "
                                       "one thread)"}}
        cpu.update(oracle_bandwidth_rows())

    if rank == 0:
        line = {
            "metric": "qlinear TFLOPS (NVFP4 W4A4 + rank-32 low-rank), whole step",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "ms_per_step_eager": args.ms_eager,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "nvfp4(e2m1+ue4m3)xnvfp4->f32 acc, bf16 out", "data": "synthetic",
            "config": {"workload": WORKLOAD, "m": M, "k": K, "n": N, "rank": RANK, "out": "bf16",
                       "l2": "4 rotating input/output sets (~620 MB > 126 MB L2), no flush in the step loop; "
                             "bandwidth rows flushed (256 MiB read) before each launch",
                       "parallelism": "dp%d (independent batch per GPU)" % world,
                       "launch": "the timed steps replay CUDA graphs of 20 consecutive steps (60 kernels with "
                                 "programmatic edges, captured once before timing) and of the K mod 20 left; "
                                 "ms_per_step_eager: the same steps launched eagerly through the Python API"},
            "roofline": {"bound": "tensor", "kernel": "k_gemm<NVFP4> (main + low-rank up MMAs, fused epilogue)",
                         "achieved": gemm_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
                         "frac": gemm_tflops / fp4_peak, "traffic": profiles_traffic,
                         "peak_note": "measured bf16 burst %.1f TF/s x 4 (nominal dense FP4:BF16), of %s"
                                      % (peaks["bf16_tflops"], peaks["src"]),
                         "gemm_ms": gemm_ms, "flops_per_launch": gemm_flops,
                         "timing": "CUDA-graph replay of 100 launches over the 4 rotating sets, on the bench's "
                                   "stream, after the timed steps"},
            "rows": rows,
            "e2e": {"value": world * FLOP_STEP / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2, "ms_per_step": e2e_ms,
                    "how": "per step: X from pinned host memory on a copy stream, the three kernels, Y to pinned "
                           "host memory on another stream; copies overlap the neighbouring steps' kernels"},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)   # ~0.3 s timed: a few clock samples
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--rows", default="all", choices=["all", "none"],
                    help="'none': only the timed steps, the dominant kernel's timing, e2e and the CPU baseline")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = _dist_init()
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
