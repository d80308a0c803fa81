// capi.cu -- the extern "C" boundary declared in include/mxq.h: argument
// validation (all on the host, before any launch), buffer-size queries,
// format routing, and dispatch to the kernel launchers.
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstring>
#include <mutex>

#include "../../include/mxq.h"
#include "mxq_formats.cuh"
#include "mxq_internal.h"

using namespace mxq;

namespace {

bool valid_fmt(int32_t f) { return f >= 0 && f < MXQ_NUM_FMT; }
bool valid_dtype(int32_t d) { return d == MXQ_F32 || d == MXQ_BF16; }
bool valid_layout(int32_t l) { return l == MXQ_LAYOUT_CANONICAL || l == MXQ_LAYOUT_MMA; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_hadamard(int32_t b, int64_t cols) {
    if (b == 0) return true;
    return b >= 2 && b <= 256 && (b & (b - 1)) == 0 && cols % b == 0;
}

// Shape rule shared by the quantizers: 16-element chunks and whole blocks.
bool valid_shape(int32_t fmt, int64_t rows, int64_t cols) {
    if (rows < 0 || cols < 0 || cols % 16) return false;
    int blk = fmt_block(fmt);
    if (blk && cols % blk) return false;
    if (rows > (int64_t)1 << 31 || cols > (int64_t)1 << 31) return false;
    if (rows * (cols / 16) >= ((int64_t)1 << 31)) return false;   // chunk indices are 31-bit
    return true;
}

// The last CUDA error a call of this host thread returned as MXQ_ECUDA.
thread_local cudaError_t g_last_cuda = cudaSuccess;
mxq_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return MXQ_OK;
    g_last_cuda = e;
    return MXQ_ECUDA;
}

int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

// Arguments of mxq_quantize_lowrank other than the workspace.
mxq_status check_quantize_lowrank(const void *x, int32_t xdtype, int64_t m, int64_t k, int32_t fmt,
                                  int32_t hadamard_b, const void *l1, int32_t r, const float *w_tensor_scale,
                                  const void *codes, const void *scales, const float *tensor_scale, const void *tp) {
    if (!valid_fmt(fmt) || !valid_dtype(xdtype) || !valid_shape(fmt, m, k) || !valid_hadamard(hadamard_b, k))
        return MXQ_EINVAL;
    if (fmt == MXQ_INT8_ROW) return MXQ_EUNSUPPORTED;   // its GEMM takes no branch
    if (k <= 0 || r < 1 || r > 32) return MXQ_EINVAL;
    if (fmt_tensor_scaled(fmt) && (!tensor_scale || !w_tensor_scale)) return MXQ_EINVAL;
    if (m > 0 && (!x || !codes || !tp || !l1 || !aligned16(x) || !aligned16(codes) || !aligned16(tp)))
        return MXQ_EINVAL;
    if (m > 0 && fmt != MXQ_FP8_TENSOR && !scales) return MXQ_EINVAL;
    return MXQ_OK;
}

}  // namespace

extern "C" {

const char *mxq_last_cuda_error_string(void) { return cudaGetErrorString(g_last_cuda); }

const char *mxq_status_string(mxq_status st) {
    switch (st) {
    case MXQ_OK: return "ok";
    case MXQ_EINVAL: return "invalid argument";
    case MXQ_EUNSUPPORTED: return "unsupported format, combination or device";
    case MXQ_ECUDA: return "CUDA error";
    case MXQ_ETIMEOUT: return "a bounded device wait ran out";
    case MXQ_ENOSPACE: return "workspace too small";
    }
    return "unknown status";
}

int mxq_device_supported(int device) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess) return 0;
    return major == 10;
}

mxq_status mxq_check(void *stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return from_cuda(e);
    unsigned int w = 0;
    e = read_and_clear_error(&w);
    if (e != cudaSuccess) return from_cuda(e);
    return w ? MXQ_ETIMEOUT : MXQ_OK;
}

mxq_status mxq_selftest_wait_timeout(uint32_t wait_us, void *stream) {
    if (wait_us < 1 || wait_us > 1000000) return MXQ_EINVAL;
    return from_cuda(launch_wait_selftest(1000ull * wait_us, (cudaStream_t)stream));
}

mxq_status mxq_codes_bytes(int32_t fmt, int64_t rows, int64_t cols, int32_t layout, size_t *bytes) {
    if (!valid_fmt(fmt) || !valid_layout(layout) || !bytes || !valid_shape(fmt, rows, cols)) return MXQ_EINVAL;
    const bool int4_unpacked = (fmt == MXQ_INT4_G32 || fmt == MXQ_INT4_G64) && layout == MXQ_LAYOUT_MMA;
    *bytes = (size_t)(rows * cols / ((fmt_is4(fmt) && !int4_unpacked) ? 2 : 1));
    return MXQ_OK;
}

mxq_status mxq_scales_bytes(int32_t fmt, int64_t rows, int64_t cols, int32_t layout, size_t *bytes) {
    if (!valid_fmt(fmt) || !valid_layout(layout) || !bytes || !valid_shape(fmt, rows, cols)) return MXQ_EINVAL;
    switch (fmt) {
    case MXQ_MXFP8:
    case MXQ_MXFP4:
    case MXQ_NVFP4: {
        int64_t S = cols / fmt_block(fmt);
        *bytes = layout == MXQ_LAYOUT_CANONICAL ? (size_t)(rows * S) : (size_t)(round_up(rows, 128) * round_up(S, 16));
        break;
    }
    case MXQ_INT4_G32:
    case MXQ_INT4_G64: *bytes = (size_t)(rows * (cols / fmt_block(fmt)) * 4); break;
    case MXQ_INT8_ROW: *bytes = (size_t)(rows * 4); break;
    default: *bytes = 0;
    }
    return MXQ_OK;
}

mxq_status mxq_quantize_workspace_bytes(int32_t fmt, size_t *bytes) {
    if (!valid_fmt(fmt) || !bytes) return MXQ_EINVAL;
    *bytes = fmt_tensor_scaled(fmt) ? kLrHeader : 0;   // the amax word and per-CTA maxima
    return MXQ_OK;
}

mxq_status mxq_quantize(const void *x, int32_t xdtype, int64_t rows, int64_t cols, int32_t fmt, int32_t hadamard_b,
                        int32_t layout, void *codes, void *scales, float *tensor_scale, void *workspace,
                        size_t workspace_bytes, void *stream) {
    if (!valid_fmt(fmt) || !valid_dtype(xdtype) || !valid_layout(layout) || !valid_shape(fmt, rows, cols) ||
        !valid_hadamard(hadamard_b, cols))
        return MXQ_EINVAL;
    const int64_t n = rows * cols;
    if (n > 0 && (!x || !codes || !aligned16(x) || !aligned16(codes))) return MXQ_EINVAL;
    if (n > 0 && fmt != MXQ_FP8_TENSOR && !scales) return MXQ_EINVAL;
    if (fmt_tensor_scaled(fmt) && !tensor_scale) return MXQ_EINVAL;
    size_t ws = 0, sb = 0;
    mxq_quantize_workspace_bytes(fmt, &ws);
    if (ws && (!workspace || workspace_bytes < ws)) return workspace ? MXQ_ENOSPACE : MXQ_EINVAL;
    mxq_scales_bytes(fmt, rows, cols, layout, &sb);
    return from_cuda(launch_quantize(x, xdtype == MXQ_BF16, rows, cols, fmt, hadamard_b, layout, codes, scales, sb,
                                     tensor_scale, (unsigned int *)workspace, (cudaStream_t)stream));
}

mxq_status mxq_dequantize(const mxq_qtensor *q, void *y, int32_t ydtype, void *stream) {
    if (!q || !valid_fmt(q->fmt) || !valid_layout(q->layout) || !valid_dtype(ydtype) ||
        !valid_shape(q->fmt, q->rows, q->cols))
        return MXQ_EINVAL;
    if (q->rows * q->cols > 0) {
        if (!q->codes || !y || !aligned16(q->codes) || !aligned16(y)) return MXQ_EINVAL;
        if (q->fmt != MXQ_FP8_TENSOR && !q->scales) return MXQ_EINVAL;
        if (fmt_tensor_scaled(q->fmt) && !q->tensor_scale) return MXQ_EINVAL;
    }
    return from_cuda(launch_dequantize(q->fmt, q->layout, q->rows, q->cols, q->codes, q->scales, q->tensor_scale, y,
                                       ydtype == MXQ_BF16, (cudaStream_t)stream));
}

mxq_status mxq_hadamard_block(const void *x, void *y, int32_t dtype, int64_t rows, int64_t cols, int32_t b,
                              void *stream) {
    if (!valid_dtype(dtype) || rows < 0 || cols < 0 || cols % 16 || b == 0 || !valid_hadamard(b, cols))
        return MXQ_EINVAL;
    if (rows * cols > 0 && (!x || !y || !aligned16(x) || !aligned16(y))) return MXQ_EINVAL;
    return from_cuda(launch_hadamard(x, y, dtype == MXQ_BF16, rows, cols, b, (cudaStream_t)stream));
}

mxq_status mxq_cast(const float *x, int64_t n, int32_t elem, uint8_t *out, void *stream) {
    if (n < 0 || (elem != 0 && elem != 1)) return MXQ_EINVAL;
    if (n > 0 && (!x || !out)) return MXQ_EINVAL;
    return from_cuda(launch_cast(x, n, elem, out, (cudaStream_t)stream));
}

mxq_status mxq_select_workspace_bytes(const int32_t *candidates, int32_t ncand, size_t *bytes) {
    if (!candidates || ncand < 1 || ncand > kMaxCandidates || !bytes) return MXQ_EINVAL;
    *bytes = kLrHeader;   // the amax word, or per-CTA maxima from byte 256
    return MXQ_OK;
}

mxq_status mxq_select_weight_format(const void *w, int32_t wdtype, int64_t n, int64_t k, const int32_t *candidates,
                                    int32_t ncand, uint8_t *fmt_per_channel, double *sse, void *workspace,
                                    size_t workspace_bytes, void *stream) {
    if (!valid_dtype(wdtype) || !candidates || ncand < 1 || ncand > kMaxCandidates || n < 0 || k < 0 || k % 16)
        return MXQ_EINVAL;
    int cands[kMaxCandidates];
    for (int j = 0; j < ncand; j++) {
        if (!valid_fmt(candidates[j]) || !valid_shape(candidates[j], n, k)) return MXQ_EINVAL;
        cands[j] = candidates[j];
    }
    if (n > 0 && (!w || !fmt_per_channel || !aligned16(w))) return MXQ_EINVAL;
    if (!workspace) return MXQ_EINVAL;
    if (workspace_bytes < kLrHeader) return MXQ_ENOSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MXQ_EINVAL;
    const cudaError_t e = launch_select_fixed(w, wdtype == MXQ_BF16, n, k, cands, ncand, fmt_per_channel, sse,
                                              (float *)((char *)workspace + 256), (cudaStream_t)stream);
    if (e != cudaErrorNotSupported) return from_cuda(e);
    return from_cuda(launch_select(w, wdtype == MXQ_BF16, n, k, cands, ncand, fmt_per_channel, sse,
                                   (unsigned int *)workspace, (cudaStream_t)stream));
}

mxq_status mxq_quantize_mse_workspace_bytes(int64_t rows, int64_t cols, size_t *bytes) {
    if (rows < 0 || cols < 0 || cols % 16 || !bytes) return MXQ_EINVAL;
    *bytes = mse_workspace_bytes(rows, cols);
    return MXQ_OK;
}

mxq_status mxq_quantize_mse(const void *w, int32_t wdtype, int64_t rows, int64_t cols, int32_t fmt,
                            int32_t iters, int32_t layout, void *codes, void *scales, float *tensor_scale,
                            double *sse, void *workspace, size_t workspace_bytes, void *stream) {
    if (!valid_fmt(fmt) || !valid_dtype(wdtype) || !valid_layout(layout) || iters < 0) return MXQ_EINVAL;
    if (fmt != MXQ_NVFP4) return MXQ_EUNSUPPORTED;
    if (!valid_shape(fmt, rows, cols) || !tensor_scale) return MXQ_EINVAL;
    const int64_t n = rows * cols;
    if (n > 0 && (!w || !codes || !scales || !aligned16(w) || !aligned16(codes))) return MXQ_EINVAL;
    size_t need = 0, sb = 0;
    mxq_quantize_mse_workspace_bytes(rows, cols, &need);
    if (!workspace) return MXQ_EINVAL;
    if (workspace_bytes < need) return MXQ_ENOSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MXQ_EINVAL;
    mxq_scales_bytes(fmt, rows, cols, layout, &sb);
    return from_cuda(launch_quantize_mse(w, wdtype == MXQ_BF16, rows, cols, iters, layout, codes, scales, sb,
                                         tensor_scale, sse, workspace, (cudaStream_t)stream));
}

static bool valid_grid(float g) { return g >= 1.0f && g <= 2.0f; }

mxq_status mxq_quantize_mx_grid(const void *x, int32_t xdtype, int64_t rows, int64_t cols, int32_t fmt,
                                int32_t hadamard_b, float grid_scale, int32_t layout, void *codes, void *scales,
                                void *stream) {
    if (!valid_fmt(fmt) || !valid_dtype(xdtype) || !valid_layout(layout)) return MXQ_EINVAL;
    if (fmt != MXQ_MXFP4 && fmt != MXQ_MXFP8) return MXQ_EUNSUPPORTED;
    if (!valid_shape(fmt, rows, cols) || !valid_hadamard(hadamard_b, cols) || !valid_grid(grid_scale))
        return MXQ_EINVAL;
    const int64_t n = rows * cols;
    if (n > 0 && (!x || !codes || !scales || !aligned16(x) || !aligned16(codes))) return MXQ_EINVAL;
    size_t sb = 0;
    mxq_scales_bytes(fmt, rows, cols, layout, &sb);
    return from_cuda(launch_quantize(x, xdtype == MXQ_BF16, rows, cols, fmt, hadamard_b, layout, codes, scales, sb,
                                     nullptr, nullptr, (cudaStream_t)stream, nullptr, false, grid_scale));
}

mxq_status mxq_fit_mx_grid_workspace_bytes(int64_t rows, int64_t cols, int32_t n, size_t *bytes) {
    if (rows < 0 || cols < 0 || cols % 32 || n < 1 || n > kMaxCandidates || !bytes) return MXQ_EINVAL;
    *bytes = mx_grid_workspace_bytes(rows, cols, n);
    return MXQ_OK;
}

mxq_status mxq_fit_mx_grid(const void *w, int32_t wdtype, int64_t rows, int64_t cols, int32_t fmt,
                           int32_t hadamard_b, const float *grid_scales, int32_t n, double *sse, void *workspace,
                           size_t workspace_bytes, void *stream) {
    if (!valid_fmt(fmt) || !valid_dtype(wdtype)) return MXQ_EINVAL;
    if (fmt != MXQ_MXFP4 && fmt != MXQ_MXFP8) return MXQ_EUNSUPPORTED;
    if (!valid_shape(fmt, rows, cols) || !valid_hadamard(hadamard_b, cols)) return MXQ_EINVAL;
    if (n < 1 || n > kMaxCandidates || !grid_scales || !sse) return MXQ_EINVAL;
    for (int j = 0; j < n; j++)
        if (!valid_grid(grid_scales[j])) return MXQ_EINVAL;
    if (rows * cols > 0 && (!w || !aligned16(w))) return MXQ_EINVAL;
    size_t need = 0;
    mxq_fit_mx_grid_workspace_bytes(rows, cols, n, &need);
    if (!workspace) return MXQ_EINVAL;
    if (workspace_bytes < need) return MXQ_ENOSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MXQ_EINVAL;
    return from_cuda(launch_fit_mx_grid(w, wdtype == MXQ_BF16, rows, cols, fmt, hadamard_b, grid_scales, n, sse,
                                        workspace, (cudaStream_t)stream));
}

static bool copy_candidates(const int32_t *candidates, int32_t ncand, int *out) {
    if (!candidates || ncand < 1 || ncand > kMaxCandidates) return false;
    for (int j = 0; j < ncand; j++) {
        if (!valid_fmt(candidates[j])) return false;
        out[j] = candidates[j];
    }
    return true;
}

mxq_status mxq_calibrate_workspace_bytes(int64_t rows, int64_t cols, int32_t ncand, size_t *bytes) {
    if (rows < 0 || cols < 0 || cols % 64 || ncand < 1 || ncand > kMaxCandidates || !bytes) return MXQ_EINVAL;
    *bytes = calib_workspace_bytes(rows, cols, ncand);
    return MXQ_OK;
}

mxq_status mxq_calibrate_activation(const void *x, int32_t xdtype, int64_t rows, int64_t cols,
                                    const int32_t *candidates, int32_t ncand, double *sse_accum,
                                    double *moments_accum, void *workspace, size_t workspace_bytes, void *stream) {
    int cands[kMaxCandidates];
    if (!valid_dtype(xdtype) || !copy_candidates(candidates, ncand, cands)) return MXQ_EINVAL;
    if (rows < 0 || cols < 0 || cols % 64 || rows * (cols / 16) >= ((int64_t)1 << 31)) return MXQ_EINVAL;
    if (!sse_accum || !moments_accum) return MXQ_EINVAL;
    if (rows * cols > 0 && (!x || !aligned16(x))) return MXQ_EINVAL;
    size_t need = 0;
    mxq_calibrate_workspace_bytes(rows, cols, ncand, &need);
    if (!workspace) return MXQ_EINVAL;
    if (workspace_bytes < need) return MXQ_ENOSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MXQ_EINVAL;
    return from_cuda(launch_calibrate(x, xdtype == MXQ_BF16, rows, cols, cands, ncand, sse_accum, moments_accum,
                                      workspace, (cudaStream_t)stream));
}

mxq_status mxq_calibrate_pick(const double *sse_accum, const int32_t *candidates, int32_t ncand, int32_t forced_fmt,
                              uint8_t *entry, void *stream) {
    int cands[kMaxCandidates];
    if (!copy_candidates(candidates, ncand, cands) || !sse_accum || !entry) return MXQ_EINVAL;
    if (forced_fmt >= 0 && !valid_fmt(forced_fmt)) return MXQ_EINVAL;
    return from_cuda(launch_calib_pick(sse_accum, cands, ncand, forced_fmt < 0 ? -1 : forced_fmt, entry,
                                       (cudaStream_t)stream));
}

mxq_status mxq_lowrank_down(const void *x, int32_t xdtype, int64_t m, int64_t k, const void *l1, int32_t r, float *t,
                            void *stream) {
    if (!valid_dtype(xdtype) || m < 0 || k <= 0 || k % 16 || r < 1 || r > 32) return MXQ_EINVAL;
    if (m > 0 && (!x || !l1 || !t || !aligned16(x))) return MXQ_EINVAL;
    return from_cuda(launch_lowrank_down(x, xdtype == MXQ_BF16, m, k, l1, r, t, nullptr, nullptr, nullptr,
                                         (cudaStream_t)stream));
}

mxq_status mxq_lowrank_packed_bytes(int64_t m, size_t *bytes) {
    if (m < 0 || !bytes) return MXQ_EINVAL;
    *bytes = (size_t)(m * 64 * 2);
    return MXQ_OK;
}

mxq_status mxq_lowrank_down_packed(const void *x, int32_t xdtype, int64_t m, int64_t k, const void *l1, int32_t r,
                                   const float *x_tensor_scale, const float *w_tensor_scale, void *tp, void *stream) {
    if (!valid_dtype(xdtype) || m < 0 || k <= 0 || k % 16 || r < 1 || r > 32) return MXQ_EINVAL;
    if (!x_tensor_scale != !w_tensor_scale) return MXQ_EINVAL;
    if (m > 0 && (!x || !l1 || !tp || !aligned16(x) || !aligned16(tp))) return MXQ_EINVAL;
    return from_cuda(launch_lowrank_down(x, xdtype == MXQ_BF16, m, k, l1, r, nullptr, x_tensor_scale,
                                         w_tensor_scale, tp, (cudaStream_t)stream));
}

mxq_status mxq_lowrank_pack_t(const float *t, int32_t r, int64_t m, const float *x_tensor_scale,
                              const float *w_tensor_scale, void *tp, void *stream) {
    if (r < 1 || r > 32 || m < 0 || (!x_tensor_scale != !w_tensor_scale)) return MXQ_EINVAL;
    if (m > 0 && (!t || !tp || !aligned16(tp))) return MXQ_EINVAL;
    return from_cuda(launch_pack_t(t, r, m, x_tensor_scale, w_tensor_scale, tp, (cudaStream_t)stream));
}

mxq_status mxq_quantize_lowrank_workspace_bytes(int64_t m, int32_t r, size_t *bytes) {
    if (m < 0 || r < 1 || r > 32 || !bytes) return MXQ_EINVAL;
    *bytes = kLrHeader + (size_t)(m * r * 4);
    return MXQ_OK;
}

mxq_status mxq_quantize_lowrank(const void *x, int32_t xdtype, int64_t m, int64_t k, int32_t fmt, int32_t hadamard_b,
                                const void *l1, int32_t r, const float *w_tensor_scale, void *codes, void *scales,
                                float *tensor_scale, void *tp, void *workspace, size_t workspace_bytes,
                                void *stream) {
    const mxq_status chk = check_quantize_lowrank(x, xdtype, m, k, fmt, hadamard_b, l1, r, w_tensor_scale, codes,
                                                  scales, tensor_scale, tp);
    if (chk != MXQ_OK) return chk;
    const bool ts = fmt_tensor_scaled(fmt);
    size_t need = 0, sb = 0;
    mxq_quantize_lowrank_workspace_bytes(m, r, &need);
    if (!workspace) return MXQ_EINVAL;
    if (workspace_bytes < need) return MXQ_ENOSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MXQ_EINVAL;
    mxq_scales_bytes(fmt, m, k, MXQ_LAYOUT_MMA, &sb);
    cudaStream_t s = (cudaStream_t)stream;
    unsigned int *amax = (unsigned int *)workspace;
    float *slots = (float *)((char *)workspace + 256);
    float *t = (float *)((char *)workspace + kLrHeader);
    const bool bf = xdtype == MXQ_BF16;
    cudaError_t e = cudaSuccess;
    bool amax_ready = false;
    int n_slots = 0;
    if (ts && hadamard_b == 0) {
        // one read of x from HBM gives both the tensor amax and t: the
        // tensor-core kernel writes per-warp maxima and the mma.sync kernels
        // per-CTA maxima (every slot written, so no clearing: the kernels
        // follow each other with no memset between); only a grid with more
        // CTAs than slots folds into a zeroed word
        e = bf ? launch_lowrank_tc(x, m, k, l1, r, t, nullptr, nullptr, nullptr, slots, &n_slots, s)
               : cudaErrorNotSupported;
        if (e == cudaErrorNotSupported) {   // the mma.sync kernels: one maximum per CTA, still no clearing
            n_slots = 0;
            e = launch_lowrank_down(x, bf, m, k, l1, r, t, nullptr, nullptr, nullptr, s, nullptr, slots, &n_slots);
        }
        if (e == cudaErrorNotSupported) {   // more CTAs than slots: fold into a cleared word
            n_slots = 0;
            e = cudaMemsetAsync(amax, 0, sizeof(unsigned int), s);
            if (e == cudaSuccess) e = launch_lowrank_down(x, bf, m, k, l1, r, t, nullptr, nullptr, nullptr, s, amax);
        }
        amax_ready = true;
    } else {
        e = launch_lowrank_down(x, bf, m, k, l1, r, t, nullptr, nullptr, nullptr, s);
    }
    if (e != cudaSuccess) return from_cuda(e);
    PackT pack{t, r, w_tensor_scale, tp};
    return from_cuda(launch_quantize(x, bf, m, k, fmt, hadamard_b, MXQ_LAYOUT_MMA, codes, scales, sb, tensor_scale,
                                     amax, s, &pack, amax_ready, 1.0f, slots, n_slots));
}

mxq_status mxq_qlinear_w4a16_workspace_bytes(int64_t m, int64_t n, int64_t k, size_t *bytes) {
    if (!bytes || m < 0 || n < 0 || k <= 0 || k % 64 || n >= ((int64_t)1 << 31) || k >= ((int64_t)1 << 31))
        return MXQ_EINVAL;
    *bytes = m >= 512 ? (size_t)(n * k * 2) : 0;   // below that, the fused kernel is the faster route
    return MXQ_OK;
}

mxq_status mxq_qlinear_w4a16(const void *x, int64_t m, int64_t k, const mxq_qtensor *wq, void *y, int32_t ydtype,
                             void *workspace, size_t workspace_bytes, void *stream) {
    if (!wq || !valid_dtype(ydtype) || m < 0 || k <= 0 || k % 64) return MXQ_EINVAL;
    if (wq->fmt != MXQ_INT4_G32 && wq->fmt != MXQ_INT4_G64) return MXQ_EUNSUPPORTED;
    if (wq->layout != MXQ_LAYOUT_CANONICAL || wq->cols != k || wq->rows < 0) return MXQ_EINVAL;
    if (m >= ((int64_t)1 << 31) || wq->rows >= ((int64_t)1 << 31) || k >= ((int64_t)1 << 31)) return MXQ_EINVAL;
    // the kernel counts 128 x 128 tiles and their 64-column stages in 32-bit integers; each factor
    // is below 2^24 here, so the tile count (< 2^48) is exact, and the product is formed only once
    // the tile count is known to be below 2^31
    const int64_t wa_tiles = ((m + 127) / 128) * ((wq->rows + 127) / 128);
    if (wa_tiles >= ((int64_t)1 << 31) || wa_tiles * (k / 64) >= ((int64_t)1 << 31)) return MXQ_EINVAL;
    if (m > 0 && wq->rows > 0 && (!x || !y || !wq->codes || !wq->scales || !aligned16(x) || !aligned16(wq->codes)))
        return MXQ_EINVAL;
    size_t need = 0;
    mxq_qlinear_w4a16_workspace_bytes(m, wq->rows, k, &need);
    if (workspace && need > 0 && workspace_bytes >= need && m > 0 && wq->rows > 0) {
        if (!aligned16(workspace)) return MXQ_EINVAL;
        // the bf16 GEMM counts 256-row x 256-column tiles and their 64-element stages in 32-bit integers
        if (((m + 255) / 256) * ((wq->rows + 255) / 256) * (k / 64) >= ((int64_t)1 << 31)) return MXQ_EINVAL;
        cudaStream_t s = (cudaStream_t)stream;
        // W16 = bf16(RN32(q s)), the dequantizer's rounding, written once
        cudaError_t e = launch_dequantize(wq->fmt, MXQ_LAYOUT_CANONICAL, wq->rows, k, wq->codes, wq->scales, nullptr,
                                          workspace, true, s);
        if (e != cudaSuccess) return from_cuda(e);
        GemmOperands op;
        memset(&op, 0, sizeof(op));
        op.fmt = wq->fmt;
        op.m = m;
        op.n = wq->rows;
        op.k = k;
        op.a_codes = x;
        op.b_codes = workspace;
        op.y = y;
        op.y_bf16 = ydtype == MXQ_BF16;
        return from_cuda(launch_gemm_bf16(op, s));
    }
    return from_cuda(launch_w4a16(x, m, k, (const uint8_t *)wq->codes, (const float *)wq->scales, wq->rows,
                                  wq->fmt == MXQ_INT4_G32 ? 32 : 64, y, ydtype == MXQ_BF16, (cudaStream_t)stream));
}

mxq_status mxq_lowrank_pack_l2(const void *l2, int32_t r, int64_t n, void *l2p, void *stream) {
    if (r < 1 || r > 32 || n < 0) return MXQ_EINVAL;
    if (n > 0 && (!l2 || !l2p || !aligned16(l2p))) return MXQ_EINVAL;
    return from_cuda(launch_pack_l2(l2, r, n, l2p, (cudaStream_t)stream));
}

mxq_status mxq_qlinear(const mxq_qtensor *xq, const mxq_qtensor *wq, const void *tp, const void *l2p, void *y,
                       int32_t ydtype, void *stream) {
    if (!xq || !wq || !valid_dtype(ydtype) || !y) return MXQ_EINVAL;
    if (!valid_fmt(xq->fmt) || xq->fmt != wq->fmt) return MXQ_EUNSUPPORTED;
    const int fmt = xq->fmt;
    const bool igroup = fmt == MXQ_INT4_G32 || fmt == MXQ_INT4_G64;
    if (xq->layout != MXQ_LAYOUT_MMA || wq->layout != MXQ_LAYOUT_MMA) return MXQ_EINVAL;
    const int64_t m = xq->rows, n = wq->rows, k = xq->cols;
    if (wq->cols != k || k <= 0 || m < 0 || n < 0) return MXQ_EINVAL;
    if (k % (igroup ? fmt_block(fmt) : fmt_is4(fmt) ? 64 : 32)) return MXQ_EINVAL;
    if (!valid_shape(fmt, m, k) || !valid_shape(fmt, n, k)) return MXQ_EINVAL;
    // the kernels count output tiles and their K stages in 32-bit integers
    if (((m + 127) / 128) * ((n + 127) / 128) * (k / 16) >= ((int64_t)1 << 31)) return MXQ_EINVAL;
    if (m > 0 && n > 0) {
        if (!xq->codes || !wq->codes || !aligned16(xq->codes) || !aligned16(wq->codes) || !aligned16(y))
            return MXQ_EINVAL;
        if (fmt != MXQ_FP8_TENSOR && (!xq->scales || !wq->scales)) return MXQ_EINVAL;
        if (fmt_tensor_scaled(fmt) && (!xq->tensor_scale || !wq->tensor_scale)) return MXQ_EINVAL;
    }
    if (tp) {
        if (fmt == MXQ_INT8_ROW) return MXQ_EUNSUPPORTED;
        if (!l2p || !aligned16(l2p) || !aligned16(tp)) return MXQ_EINVAL;
    }
    GemmOperands op;
    op.fmt = fmt;
    op.m = m;
    op.n = n;
    op.k = k;
    op.a_codes = xq->codes;
    op.b_codes = wq->codes;
    op.a_scales = xq->scales;
    op.b_scales = wq->scales;
    op.a_tensor_scale = xq->tensor_scale;
    op.b_tensor_scale = wq->tensor_scale;
    op.tp = tp;
    op.l2p = l2p;
    op.y = y;
    op.y_bf16 = ydtype == MXQ_BF16;
    return from_cuda(igroup ? launch_qlinear_igroup(op, (cudaStream_t)stream) : launch_qlinear(op, (cudaStream_t)stream));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of mxq_quantize_lowrank: its scratch (the tensor-amax
// word and the fp32 low-rank activation) lives in this file-scope device
// array, which every GPU that loads the library holds until the process ends.
// In host code the array's name is only a stand-in for the device object, so
// the device address is looked up once per device (with that device current)
// and cached.
namespace {
constexpr size_t kNoAllocScratchBytes = (size_t)4 << 20;   // 4 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
constexpr int kNoAllocMaxDevices = 64;
void *g_noalloc_addr[kNoAllocMaxDevices];
std::mutex g_noalloc_lock;

mxq_status noalloc_scratch(void **ptr) {
    int dev = 0;
    const cudaError_t de = cudaGetDevice(&dev);
    if (de != cudaSuccess) return from_cuda(de);
    if (dev < 0 || dev >= kNoAllocMaxDevices) return MXQ_EUNSUPPORTED;
    std::lock_guard<std::mutex> guard(g_noalloc_lock);
    if (!g_noalloc_addr[dev]) {
        void *a = nullptr;
        const cudaError_t se = cudaGetSymbolAddress(&a, g_noalloc_scratch);
        if (se != cudaSuccess) return from_cuda(se);
        if (!a) return MXQ_ECUDA;
        g_noalloc_addr[dev] = a;
    }
    *ptr = g_noalloc_addr[dev];
    return MXQ_OK;
}
}  // namespace

extern "C" {

mxq_status mxq_quantize_lowrank_noalloc(const void *x, int32_t xdtype, int64_t m, int64_t k, int32_t fmt,
                                        int32_t hadamard_b, const void *l1, int32_t r,
                                        const float *w_tensor_scale, void *codes, void *scales,
                                        float *tensor_scale, void *tp, void *stream) {
    // every argument is checked before the device array is looked up, so a
    // rejected call makes no CUDA call at all
    const mxq_status chk = check_quantize_lowrank(x, xdtype, m, k, fmt, hadamard_b, l1, r, w_tensor_scale, codes,
                                                  scales, tensor_scale, tp);
    if (chk != MXQ_OK) return chk;
    size_t need = 0;
    if (mxq_quantize_lowrank_workspace_bytes(m, r, &need) != MXQ_OK) return MXQ_EINVAL;
    if (need > kNoAllocScratchBytes) return MXQ_ENOSPACE;
    void *scratch = nullptr;
    const mxq_status st = noalloc_scratch(&scratch);
    if (st != MXQ_OK) return st;
    return mxq_quantize_lowrank(x, xdtype, m, k, fmt, hadamard_b, l1, r, w_tensor_scale, codes, scales, tensor_scale,
                                tp, scratch, kNoAllocScratchBytes, stream);
}

int32_t mxq_route(const uint8_t *table, int32_t n_layers, int32_t n_intervals, int32_t layer, int32_t step,
                  int32_t n_steps) {
    if (!table || n_layers <= 0 || n_intervals <= 0 || n_steps <= 0) return -1;
    if (layer < 0 || layer >= n_layers || step < 0 || step >= n_steps) return -1;
    const int64_t interval = (int64_t)step * n_intervals / n_steps;
    return table[(int64_t)layer * n_intervals + interval];
}

}  // extern "C"

namespace {

// Workspace of mxq_qlinear_routed, each part at a 256-byte boundary: the
// workspace of mxq_quantize_lowrank (the amax words, then t), the codes and
// scales of the quantized activation in the largest format, its tensor
// scale, and the packed low-rank operand.
struct RoutedLayout {
    size_t lowrank, codes, scales, tscale, tp, total;
};

RoutedLayout routed_layout(int64_t m, int64_t k, int32_t r) {
    RoutedLayout L;
    size_t off = 0;
    auto take = [&off](size_t bytes) {
        const size_t at = off;
        off += (bytes + 255) / 256 * 256;
        return at;
    };
    L.lowrank = take(kLrHeader + (size_t)(m * (r > 0 ? r : 0) * 4));
    L.codes = take((size_t)(m * k));                                  // 8-bit codes, or INT4 as bytes
    const size_t nv = (size_t)(round_up(m, 128) * round_up(k / 16, 16));   // NVFP4 scales bound the MX ones
    const size_t ig = (size_t)(m * (k / 32) * 4);                        // INT4_G32 fp32 group scales
    size_t sc = nv > ig ? nv : ig;
    if ((size_t)(m * 4) > sc) sc = (size_t)(m * 4);                      // INT8_ROW row scales
    L.scales = take(sc);
    L.tscale = take(4);
    L.tp = take(r > 0 ? (size_t)(m * 64 * 2) : 0);
    L.total = off;
    return L;
}

}  // namespace

extern "C" {

mxq_status mxq_qlinear_routed_workspace_bytes(int64_t m, int64_t k, int32_t r, size_t *bytes) {
    if (m < 0 || k < 0 || k % 16 || r < 0 || r > 32 || !bytes) return MXQ_EINVAL;
    if (m > ((int64_t)1 << 31) || k > ((int64_t)1 << 31) || m * (k / 16) >= ((int64_t)1 << 31)) return MXQ_EINVAL;
    *bytes = routed_layout(m, k, r).total;
    return MXQ_OK;
}

mxq_status mxq_qlinear_routed(const void *x, int32_t xdtype, int64_t m, int64_t k, const mxq_layer *layer_w,
                              const uint8_t *fmt_table, int32_t n_layers, int32_t n_intervals, int32_t layer,
                              int32_t step, int32_t n_steps, void *y, int32_t ydtype, int32_t *fmt_used,
                              void *workspace, size_t workspace_bytes, void *stream) {
    if (!layer_w || !valid_dtype(xdtype) || !valid_dtype(ydtype)) return MXQ_EINVAL;
    const int32_t fmt = mxq_route(fmt_table, n_layers, n_intervals, layer, step, n_steps);
    if (!valid_fmt(fmt)) return MXQ_EINVAL;
    if (fmt_used) *fmt_used = fmt;
    const mxq_qtensor *wq = &layer_w->w[fmt];
    if (!wq->codes || wq->fmt != fmt || wq->layout != MXQ_LAYOUT_MMA || wq->cols != k) return MXQ_EINVAL;
    const int32_t r = layer_w->r;
    if (r < 0 || r > 32 || (r > 0 && (!layer_w->l1 || !layer_w->l2p))) return MXQ_EINVAL;
    if (r > 0 && fmt == MXQ_INT8_ROW) return MXQ_EUNSUPPORTED;   // the INT8 GEMM takes no branch
    size_t need = 0;
    if (mxq_qlinear_routed_workspace_bytes(m, k, r, &need) != MXQ_OK) return MXQ_EINVAL;
    if (!workspace) return MXQ_EINVAL;
    if (workspace_bytes < need) return MXQ_ENOSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MXQ_EINVAL;
    const RoutedLayout L = routed_layout(m, k, r);
    uint8_t *ws = (uint8_t *)workspace;
    size_t cb = 0, sb = 0;
    if (mxq_codes_bytes(fmt, m, k, MXQ_LAYOUT_MMA, &cb) != MXQ_OK ||
        mxq_scales_bytes(fmt, m, k, MXQ_LAYOUT_MMA, &sb) != MXQ_OK)
        return MXQ_EINVAL;   // k not a whole number of the routed format's blocks
    mxq_qtensor xq;
    xq.fmt = fmt;
    xq.layout = MXQ_LAYOUT_MMA;
    xq.rows = m;
    xq.cols = k;
    xq.codes = ws + L.codes;
    xq.scales = sb ? ws + L.scales : nullptr;
    xq.tensor_scale = fmt_tensor_scaled(fmt) ? (const float *)(ws + L.tscale) : nullptr;
    mxq_status st;
    void *tp = nullptr;
    if (r > 0) {
        tp = ws + L.tp;
        st = mxq_quantize_lowrank(x, xdtype, m, k, fmt, layer_w->hadamard_b, layer_w->l1, r, wq->tensor_scale,
                                  (void *)xq.codes, (void *)xq.scales, (float *)xq.tensor_scale, tp, ws + L.lowrank,
                                  L.codes - L.lowrank, stream);
    } else {
        st = mxq_quantize(x, xdtype, m, k, fmt, layer_w->hadamard_b, MXQ_LAYOUT_MMA, (void *)xq.codes,
                          (void *)xq.scales, (float *)xq.tensor_scale, ws + L.lowrank, L.codes - L.lowrank, stream);
    }
    if (st != MXQ_OK) return st;
    return mxq_qlinear(&xq, wq, tp, r > 0 ? layer_w->l2p : nullptr, y, ydtype, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Per-channel mixed weight formats (mixed.cu).
namespace {

int mixed_group(int32_t f) { return f == MXQ_MXFP4 ? 0 : f == MXQ_INT4_G32 ? 1 : f == MXQ_NVFP4 ? 2 : -1; }

bool valid_mixed_weight(const mxq_mixed_weight *w) {
    if (!w || w->rows < 0 || w->cols <= 0 || w->cols % 32 || w->rows >= ((int64_t)1 << 31)) return false;
    if (w->rows * (w->cols / 16) >= ((int64_t)1 << 31)) return false;
    int64_t total = 0;
    for (int g = 0; g < 3; g++) {
        if (w->n_group[g] < 0) return false;
        total += w->n_group[g];
    }
    if (total != w->rows) return false;
    if (w->rows > 0 && (!w->choice || !w->group_index)) return false;
    if (w->n_group[0] > 0 && (!w->mx_codes || !w->mx_scales || !aligned16(w->mx_codes))) return false;
    if (w->n_group[1] > 0 && (!w->i4_codes || !w->i4_scales || !aligned16(w->i4_codes))) return false;
    if (w->n_group[2] > 0 && (!w->nv_values || !w->nv_tensor_scale || !aligned16(w->nv_values))) return false;
    return true;
}

struct MixedLayout {
    size_t sx, abf, y[3], total;
};

// The group that holds every channel, or -1: channel n is then row n of that
// group (mxq_mixed_plan keeps the channel order inside a group), so its GEMM
// writes y directly and nothing is scattered.
int mixed_single_group(const mxq_mixed_weight *w) {
    for (int g = 0; g < 3; g++)
        if (w->n_group[g] == w->rows && w->rows > 0) return g;
    return -1;
}

MixedLayout mixed_layout(int64_t m, const mxq_mixed_weight *w, int32_t ydtype) {
    MixedLayout L;
    size_t off = 0;
    auto take = [&off](size_t bytes) {
        const size_t at = off;
        off += (bytes + 255) / 256 * 256;
        return at;
    };
    const int64_t k = w->cols;
    L.sx = take(w->n_group[1] > 0 ? (size_t)(m * (k / 32) * 4) : 0);
    L.abf = take(w->n_group[2] > 0 ? (size_t)(m * k * 2) : 0);
    const size_t esz = ydtype == MXQ_BF16 ? 2 : 4;
    const int single = mixed_single_group(w);
    for (int g = 0; g < 3; g++) L.y[g] = take(single >= 0 ? 0 : (size_t)(m * w->n_group[g]) * esz);
    L.total = off;
    return L;
}

}  // namespace

extern "C" {

mxq_status mxq_mixed_plan(const uint8_t *choice, int64_t n, int64_t n_group[3], int32_t *group_index) {
    if (!n_group || n < 0 || n >= ((int64_t)1 << 31) || (n > 0 && (!choice || !group_index))) return MXQ_EINVAL;
    int64_t cnt[3] = {0, 0, 0};
    for (int64_t i = 0; i < n; i++) {
        const int g = mixed_group(choice[i]);
        if (g < 0) return MXQ_EINVAL;
        group_index[i] = (int32_t)cnt[g]++;
    }
    for (int g = 0; g < 3; g++) n_group[g] = cnt[g];
    return MXQ_OK;
}

mxq_status mxq_mixed_weight_bytes(const int64_t n_group[3], int64_t k, size_t bytes[5]) {
    if (!n_group || !bytes || k <= 0 || k % 32) return MXQ_EINVAL;
    for (int g = 0; g < 3; g++)
        if (n_group[g] < 0 || n_group[g] * (k / 16) >= ((int64_t)1 << 31)) return MXQ_EINVAL;
    bytes[0] = (size_t)(n_group[0] * k);
    if (mxq_scales_bytes(MXQ_MXFP8, n_group[0], k, MXQ_LAYOUT_MMA, &bytes[1]) != MXQ_OK) return MXQ_EINVAL;
    bytes[2] = (size_t)(n_group[1] * k);
    bytes[3] = (size_t)(n_group[1] * (k / 32) * 4);
    bytes[4] = (size_t)(n_group[2] * k * 2);
    return MXQ_OK;
}

mxq_status mxq_mixed_prepare(const mxq_qtensor *w_mxfp4, const mxq_qtensor *w_int4, const mxq_qtensor *w_nvfp4,
                             const mxq_mixed_weight *out, void *stream) {
    if (!w_mxfp4 || !w_int4 || !w_nvfp4 || !valid_mixed_weight(out)) return MXQ_EINVAL;
    const mxq_qtensor *ws[3] = {w_mxfp4, w_int4, w_nvfp4};
    const int32_t fmts[3] = {MXQ_MXFP4, MXQ_INT4_G32, MXQ_NVFP4};
    for (int g = 0; g < 3; g++) {
        const mxq_qtensor *q = ws[g];
        if (q->fmt != fmts[g] || q->layout != MXQ_LAYOUT_CANONICAL || q->rows != out->rows || q->cols != out->cols)
            return MXQ_EINVAL;
        if (out->rows > 0 && (!q->codes || !q->scales)) return MXQ_EINVAL;
    }
    if (out->rows > 0 && !w_nvfp4->tensor_scale) return MXQ_EINVAL;
    size_t bytes[5];
    if (mxq_mixed_weight_bytes(out->n_group, out->cols, bytes) != MXQ_OK) return MXQ_EINVAL;
    MixedPrep q;
    q.n = out->rows;
    q.k = out->cols;
    for (int g = 0; g < 3; g++) q.n_group[g] = out->n_group[g];
    q.choice = out->choice;
    q.group_index = out->group_index;
    q.mx_codes_c = w_mxfp4->codes;
    q.mx_scales_c = w_mxfp4->scales;
    q.i4_codes_c = w_int4->codes;
    q.i4_scales_c = (const float *)w_int4->scales;
    q.nv_codes_c = w_nvfp4->codes;
    q.nv_scales_c = w_nvfp4->scales;
    q.mx_codes = out->mx_codes;
    q.mx_scales = out->mx_scales;
    q.mx_scales_bytes = out->n_group[0] > 0 ? bytes[1] : 0;
    q.i4_codes = out->i4_codes;
    q.i4_scales = out->i4_scales;
    q.nv_vals = out->nv_values;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = launch_mixed_prep(q, s);
    if (e == cudaSuccess && out->n_group[2] > 0 && out->nv_tensor_scale != w_nvfp4->tensor_scale)
        e = cudaMemcpyAsync((void *)out->nv_tensor_scale, w_nvfp4->tensor_scale, sizeof(float),
                            cudaMemcpyDeviceToDevice, s);
    return from_cuda(e);
}

mxq_status mxq_qlinear_mixed_workspace_bytes(int64_t m, const mxq_mixed_weight *w, int32_t ydtype, size_t *bytes) {
    if (!bytes || m < 0 || m >= ((int64_t)1 << 31) || !valid_dtype(ydtype) || !valid_mixed_weight(w)) return MXQ_EINVAL;
    *bytes = mixed_layout(m, w, ydtype).total;
    return MXQ_OK;
}

mxq_status mxq_qlinear_mixed(const mxq_qtensor *xq, const mxq_mixed_weight *w, void *y, int32_t ydtype,
                             void *workspace, size_t workspace_bytes, void *stream) {
    if (!xq || !valid_dtype(ydtype) || !valid_mixed_weight(w)) return MXQ_EINVAL;
    if (xq->fmt != MXQ_MXFP8 || xq->layout != MXQ_LAYOUT_MMA || xq->cols != w->cols) return MXQ_EINVAL;
    const int64_t m = xq->rows, n = w->rows, k = w->cols;
    if (!valid_shape(MXQ_MXFP8, m, k) || m >= ((int64_t)1 << 31)) return MXQ_EINVAL;
    // the GEMM kernels count output tiles and their K stages in 32-bit integers
    const int64_t tiles = ((m + 127) / 128) * ((n + 127) / 128);
    if (tiles >= ((int64_t)1 << 31) || tiles * (k / 16) >= ((int64_t)1 << 31)) return MXQ_EINVAL;
    if (m == 0 || n == 0) return MXQ_OK;
    if (!y || !aligned16(y) || !xq->codes || !xq->scales || !aligned16(xq->codes)) return MXQ_EINVAL;
    size_t need = 0;
    mxq_qlinear_mixed_workspace_bytes(m, w, ydtype, &need);
    if (!workspace) return MXQ_EINVAL;
    if (workspace_bytes < need) return MXQ_ENOSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MXQ_EINVAL;
    const MixedLayout L = mixed_layout(m, w, ydtype);
    uint8_t *ws = (uint8_t *)workspace;
    cudaStream_t s = (cudaStream_t)stream;
    const bool ybf = ydtype == MXQ_BF16;
    cudaError_t e = cudaSuccess;
    const int single = mixed_single_group(w);
    const void *ybuf[3] = {ws + L.y[0], ws + L.y[1], ws + L.y[2]};
    if (single >= 0) ybuf[single] = y;
    auto operands = [&](int fmt, int64_t rows_b, int g) {
        GemmOperands op;
        memset(&op, 0, sizeof(op));
        op.fmt = fmt;
        op.m = m;
        op.n = rows_b;
        op.k = k;
        op.y = (void *)ybuf[g];
        op.y_bf16 = ybf;
        return op;
    };
    if (w->n_group[0] > 0) {   // MXFP4 rows as E4M3 against the MXFP8 codes, block scales on the tensor cores
        GemmOperands op = operands(MXQ_MXFP8, w->n_group[0], 0);
        op.a_codes = xq->codes;
        op.a_scales = xq->scales;
        op.b_codes = w->mx_codes;
        op.b_scales = w->mx_scales;
        e = launch_qlinear(op, s);
    }
    if (e == cudaSuccess && w->n_group[1] > 0) {   // INT4-g32 rows: per-group products, scales in the epilogue
        float *sx = (float *)(ws + L.sx);
        e = launch_mx_scales_f32(xq->scales, m, k, sx, s);
        GemmOperands op = operands(MXQ_INT4_G32, w->n_group[1], 1);
        op.a_codes = xq->codes;
        op.a_scales = sx;
        op.b_codes = w->i4_codes;
        op.b_scales = w->i4_scales;
        if (e == cudaSuccess) e = launch_qlinear_igroup(op, s);
    }
    if (e == cudaSuccess && w->n_group[2] > 0) {   // NVFP4 rows as bf16 against the bf16 activation
        void *abf = ws + L.abf;
        e = launch_dequantize(MXQ_MXFP8, MXQ_LAYOUT_MMA, m, k, xq->codes, xq->scales, nullptr, abf, true, s);
        GemmOperands op = operands(MXQ_NVFP4, w->n_group[2], 2);
        op.a_codes = abf;
        op.b_codes = w->nv_values;
        op.b_tensor_scale = w->nv_tensor_scale;
        if (e == cudaSuccess) e = launch_gemm_bf16(op, s);
    }
    if (e == cudaSuccess && single < 0)
        e = launch_mixed_scatter(ybuf, w->n_group, w->choice, w->group_index, y, ybf, m, n, s);
    return from_cuda(e);
}

}  // extern "C"
