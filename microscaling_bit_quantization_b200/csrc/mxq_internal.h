// mxq_internal.h -- host-side launchers shared between the kernel files and
// the C ABI layer.  Arguments are validated by the C ABI before any call.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

namespace mxq {

constexpr int kMaxCandidates = 8;

// Launch state that belongs to a device: a kernel's dynamic shared memory
// opt-in (cudaFuncSetAttribute) is set per device, and SM counts and
// occupancy differ between devices, so launchers keep such state per device
// index.  Devices 0 .. kMaxDevices-1 are supported.
constexpr int kMaxDevices = 64;

// Index of the current device, or -1 when it cannot be read or is out of range.
inline int current_device_index() {
    int d = -1;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return -1;
    return d;
}

// SM count of the current device (148 when it cannot be read), cached per device.
inline int sm_count() {
    static std::atomic<int> cache[kMaxDevices];
    const int d = current_device_index();
    if (d < 0) return 148;
    int c = cache[d].load(std::memory_order_relaxed);
    if (c <= 0) {
        if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || c <= 0) c = 148;
        cache[d].store(c, std::memory_order_relaxed);
    }
    return c;
}

// Runs `setup` (returning cudaError_t) once per device, on the current device;
// a setup that fails is retried on the next call.  Two threads may both run
// it the first time, which is harmless for attribute settings.
struct PerDeviceOnce {
    std::atomic<bool> done[kMaxDevices];
    template <typename F>
    cudaError_t run(F &&setup) {
        const int d = current_device_index();
        if (d < 0) return cudaErrorInvalidDevice;
        if (done[d].load(std::memory_order_acquire)) return cudaSuccess;
        const cudaError_t e = setup();
        if (e == cudaSuccess) done[d].store(true, std::memory_order_release);
        return e;
    }
};

// Launch attribute of the kernels on the activation -> GEMM chain
// (k_lowrank_tc, k_quantize, k_gemm): the kernel may be scheduled while
// the previous kernel in the stream finishes; it overlaps only its setup
// (barriers, TMEM, launch latency) and waits (pdl_wait) before touching
// global memory.
inline cudaLaunchAttribute pdl_attribute() {
    cudaLaunchAttribute a;
    a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a.val.programmaticStreamSerializationAllowed = 1;
    return a;
}

// Workspace of mxq_quantize_lowrank: the amax word at 0, the per-warp maxima
// of k_lowrank_tc from byte 256 (at most kAmaxSlots), T from kLrHeader.
constexpr size_t kLrHeader = 4096;
constexpr int kAmaxSlots = (int)((kLrHeader - 256) / 4);

cudaError_t launch_amax(const void *x, bool bf16, int64_t rows, int64_t cols, int hadamard_b,
                        unsigned int *amax_word, cudaStream_t s);
// Optional duty of the quantizer: pack the low-rank activation t (rows x r
// fp32) into tp (rows x 64 bf16) divided by s_x * *w_ts (tensor-scaled
// formats) or by 1.
struct PackT {
    const float *t;
    int r;
    const float *w_ts;
    void *tp;
};
// amax_ready: the tensor amax is already in *amax_word (skip the amax pass).
cudaError_t launch_quantize(const void *x, bool bf16, int64_t rows, int64_t cols, int fmt, int hadamard_b,
                            int layout, void *codes, void *scales, size_t scales_bytes, float *tensor_scale,
                            unsigned int *amax_word, cudaStream_t s, const PackT *pack = nullptr,
                            bool amax_ready = false, float mx_grid = 1.0f, const float *amax_slots = nullptr,
                            int n_slots = 0);
// Squared error of the (rotated) tensor under MX quantization with each of
// n <= kMaxCandidates grid scales (mse.cu); sse: device double[n].
size_t mx_grid_workspace_bytes(int64_t rows, int64_t cols, int n);
// Activation-format calibration (mse.cu): adds each candidate's squared
// error to sse_accum[j] and (sum x^2, sum x^4) to moments_accum[0..1].
size_t calib_workspace_bytes(int64_t rows, int64_t cols, int ncand);
cudaError_t launch_calibrate(const void *x, bool bf16, int64_t rows, int64_t cols, const int *cands, int ncand,
                             double *sse_accum, double *moments_accum, void *workspace, cudaStream_t s);
cudaError_t launch_calib_pick(const double *sse_accum, const int *cands, int ncand, int forced, uint8_t *entry,
                              cudaStream_t s);
cudaError_t launch_fit_mx_grid(const void *w, bool bf16, int64_t rows, int64_t cols, int fmt, int hadamard_b,
                               const float *grid_scales, int n, double *sse, void *workspace, cudaStream_t s);
// NVFP4 with block and tensor scales fitted to the squared error (mse.cu);
// workspace of mse_workspace_bytes, 256-byte aligned.
size_t mse_workspace_bytes(int64_t rows, int64_t cols);
cudaError_t launch_quantize_mse(const void *w, bool bf16, int64_t rows, int64_t cols, int iters, int layout,
                                void *codes, void *scales, size_t scales_bytes, float *tensor_scale, double *sse,
                                void *workspace, cudaStream_t s);
cudaError_t launch_dequantize(int fmt, int layout, int64_t rows, int64_t cols, const void *codes,
                              const void *scales, const float *tensor_scale, void *y, bool bf16_out,
                              cudaStream_t s);
cudaError_t launch_hadamard(const void *x, void *y, bool bf16, int64_t rows, int64_t cols, int b,
                            cudaStream_t s);
cudaError_t launch_cast(const float *x, int64_t n, int elem, uint8_t *out, cudaStream_t s);
cudaError_t launch_select(const void *w, bool bf16, int64_t n, int64_t k, const int *cands, int ncand,
                          uint8_t *choice, double *sse, unsigned int *amax_word, cudaStream_t s);
// The same selection for the fixed candidate sets {MXFP4, NVFP4, INT4_G32}
// and {MXFP8, INT8_ROW, FP8_TENSOR} (any order) with k % 64 == 0, by a kernel
// specialized to the set; amax_slots: room for 2 x SM-count floats (the
// per-CTA maxima of the tensor-amax pass).  Returns cudaErrorNotSupported,
// launching nothing, for other sets and shapes.
cudaError_t launch_select_fixed(const void *w, bool bf16, int64_t n, int64_t k, const int *cands, int ncand,
                                uint8_t *choice, double *sse, float *amax_slots, cudaStream_t s);

// t (m x r fp32) when tp is null; else the packed GEMM operand tp (m x 64
// bf16, [hi | lo] of t / (xs * ws), xs = ws = null meaning 1).  With
// amax_word (and tp null) the max |x| of the whole tensor is also
// atomically folded into *amax_word (which must be zeroed beforehand); with
// amax_slots instead, one maximum per CTA is written to amax_slots (every
// slot written, *n_slots of them, so nothing needs clearing), or
// cudaErrorNotSupported (nothing launched) when more than kAmaxSlots CTAs
// would be needed.
cudaError_t launch_lowrank_down(const void *x, bool bf16, int64_t m, int64_t k, const void *l1, int r,
                                float *t, const float *xs, const float *ws, void *tp, cudaStream_t s,
                                unsigned int *amax_word = nullptr, float *amax_slots = nullptr,
                                int *n_slots = nullptr);
// Tensor-core down-projection of bf16 x (one pass over x): writes t (m x r
// fp32) or, when t is null, the packed operand tp (as launch_lowrank_down);
// with amax_word (zeroed beforehand) also folds in max |x|.  Returns
// cudaErrorNotSupported, launching nothing, for shapes it does not take
// (k % 8, unaligned x, a K slice that does not fit in shared memory).
// amax_slots: null, or room for kAmaxSlots floats receiving per-warp maxima
// of |x| (*n_slots of them, every one written).  cudaErrorNotSupported: a
// shape this kernel does not take (nothing launched).
cudaError_t launch_lowrank_tc(const void *x, int64_t m, int64_t k, const void *l1, int r, float *t, void *tp,
                              const float *xs, const float *ws, float *amax_slots, int *n_slots, cudaStream_t s);
cudaError_t launch_pack_l2(const void *l2, int r, int64_t n, void *l2p, cudaStream_t s);
cudaError_t launch_pack_t(const float *t, int r, int64_t m, const float *xs, const float *ws, void *tp,
                          cudaStream_t s);

struct GemmOperands {
    int fmt;
    int64_t m, n, k;
    const void *a_codes, *b_codes;         // MMA layout
    const void *a_scales, *b_scales;       // byte scales (MMA layout) or fp32 row scales (INT8)
    const float *a_tensor_scale, *b_tensor_scale;
    const void *tp;                        // packed low-rank activation (m x 64 bf16) or null
    const void *l2p;                       // packed up-projection (n x 64 bf16)
    void *y;
    bool y_bf16;
};
cudaError_t launch_qlinear(const GemmOperands &op, cudaStream_t s);
// bf16 x bf16 operands (a_codes m x k, b_codes n x k, k % 16 == 0) on the
// same kernel with kind::f16 MMAs; y = acc * (*b_tensor_scale, or 1 when
// null); no low-rank branch (tp must be null).
cudaError_t launch_gemm_bf16(const GemmOperands &op, cudaStream_t s);
// INT4_G32 / INT4_G64 operands (E4M3 code bytes, transposed fp32 group scales).
cudaError_t launch_qlinear_igroup(const GemmOperands &op, cudaStream_t s);

// 2-D tiled tensor map (row-major, `row_bytes` between rows) through the
// driver entry point; false when the driver rejects it.
bool encode_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz);

// Per-channel mixed weight formats (mixed.cu).  Groups in the order MXFP4,
// INT4_G32, NVFP4; group_index[n] is channel n's row in its group.
struct MixedPrep {
    int64_t n, k, n_group[3];
    const uint8_t *choice;                  // device uint8[n]
    const int32_t *group_index;             // device int32[n]
    const void *mx_codes_c, *mx_scales_c;   // the whole weight in canonical MXFP4
    const void *i4_codes_c;                 // ... in canonical INT4_G32
    const float *i4_scales_c;
    const void *nv_codes_c, *nv_scales_c;   // ... in canonical NVFP4
    void *mx_codes, *mx_scales;             // outputs (see mxq_mixed_weight in mxq.h)
    size_t mx_scales_bytes;
    void *i4_codes;
    float *i4_scales;
    void *nv_vals;
};
cudaError_t launch_mixed_prep(const MixedPrep &q, cudaStream_t s);
// E8M0 scales (MMA layout) of an m x k MX tensor as fp32 [k/32][m].
cudaError_t launch_mx_scales_f32(const void *scales_mma, int64_t m, int64_t k, float *out, cudaStream_t s);
cudaError_t launch_mixed_scatter(const void *const ybuf[3], const int64_t n_group[3], const uint8_t *choice,
                                 const int32_t *group_index, void *y, bool y_bf16, int64_t m, int64_t n,
                                 cudaStream_t s);

// Device error word (bounded waits that ran out); read-and-clear, and its
// device address on the current device (for kernels of other files).
cudaError_t read_and_clear_error(unsigned int *value);
// W4A16 linear (w4a16.cu): y = bf16(x) . bf16(RN32(q s))^T, x m x k bf16,
// codes n x k/2 canonical INT4, scales n x k/g fp32; k % 64 == 0.
cudaError_t launch_w4a16(const void *x, int64_t m, int64_t k, const uint8_t *codes, const float *scales, int64_t n,
                         int g, void *y, bool y_bf16, cudaStream_t s);
// One bounded wait that runs out (gemm.cu): latches the error word.
cudaError_t launch_wait_selftest(unsigned long long limit_ns, cudaStream_t s);
cudaError_t error_word_address(unsigned int **ptr);

}  // namespace mxq
