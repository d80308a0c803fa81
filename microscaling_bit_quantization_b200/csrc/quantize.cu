// quantize.cu -- HBM-bound kernels of the hot path: tensor amax, fused
// block-diagonal Hadamard + block-scaled quantization, dequantization,
// standalone Hadamard, element casts, and per-channel format selection.
//
// Work mapping shared by all kernels: a row of `cols` elements is cut into
// 16-element chunks; lane i of a warp owns chunk (32*w + i), so a warp reads
// 32 consecutive chunks (1 KB of bf16) and every quantization block (16, 32
// or 64 elements) or Hadamard block (<= 256 elements) lies in aligned lanes
// of one warp.  Block maxima and cross-lane butterflies use warp shuffles.
// Loads are 16-byte vectors; codes are stored as 8- or 16-byte vectors.
#include <cuda_runtime.h>

#include <cstring>

#include "mxq_formats.cuh"
#include "mxq_internal.h"

namespace mxq {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

// Number of CTAs for a grid-stride loop over `warp_tiles` warp tiles.
inline int grid_for(int64_t warp_tiles, int sm_count) {
    int64_t ctas = (warp_tiles + (kThreads / 32) - 1) / (kThreads / 32);
    int64_t cap = (int64_t)sm_count * 8;
    return (int)(ctas < 1 ? 1 : (ctas > cap ? cap : ctas));
}

// ------------------------------------------------------------------ amax

// Max over the CTA, then one atomicMax on the word (non-negative floats
// order like their bit patterns).  All threads of the CTA must call this.
__device__ __forceinline__ void cta_max_to_word(float m, unsigned int *word) {
    __shared__ float wmax[kThreads / 32];
    m = group_max<32>(m);
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < kThreads / 32 ? wmax[threadIdx.x] : 0.0f;
        v = group_max<32>(v);
        if (threadIdx.x == 0 && v > 0.0f) atomicMax(word, __float_as_uint(v));
    }
}

// Bytes of four consecutive scale columns s..s+3 (held by lanes lane,
// lane+L, lane+2L, lane+3L) as one little-endian word, for the lane whose
// scale column is a multiple of 4.  All lanes must call this.
template <int L>
__device__ __forceinline__ uint32_t gather4(uint32_t byte) {
    uint32_t b1 = __shfl_down_sync(0xFFFFFFFFu, byte, L);
    uint32_t b2 = __shfl_down_sync(0xFFFFFFFFu, byte, 2 * L);
    uint32_t b3 = __shfl_down_sync(0xFFFFFFFFu, byte, 3 * L);
    return (byte & 0xFFu) | ((b1 & 0xFFu) << 8) | ((b2 & 0xFFu) << 16) | ((b3 & 0xFFu) << 24);
}

// ------------------------------------------------------------------ quantize

struct QuantArgs {
    int64_t rows, cols, total_chunks;
    int hadamard_b;
    int layout;              // 0 canonical, 1 MMA
    int64_t s_pad;           // padded scale columns (MMA layout)
    uint8_t *codes;
    void *scales;
    float *tensor_scale;     // written by chunk 0 (NVFP4, FP8_TENSOR)
    const unsigned int *amax_word;
    int combine;             // scale bytes stored as 32-bit words (scale columns per row % 4 == 0)
    // optional packed low-rank operand: tp[row] = [hi | lo] of t[row] / (s_x * *w_ts)
    const float *t;
    int r;
    const float *w_ts;
    __nv_bfloat16 *tp;
    unsigned int *err;       // device error word (a bounded wait that ran out)
};

// Staged input: persistent CTAs bring 16 KB tiles of x into a ring of
// kQStages shared-memory buffers with one cp.async.bulk each (completion on
// an mbarrier), then encode from shared memory.
constexpr int kQStages = 4, kQTileBytes = 16384, kQSmem = kQStages * kQTileBytes;
constexpr unsigned int kErrTimeoutQuant = 8u;

__device__ __forceinline__ uint32_t smem_addr(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void q_bar_init(uint64_t *bar) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(bar)));
}
__device__ __forceinline__ void q_bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(dst)),
                 "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}
// Bounded wait (about 2 s of polling) for phase `parity` of the barrier.
__device__ __forceinline__ bool q_bar_wait(uint64_t *bar, uint32_t parity) {
    for (long long i = 0; i < (1ll << 26); i++) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_addr(bar)), "r"(parity)
            : "memory");
        if (ok) return true;
    }
    return false;
}

__device__ __forceinline__ void load16_shared(const float *p, float v[16]) {
    const float4 *q = reinterpret_cast<const float4 *>(p);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        float4 t = q[i];
        v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
    }
}
__device__ __forceinline__ void load16_shared(const __nv_bfloat16 *p, float v[16]) {
    const uint4 *q = reinterpret_cast<const uint4 *>(p);
#pragma unroll
    for (int i = 0; i < 2; i++) {
        uint4 t = q[i];
        uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
            v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
            v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    }
}

template <typename T, int F>
__global__ void __launch_bounds__(kThreads) k_quantize(const T *__restrict__ x, QuantArgs a) {
    constexpr int BLK = fmt_block(F) ? fmt_block(F) : 16;
    constexpr int G = BLK ? BLK / 16 : 1;   // lanes per quantization block
    constexpr int CPT = kQTileBytes / (16 * (int)sizeof(T));   // chunks per staged tile
    extern __shared__ __align__(128) uint8_t q_smem[];
    __shared__ uint64_t q_bars[kQStages];
    const int lane = lane_id();
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t ntiles = (a.total_chunks + CPT - 1) / CPT;
    const int64_t chunks_per_row = a.cols >> 4;
    auto issue = [&](int64_t tile, int stage) {
        const int64_t n = a.total_chunks - tile * CPT;
        const uint32_t bytes = (uint32_t)((n < CPT ? n : CPT) * 16 * (int64_t)sizeof(T));
        q_bulk_load(q_smem + stage * kQTileBytes, x + tile * CPT * 16, bytes, &q_bars[stage]);
    };
    if (threadIdx.x == 0) {
        for (int i = 0; i < kQStages; i++) q_bar_init(&q_bars[i]);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int i = 0; i < kQStages; i++) {
            const int64_t tile = blockIdx.x + (int64_t)i * gridDim.x;
            if (tile < ntiles) issue(tile, i);
        }
    }
    __syncthreads();

    float s_t = 1.0f;
    if (F == kNVFP4 || F == kFP8Tensor) {
        float amax_t = __uint_as_float(*a.amax_word);
        s_t = F == kNVFP4 ? nvfp4_tensor_scale(amax_t) : fp8_tensor_scale(amax_t);
        if (blockIdx.x == 0 && threadIdx.x == 0) *a.tensor_scale = s_t;
    }

    bool failed = false;
    float tensor_max = 0.0f;
    int64_t it = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, it++) {
      const int stage = (int)(it % kQStages);
      if (!q_bar_wait(&q_bars[stage], (uint32_t)((it / kQStages) & 1))) {
          failed = true;
          break;
      }
      const T *tx = reinterpret_cast<const T *>(q_smem + stage * kQTileBytes);
#pragma unroll 1
      for (int jc = 0; jc < CPT / kThreads; jc++) {
        const int cit = threadIdx.x + jc * kThreads;   // chunk within the tile
        const int64_t c = tile * CPT + cit;
        const bool valid = c < a.total_chunks;
        float v[16];
        if (valid) load16_shared(tx + cit * 16, v);
        else {
#pragma unroll
            for (int i = 0; i < 16; i++) v[i] = 0.0f;
        }
        if (a.hadamard_b) hadamard_chunk(v, a.hadamard_b, lane);
        const int64_t row = c / chunks_per_row;
        const int64_t col0 = (c - row * chunks_per_row) << 4;
        float amax = amax16(v);
        if (F == kNumFmt) {   // tensor-amax pass only
            tensor_max = fmaxf(tensor_max, amax);
            continue;
        }
        if (G > 1) amax = group_max<G>(amax);

        if (F == kMXFP8 || F == kMXFP4) {
            float inv = 0.0f;
            uint32_t sb = 127;
            if (amax > 0.0f) sb = mx_scale(amax, F == kMXFP8 ? 8 : 2, inv);
            if (valid) {
                if (F == kMXFP8) {
                    uint32_t w[4];
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        uint32_t b0 = 0, b1 = 0, b2 = 0, b3 = 0;
                        if (amax > 0.0f) {
                            b0 = enc_e4m3(__fmul_rn(v[4 * j], inv));
                            b1 = enc_e4m3(__fmul_rn(v[4 * j + 1], inv));
                            b2 = enc_e4m3(__fmul_rn(v[4 * j + 2], inv));
                            b3 = enc_e4m3(__fmul_rn(v[4 * j + 3], inv));
                        }
                        w[j] = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
                    }
                    *reinterpret_cast<uint4 *>(a.codes + c * 16) = make_uint4(w[0], w[1], w[2], w[3]);
                } else {
                    uint32_t w[2];
#pragma unroll
                    for (int j = 0; j < 2; j++) {
                        uint32_t acc = 0;
#pragma unroll
                        for (int k = 0; k < 4; k++) {
                            uint32_t byte = 0;
                            if (amax > 0.0f)
                                byte = enc_e2m1x2(__fmul_rn(v[8 * j + 2 * k], inv), __fmul_rn(v[8 * j + 2 * k + 1], inv));
                            acc |= byte << (8 * k);
                        }
                        w[j] = acc;
                    }
                    *reinterpret_cast<uint2 *>(a.codes + c * 8) = make_uint2(w[0], w[1]);
                }
            }
            const uint32_t word = gather4<2>(sb);
            if (valid) {
                const int64_t s = col0 >> 5;
                uint8_t *sc = reinterpret_cast<uint8_t *>(a.scales);
                const int64_t off = a.layout == 0 ? row * (a.cols >> 5) + s : mma_scale_offset(row, s, a.s_pad);
                if (a.combine) {
                    if ((lane & 7) == 0) *reinterpret_cast<uint32_t *>(sc + off) = word;
                } else if ((lane & 1) == 0) {
                    sc[off] = (uint8_t)sb;
                }
            }
        } else if (F == kNVFP4) {
            float d;
            uint32_t e4 = nvfp4_block_scale(amax, s_t, d);
            if (valid) {
                const Recip rd = recip_of(d);
                uint32_t w[2];
#pragma unroll
                for (int j = 0; j < 2; j++) {
                    uint32_t acc = 0;
#pragma unroll
                    for (int k = 0; k < 4; k++) {
                        uint32_t byte = 0;
                        if (e4) byte = e2m1x2_quot(v[8 * j + 2 * k], v[8 * j + 2 * k + 1], rd);
                        acc |= byte << (8 * k);
                    }
                    w[j] = acc;
                }
                *reinterpret_cast<uint2 *>(a.codes + c * 8) = make_uint2(w[0], w[1]);
            }
            const uint32_t word = gather4<1>(e4);
            if (valid) {
                const int64_t s = col0 >> 4;
                uint8_t *sc = reinterpret_cast<uint8_t *>(a.scales);
                const int64_t off = a.layout == 0 ? c : mma_scale_offset(row, s, a.s_pad);
                if (a.combine) {
                    if ((lane & 3) == 0) *reinterpret_cast<uint32_t *>(sc + off) = word;
                } else {
                    sc[off] = (uint8_t)e4;
                }
            }
        } else if (F == kINT4G32 || F == kINT4G64) {
            float s = __fdiv_rn(amax, 7.0f);
            const Recip rs = recip_of(s);
            if (valid) {
                if (a.layout == 0) {
                    uint32_t w[2];
#pragma unroll
                    for (int j = 0; j < 2; j++) {
                        uint32_t acc = 0;
#pragma unroll
                        for (int k = 0; k < 8; k++) acc |= ((uint32_t)int_code_quot(v[8 * j + k], rs, 7) & 0xFu) << (4 * k);
                        w[j] = acc;
                    }
                    *reinterpret_cast<uint2 *>(a.codes + c * 8) = make_uint2(w[0], w[1]);
                } else {
                    uint32_t w[4];
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        uint32_t acc = 0;
#pragma unroll
                        for (int k = 0; k < 4; k++) acc |= ((uint32_t)int_code_quot(v[4 * j + k], rs, 7) & 0xFFu) << (8 * k);
                        w[j] = acc;
                    }
                    *reinterpret_cast<uint4 *>(a.codes + c * 16) = make_uint4(w[0], w[1], w[2], w[3]);
                }
                if ((lane & (G - 1)) == 0) {
                    float *sc = reinterpret_cast<float *>(a.scales);
                    int64_t g = col0 / BLK;
                    if (a.layout == 0) sc[row * (a.cols / BLK) + g] = s;
                    else sc[g * a.rows + row] = s;
                }
            }
        } else if (F == kFP8Tensor) {
            if (valid) {
                const Recip rs = recip_of(s_t);
                uint32_t w[4];
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    uint32_t acc = 0;
#pragma unroll
                    for (int k = 0; k < 4; k++) acc |= e4m3_quot(v[4 * j + k], rs) << (8 * k);
                    w[j] = acc;
                }
                *reinterpret_cast<uint4 *>(a.codes + c * 16) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
      }
      __syncthreads();   // the stage is free again
      if (threadIdx.x == 0) {
          const int64_t next = tile + (int64_t)kQStages * gridDim.x;
          if (next < ntiles) issue(next, stage);
      }
    }
    if (failed) {
        if (threadIdx.x == 0) atomicOr(a.err, kErrTimeoutQuant);
        return;
    }
    if (F == kNumFmt) {
        cta_max_to_word(tensor_max, const_cast<unsigned int *>(a.amax_word));
        return;
    }
    if (a.tp) {
        // packed low-rank operand, one row per warp, one value per lane:
        // u = t / alpha, hi = bf16(u), lo = bf16(u - hi), zeros past r
        const bool ts = F == kNVFP4 || F == kFP8Tensor;
        const float alpha = ts ? __fmul_rn(s_t, *a.w_ts) : 1.0f;
        for (int64_t row = warp; row < a.rows; row += nwarps) {
            float u = lane < a.r ? a.t[row * a.r + lane] : 0.0f;
            if (ts) u = __fdiv_rn(u, alpha);
            const __nv_bfloat16 hi = __float2bfloat16_rn(u);
            a.tp[row * 64 + lane] = hi;
            a.tp[row * 64 + 32 + lane] = __float2bfloat16_rn(__fsub_rn(u, __bfloat162float(hi)));
        }
    }
}

// INT8 per row: one warp per row, two passes (row amax, then codes).
template <typename T>
__global__ void __launch_bounds__(kThreads) k_quantize_int8_row(const T *__restrict__ x, QuantArgs a) {
    const int lane = lane_id();
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t cpr = a.cols >> 4;
    for (int64_t row = warp; row < a.rows; row += nwarps) {
        const T *xr = x + row * a.cols;
        float m = 0.0f;
        for (int64_t c0 = 0; c0 < cpr; c0 += 32) {
            int64_t c = c0 + lane;
            float v[16];
            if (c < cpr) load16(xr + c * 16, v);
            else {
#pragma unroll
                for (int i = 0; i < 16; i++) v[i] = 0.0f;
            }
            if (a.hadamard_b) hadamard_chunk(v, a.hadamard_b, lane);
            m = fmaxf(m, amax16(v));
        }
        m = group_max<32>(m);
        const float s = __fdiv_rn(m, 127.0f);
        const Recip rs = recip_of(s);
        for (int64_t c0 = 0; c0 < cpr; c0 += 32) {
            int64_t c = c0 + lane;
            float v[16];
            if (c < cpr) load16(xr + c * 16, v);
            else {
#pragma unroll
                for (int i = 0; i < 16; i++) v[i] = 0.0f;
            }
            if (a.hadamard_b) hadamard_chunk(v, a.hadamard_b, lane);
            if (c < cpr) {
                uint32_t w[4];
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    uint32_t acc = 0;
#pragma unroll
                    for (int k = 0; k < 4; k++) acc |= ((uint32_t)int_code_quot(v[4 * j + k], rs, 127) & 0xFFu) << (8 * k);
                    w[j] = acc;
                }
                *reinterpret_cast<uint4 *>(a.codes + (row * cpr + c) * 16) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
        if (lane == 0) reinterpret_cast<float *>(a.scales)[row] = s;
    }
}

// ------------------------------------------------------------------ dequantize

struct DequantArgs {
    int64_t rows, cols, total_chunks;
    int layout;
    int64_t s_pad;
    const uint8_t *codes;
    const void *scales;
    const float *tensor_scale;
};

template <int F>
__device__ __forceinline__ void dequant_chunk(const DequantArgs &a, int64_t c, float out[16]) {
    constexpr int BLK = fmt_block(F) ? fmt_block(F) : 16;
    const int64_t cpr = a.cols >> 4;
    const int64_t row = c / cpr;
    const int64_t col0 = (c - row * cpr) << 4;
    uint32_t code[16];
    const bool unpacked_int4 = (F == kINT4G32 || F == kINT4G64) && a.layout == 1;
    if (fmt_is4(F) && !unpacked_int4) {
        uint2 w = *reinterpret_cast<const uint2 *>(a.codes + c * 8);
        uint32_t ww[2] = {w.x, w.y};
#pragma unroll
        for (int i = 0; i < 16; i++) code[i] = (ww[i >> 3] >> (4 * (i & 7))) & 0xFu;
    } else {
        uint4 w = *reinterpret_cast<const uint4 *>(a.codes + c * 16);
        uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 16; i++) code[i] = (ww[i >> 2] >> (8 * (i & 3))) & 0xFFu;
    }
    const uint8_t *sb = reinterpret_cast<const uint8_t *>(a.scales);
    const float *sf = reinterpret_cast<const float *>(a.scales);
    if (F == kMXFP8 || F == kMXFP4) {
        int64_t s = col0 >> 5;
        float X = dec_e8m0(a.layout == 0 ? sb[row * (a.cols >> 5) + s] : sb[mma_scale_offset(row, s, a.s_pad)]);
#pragma unroll
        for (int i = 0; i < 16; i++) out[i] = __fmul_rn(F == kMXFP8 ? dec_e4m3(code[i]) : dec_e2m1(code[i]), X);
    } else if (F == kNVFP4) {
        int64_t s = col0 >> 4;
        float e4 = dec_e4m3(a.layout == 0 ? sb[c] : sb[mma_scale_offset(row, s, a.s_pad)]);
        float st = *a.tensor_scale;
#pragma unroll
        for (int i = 0; i < 16; i++) out[i] = __fmul_rn(__fmul_rn(dec_e2m1(code[i]), e4), st);
    } else if (F == kINT4G32 || F == kINT4G64) {
        int64_t g = col0 / BLK;
        float s = a.layout == 0 ? sf[row * (a.cols / BLK) + g] : sf[g * a.rows + row];
#pragma unroll
        for (int i = 0; i < 16; i++) {
            int q = unpacked_int4 ? (int)(int8_t)code[i] : ((code[i] & 8u) ? (int)code[i] - 16 : (int)code[i]);
            out[i] = __fmul_rn((float)q, s);
        }
    } else if (F == kINT8Row) {
        float s = sf[row];
#pragma unroll
        for (int i = 0; i < 16; i++) out[i] = __fmul_rn((float)(int8_t)code[i], s);
    } else {
        float s = *a.tensor_scale;
#pragma unroll
        for (int i = 0; i < 16; i++) out[i] = __fmul_rn(dec_e4m3(code[i]), s);
    }
}

template <typename T, int F>
__global__ void __launch_bounds__(kThreads) k_dequantize(DequantArgs a, T *__restrict__ y) {
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t c = (int64_t)blockIdx.x * kThreads + threadIdx.x; c < a.total_chunks; c += stride) {
        float v[16];
        dequant_chunk<F>(a, c, v);
        store16(y + c * 16, v);
    }
}

// ------------------------------------------------------------------ Hadamard

template <typename T>
__global__ void __launch_bounds__(kThreads) k_hadamard(const T *x, T *y, int64_t total_chunks, int b) {
    const int lane = lane_id();
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t tiles = (total_chunks + 31) >> 5;
    for (int64_t t = warp; t < tiles; t += nwarps) {
        int64_t c = (t << 5) + lane;
        float v[16];
        if (c < total_chunks) load16(x + c * 16, v);
        else {
#pragma unroll
            for (int i = 0; i < 16; i++) v[i] = 0.0f;
        }
        hadamard_chunk(v, b, lane);
        if (c < total_chunks) store16(y + c * 16, v);
    }
}

// ------------------------------------------------------------------ cast

__global__ void __launch_bounds__(kThreads) k_cast(const float *__restrict__ x, int64_t n, int elem,
                                                  uint8_t *__restrict__ out) {
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n; i += stride) {
        float v = x[i];
        out[i] = elem == 0 ? enc_e4m3(v) : (uint8_t)(enc_e2m1x2(v, 0.0f) & 0xFu);
    }
}

// ------------------------------------------------------------------ selection

struct SelectArgs {
    int64_t n, k;
    int ncand;
    int cand[kMaxCandidates];
    const unsigned int *amax_word;   // tensor amax of w
    uint8_t *choice;
    double *sse;                     // may be null
};

// Squared reconstruction error of one 16-element chunk under format F,
// binary64, from the exact dequantized values.  `amax` is the block max
// (already reduced over the block's lanes), `rowamax` the row max, `tamax`
// the tensor max.
__device__ __forceinline__ double chunk_sse(int F, const float v[16], float amax, float rowamax, float tamax) {
    double acc = 0.0;
    auto add = [&](int i, double deq) {
        double d = __dsub_rn((double)v[i], deq);
        acc = __dadd_rn(acc, __dmul_rn(d, d));
    };
    if (F == kMXFP8 || F == kMXFP4) {
        if (amax == 0.0f) {
#pragma unroll
            for (int i = 0; i < 16; i++) add(i, 0.0);
            return acc;
        }
        float inv;
        int e = (int)mx_scale(amax, F == kMXFP8 ? 8 : 2, inv) - 127;
        double X = exp2i_f64(e);
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            float a0 = __fmul_rn(v[i], inv), a1 = __fmul_rn(v[i + 1], inv);
            double q0, q1;
            if (F == kMXFP8) {
                q0 = dec_e4m3(enc_e4m3(a0));
                q1 = dec_e4m3(enc_e4m3(a1));
            } else {
                uint32_t b = enc_e2m1x2(a0, a1);
                q0 = dec_e2m1(b & 0xFu);
                q1 = dec_e2m1(b >> 4);
            }
            add(i, q0 * X);
            add(i + 1, q1 * X);
        }
    } else if (F == kNVFP4) {
        float st = nvfp4_tensor_scale(tamax), d;
        uint32_t e4 = nvfp4_block_scale(amax, st, d);
        double S = (double)dec_e4m3(e4) * (double)st;
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            double q0 = 0.0, q1 = 0.0;
            if (e4) {
                uint32_t b = enc_e2m1x2(__fdiv_rn(v[i], d), __fdiv_rn(v[i + 1], d));
                q0 = dec_e2m1(b & 0xFu);
                q1 = dec_e2m1(b >> 4);
            }
            add(i, q0 * S);
            add(i + 1, q1 * S);
        }
    } else if (F == kINT4G32 || F == kINT4G64 || F == kINT8Row) {
        float s = F == kINT8Row ? __fdiv_rn(rowamax, 127.0f) : __fdiv_rn(amax, 7.0f);
        int qmax = F == kINT8Row ? 127 : 7;
#pragma unroll
        for (int i = 0; i < 16; i++) add(i, (double)int_code(v[i], s, qmax) * (double)s);
    } else {   // FP8 tensor
        float s = fp8_tensor_scale(tamax);
#pragma unroll
        for (int i = 0; i < 16; i++) add(i, (double)dec_e4m3(enc_e4m3(__fdiv_rn(v[i], s))) * (double)s);
    }
    return acc;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) k_select(const T *__restrict__ w, SelectArgs a) {
    const int lane = lane_id();
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t cpr = a.k >> 4;
    const float tamax = a.amax_word ? __uint_as_float(*a.amax_word) : 0.0f;
    bool need_row = false;
    for (int j = 0; j < a.ncand; j++) need_row |= a.cand[j] == kINT8Row;
    for (int64_t row = warp; row < a.n; row += nwarps) {
        const T *wr = w + row * a.k;
        float rowamax = 0.0f;
        if (need_row) {
            for (int64_t c0 = 0; c0 < cpr; c0 += 32) {
                float v[16];
                if (c0 + lane < cpr) {
                    load16(wr + (c0 + lane) * 16, v);
                    rowamax = fmaxf(rowamax, amax16(v));
                }
            }
            rowamax = group_max<32>(rowamax);
        }
        double sse[kMaxCandidates];
#pragma unroll
        for (int j = 0; j < kMaxCandidates; j++) sse[j] = 0.0;
        for (int64_t c0 = 0; c0 < cpr; c0 += 32) {
            const int64_t c = c0 + lane;
            const bool valid = c < cpr;
            float v[16];
            if (valid) load16(wr + c * 16, v);
            else {
#pragma unroll
                for (int i = 0; i < 16; i++) v[i] = 0.0f;
            }
            const float m1 = amax16(v);
            const float m2 = group_max<2>(m1);
            const float m4 = group_max<4>(m2);
#pragma unroll
            for (int j = 0; j < kMaxCandidates; j++) {
                if (j < a.ncand) {
                    int F = a.cand[j];
                    float bm = F == kNVFP4 ? m1 : (F == kINT4G64 ? m4 : m2);
                    double e = chunk_sse(F, v, bm, rowamax, tamax);
                    if (valid) sse[j] = __dadd_rn(sse[j], e);
                }
            }
        }
        int best = 0;
        double bestv = 0.0;
#pragma unroll
        for (int j = 0; j < kMaxCandidates; j++) {
            if (j < a.ncand) {
                double s = sse[j];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) s = __dadd_rn(s, __shfl_xor_sync(0xFFFFFFFFu, s, o));
                if (a.sse && lane == 0) a.sse[row * a.ncand + j] = s;
                if (j == 0 || s < bestv) {
                    best = j;
                    bestv = s;
                }
            }
        }
        if (lane == 0) a.choice[row] = (uint8_t)a.cand[best];
    }
}

}  // namespace

// ====================================================================== host

static int sm_count_cached() {
    static int count = 0;
    if (!count) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev);
        if (count <= 0) count = 148;
    }
    return count;
}

template <typename T, int F>
static void launch_qf(const T *x, const QuantArgs &a, cudaStream_t s);

cudaError_t launch_amax(const void *x, bool bf16, int64_t rows, int64_t cols, int hadamard_b,
                        unsigned int *amax_word, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(amax_word, 0, sizeof(unsigned int), s);
    if (e != cudaSuccess) return e;
    int64_t chunks = rows * cols / 16;
    if (chunks == 0) return cudaSuccess;
    QuantArgs a;
    memset(&a, 0, sizeof(a));
    a.rows = rows;
    a.cols = cols;
    a.total_chunks = chunks;
    a.hadamard_b = hadamard_b;
    a.amax_word = amax_word;
    e = error_word_address(&a.err);
    if (e != cudaSuccess) return e;
    if (bf16) launch_qf<__nv_bfloat16, kNumFmt>((const __nv_bfloat16 *)x, a, s);
    else launch_qf<float, kNumFmt>((const float *)x, a, s);
    return cudaGetLastError();
}

template <typename T, int F>
static void launch_qf(const T *x, const QuantArgs &a, cudaStream_t s) {
    static bool configured = false;
    if (!configured) {
        cudaFuncSetAttribute(k_quantize<T, F>, cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmem);
        configured = true;
    }
    constexpr int CPT = kQTileBytes / (16 * (int)sizeof(T));
    const int64_t ntiles = (a.total_chunks + CPT - 1) / CPT;
    const int64_t cap = (int64_t)sm_count_cached() * 3;   // 3 x 64 KB of ring per SM
    const int grid = (int)(ntiles < cap ? ntiles : cap);
    k_quantize<T, F><<<grid, kThreads, kQSmem, s>>>(x, a);
}

template <typename T>
static void launch_q(int fmt, int grid, const T *x, const QuantArgs &a, cudaStream_t s) {
    switch (fmt) {
    case kMXFP8: launch_qf<T, kMXFP8>(x, a, s); break;
    case kMXFP4: launch_qf<T, kMXFP4>(x, a, s); break;
    case kNVFP4: launch_qf<T, kNVFP4>(x, a, s); break;
    case kINT4G32: launch_qf<T, kINT4G32>(x, a, s); break;
    case kINT4G64: launch_qf<T, kINT4G64>(x, a, s); break;
    case kFP8Tensor: launch_qf<T, kFP8Tensor>(x, a, s); break;
    case kINT8Row: {
        int g = grid_for(a.rows, sm_count_cached());
        k_quantize_int8_row<T><<<g, kThreads, 0, s>>>(x, a);
        break;
    }
    }
}

cudaError_t launch_quantize(const void *x, bool bf16, int64_t rows, int64_t cols, int fmt, int hadamard_b,
                            int layout, void *codes, void *scales, size_t scales_bytes, float *tensor_scale,
                            unsigned int *amax_word, cudaStream_t s, const PackT *pack, bool amax_ready) {
    cudaError_t e;
    if (fmt_tensor_scaled(fmt) && !amax_ready) {
        e = launch_amax(x, bf16, rows, cols, hadamard_b, amax_word, s);
        if (e != cudaSuccess) return e;
    }
    QuantArgs a;
    a.rows = rows;
    a.cols = cols;
    a.total_chunks = rows * cols / 16;
    a.hadamard_b = hadamard_b;
    a.layout = layout;
    a.s_pad = 0;
    a.codes = (uint8_t *)codes;
    a.scales = scales;
    a.tensor_scale = tensor_scale;
    a.amax_word = amax_word;
    a.combine = fmt_byte_scales(fmt) && (cols / fmt_block(fmt)) % 4 == 0;
    a.t = pack ? pack->t : nullptr;
    a.r = pack ? pack->r : 0;
    a.w_ts = pack ? pack->w_ts : nullptr;
    a.tp = pack ? (__nv_bfloat16 *)pack->tp : nullptr;
    e = error_word_address(&a.err);
    if (e != cudaSuccess) return e;
    if (layout == 1 && fmt_byte_scales(fmt)) {
        int64_t S = cols / fmt_block(fmt);
        a.s_pad = (S + 15) / 16 * 16;
        if (a.s_pad != S || rows % 128) {   // padding bytes must read as 0
            e = cudaMemsetAsync(scales, 0, scales_bytes, s);
            if (e != cudaSuccess) return e;
        }
    }
    if (a.total_chunks == 0) {
        if (fmt_tensor_scaled(fmt)) {   // empty tensor: amax 0 -> scale 1
            static const float one = 1.0f;
            return cudaMemcpyAsync(tensor_scale, &one, sizeof(float), cudaMemcpyHostToDevice, s);
        }
        return cudaSuccess;
    }
    int grid = grid_for((a.total_chunks + 31) / 32, sm_count_cached());
    if (bf16) launch_q<__nv_bfloat16>(fmt, grid, (const __nv_bfloat16 *)x, a, s);
    else launch_q<float>(fmt, grid, (const float *)x, a, s);
    return cudaGetLastError();
}

template <typename T>
static void launch_dq(int fmt, int grid, const DequantArgs &a, T *y, cudaStream_t s) {
    switch (fmt) {
    case kMXFP8: k_dequantize<T, kMXFP8><<<grid, kThreads, 0, s>>>(a, y); break;
    case kMXFP4: k_dequantize<T, kMXFP4><<<grid, kThreads, 0, s>>>(a, y); break;
    case kNVFP4: k_dequantize<T, kNVFP4><<<grid, kThreads, 0, s>>>(a, y); break;
    case kINT4G32: k_dequantize<T, kINT4G32><<<grid, kThreads, 0, s>>>(a, y); break;
    case kINT4G64: k_dequantize<T, kINT4G64><<<grid, kThreads, 0, s>>>(a, y); break;
    case kINT8Row: k_dequantize<T, kINT8Row><<<grid, kThreads, 0, s>>>(a, y); break;
    case kFP8Tensor: k_dequantize<T, kFP8Tensor><<<grid, kThreads, 0, s>>>(a, y); break;
    }
}

cudaError_t launch_dequantize(int fmt, int layout, int64_t rows, int64_t cols, const void *codes,
                              const void *scales, const float *tensor_scale, void *y, bool bf16_out,
                              cudaStream_t s) {
    DequantArgs a;
    a.rows = rows;
    a.cols = cols;
    a.total_chunks = rows * cols / 16;
    a.layout = layout;
    a.s_pad = fmt_byte_scales(fmt) ? (cols / fmt_block(fmt) + 15) / 16 * 16 : 0;
    a.codes = (const uint8_t *)codes;
    a.scales = scales;
    a.tensor_scale = tensor_scale;
    if (a.total_chunks == 0) return cudaSuccess;
    int grid = grid_for((a.total_chunks + 31) / 32, sm_count_cached());
    if (bf16_out) launch_dq<__nv_bfloat16>(fmt, grid, a, (__nv_bfloat16 *)y, s);
    else launch_dq<float>(fmt, grid, a, (float *)y, s);
    return cudaGetLastError();
}

cudaError_t launch_hadamard(const void *x, void *y, bool bf16, int64_t rows, int64_t cols, int b,
                            cudaStream_t s) {
    int64_t chunks = rows * cols / 16;
    if (chunks == 0) return cudaSuccess;
    int grid = grid_for((chunks + 31) / 32, sm_count_cached());
    if (bf16) k_hadamard<__nv_bfloat16><<<grid, kThreads, 0, s>>>((const __nv_bfloat16 *)x, (__nv_bfloat16 *)y, chunks, b);
    else k_hadamard<float><<<grid, kThreads, 0, s>>>((const float *)x, (float *)y, chunks, b);
    return cudaGetLastError();
}

cudaError_t launch_cast(const float *x, int64_t n, int elem, uint8_t *out, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    int64_t ctas = (n + kThreads - 1) / kThreads;
    int grid = (int)(ctas > (int64_t)sm_count_cached() * 16 ? (int64_t)sm_count_cached() * 16 : ctas);
    k_cast<<<grid, kThreads, 0, s>>>(x, n, elem, out);
    return cudaGetLastError();
}

cudaError_t launch_select(const void *w, bool bf16, int64_t n, int64_t k, const int *cands, int ncand,
                          uint8_t *choice, double *sse, unsigned int *amax_word, cudaStream_t s) {
    bool need_tensor = false;
    for (int j = 0; j < ncand; j++) need_tensor |= fmt_tensor_scaled(cands[j]);
    if (need_tensor) {
        cudaError_t e = launch_amax(w, bf16, n, k, 0, amax_word, s);
        if (e != cudaSuccess) return e;
    }
    if (n == 0) return cudaSuccess;
    SelectArgs a;
    a.n = n;
    a.k = k;
    a.ncand = ncand;
    for (int j = 0; j < kMaxCandidates; j++) a.cand[j] = j < ncand ? cands[j] : 0;
    a.amax_word = need_tensor ? amax_word : nullptr;
    a.choice = choice;
    a.sse = sse;
    int grid = grid_for(n, sm_count_cached());
    if (bf16) k_select<__nv_bfloat16><<<grid, kThreads, 0, s>>>((const __nv_bfloat16 *)w, a);
    else k_select<float><<<grid, kThreads, 0, s>>>((const float *)w, a);
    return cudaGetLastError();
}

}  // namespace mxq
