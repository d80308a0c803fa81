// quantize.cu -- HBM-bound kernels of the hot path: tensor amax, fused
// block-diagonal Hadamard + block-scaled quantization, dequantization,
// standalone Hadamard, element casts, and per-channel format selection.
//
// Work mapping of the chunk kernels: a row of `cols` elements is cut into
// 16-element chunks; lane i of a warp owns chunk (32*w + i), so a warp reads
// 32 consecutive chunks (1 KB of bf16) and every quantization block (16, 32
// or 64 elements) or Hadamard block (<= 256 elements) lies in aligned lanes
// of one warp.  Block maxima and cross-lane butterflies use warp shuffles.
// Loads are 16-byte vectors; codes are stored as 8- or 16-byte vectors.  Two
// kernels that need no block structure work on 16-byte words instead: the
// tensor-amax pass of unrotated tensors (`k_amax_words`) and INT8 per row
// over long rows staged in shared memory (`k_quantize_int8_row_staged`).
#include <cuda_runtime.h>

#include <cstring>

#include "mxq_formats.cuh"
#include "mxq_internal.h"
#include "tc_ptx.cuh"

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
// order like their bit patterns).  All NT threads of the CTA must call this.
template <int NT = kThreads>
__device__ __forceinline__ void cta_max_to_word(float m, unsigned int *word) {
    __shared__ float wmax[NT / 32];
    m = group_max<32>(m);
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < NT / 32 ? wmax[threadIdx.x] : 0.0f;
        v = group_max<32>(v);
        if (threadIdx.x == 0 && v > 0.0f) atomicMax(word, __float_as_uint(v));
    }
}

// Max of n non-negative values, reduced by the whole CTA (all NT threads call
// this).
template <int NT>
__device__ __forceinline__ float cta_max_of(const float *v, int n) {
    __shared__ float wm[NT / 32];
    float m = 0.0f;
    for (int i = threadIdx.x; i < n; i += NT) m = fmaxf(m, v[i]);
    m = group_max<32>(m);
    if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
    __syncthreads();
    float r = 0.0f;
#pragma unroll
    for (int w = 0; w < NT / 32; w++) r = fmaxf(r, wm[w]);
    return r;
}

// Max over the CTA of one value per thread (all NT threads call this).
template <int NT>
__device__ __forceinline__ float cta_reduce_max(float m) {
    __shared__ float wr[NT / 32];
    m = group_max<32>(m);
    if ((threadIdx.x & 31) == 0) wr[threadIdx.x >> 5] = m;
    __syncthreads();
    float r = 0.0f;
#pragma unroll
    for (int w = 0; w < NT / 32; w++) r = fmaxf(r, wr[w]);
    return r;
}

// ------------------------------------------------------------------ quantize

struct QuantArgs {
    int64_t rows, cols, total_chunks;   // total_chunks < 2^31
    FastDiv cpr;                        // chunks per row
    int hadamard_b;
    int layout;              // 0 canonical, 1 MMA
    int64_t s_pad;           // padded scale columns (MMA layout)
    uint8_t *codes;
    void *scales;
    float *tensor_scale;     // written by chunk 0 (NVFP4, FP8_TENSOR)
    const unsigned int *amax_word;
    const float *amax_slots;  // n_slots > 0: the tensor amax is the max of these (else *amax_word)
    int n_slots;
    float *amax_out;          // amax-only pass: CTA b writes its max to amax_out[b] (null: atomicMax into the word)
    float mx_grid;           // MX grid scale g in [1, 2] (1: the OCP rule)
    // optional packed low-rank operand: tp[row] = [hi | lo] of t[row] / (s_x * *w_ts)
    const float *t;
    int r;
    const float *w_ts;
    __nv_bfloat16 *tp;
};

// Streaming structure of the quantize kernels: each CTA owns a contiguous,
// warp-aligned range of chunks; every thread encodes one chunk per step, the
// CTA's 512 threads covering 512 consecutive chunks, and keeps the raw bytes
// of its next 64 bytes of input (two bf16 chunks or one fp32 chunk) in flight
// in registers, 64 KB per SM with two CTAs, so warps never wait on each
// other and loads overlap the encoding.
constexpr int kQThreads = 512;

// Raw bytes of one 16-element chunk (32 B of bf16 or 64 B of fp32).
template <typename T>
struct RawChunk {
    uint4 q[sizeof(T) * 16 / 16];
};
template <typename T>
__device__ __forceinline__ void raw_load(RawChunk<T> &r, const T *p) {
    const uint4 *g = reinterpret_cast<const uint4 *>(p);
#pragma unroll
    for (int i = 0; i < (int)(sizeof(r.q) / 16); i++) r.q[i] = __ldg(g + i);
}
__device__ __forceinline__ void raw_unpack(const RawChunk<__nv_bfloat16> &r, float v[16]) {
    const uint32_t w[8] = {r.q[0].x, r.q[0].y, r.q[0].z, r.q[0].w, r.q[1].x, r.q[1].y, r.q[1].z, r.q[1].w};
#pragma unroll
    for (int j = 0; j < 8; j++) {
        v[2 * j] = __uint_as_float(w[j] << 16);
        v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
}
__device__ __forceinline__ void raw_unpack(const RawChunk<float> &r, float v[16]) {
#pragma unroll
    for (int i = 0; i < 4; i++) {
        v[4 * i] = __uint_as_float(r.q[i].x);
        v[4 * i + 1] = __uint_as_float(r.q[i].y);
        v[4 * i + 2] = __uint_as_float(r.q[i].z);
        v[4 * i + 3] = __uint_as_float(r.q[i].w);
    }
}

// Codes and scale of chunk c (row `row`, chunk column `colc`) from its 16
// values v and the block amax (already the max over the block's G lanes).
// All lanes of the warp must call this (no per-lane early exit), but only
// lanes with `valid` store.
template <int F>
__device__ __forceinline__ void encode_chunk(const float (&v)[16], float amax, uint32_t c, uint32_t row, uint32_t colc,
                                             bool valid, int lane, const QuantArgs &a, uint32_t s_pad4,
                                             const TensorRecip &tr, const Recip &rt) {
    constexpr int BLK = fmt_block(F) ? fmt_block(F) : 16;
    constexpr int G = BLK / 16;
    const uint32_t cpr = (uint32_t)(a.cols >> 4);
    uint8_t *scb = reinterpret_cast<uint8_t *>(a.scales);
    if (F == kMXFP8 || F == kMXFP4) {
        float inv = 0.0f;
        uint32_t sb = 127;
        if (amax > 0.0f)
            sb = a.mx_grid == 1.0f ? mx_scale(amax, F == kMXFP8 ? 8 : 2, inv)
                                   : mx_scale_grid(amax, F == kMXFP8 ? 8 : 2, a.mx_grid, inv);
        if (!valid) return;
        // inv is a power of two: v * inv is exact (or far below the smallest code)
        float u[16];
        mul8(v, inv, u);
        mul8(v + 8, inv, u + 8);
        const bool zero = !(amax > 0.0f);   // all-zero block: +0 codes
        if (F == kMXFP8) {
            uint4 w;
            w.x = zero ? 0u : cvt_e4m3x4(u[0], u[1], u[2], u[3]);
            w.y = zero ? 0u : cvt_e4m3x4(u[4], u[5], u[6], u[7]);
            w.z = zero ? 0u : cvt_e4m3x4(u[8], u[9], u[10], u[11]);
            w.w = zero ? 0u : cvt_e4m3x4(u[12], u[13], u[14], u[15]);
            *reinterpret_cast<uint4 *>(a.codes + (int64_t)c * 16) = w;
        } else {
            uint2 w;
            w.x = zero ? 0u : cvt_e2m1x8(u[0], u[1], u[2], u[3], u[4], u[5], u[6], u[7]);
            w.y = zero ? 0u : cvt_e2m1x8(u[8], u[9], u[10], u[11], u[12], u[13], u[14], u[15]);
            *reinterpret_cast<uint2 *>(a.codes + (int64_t)c * 8) = w;
        }
        if ((lane & 1) == 0) {
            const uint32_t sc = colc >> 1;
            scb[a.layout == 0 ? row * (cpr >> 1) + sc : mma_scale_offset32(row, sc, s_pad4)] = (uint8_t)sb;
        }
    } else if (F == kNVFP4) {
        float d;
        const uint32_t e4 = nvfp4_block_scale_fast(amax, tr, d);
        if (!valid) return;
        uint2 w = make_uint2(0u, 0u);   // e4 == 0: +0 codes
        if (e4) {
            const Recip rd = recip_of(d);
            w.x = e2m1x8_quot(v, rd);
            w.y = e2m1x8_quot(v + 8, rd);
        }
        *reinterpret_cast<uint2 *>(a.codes + (int64_t)c * 8) = w;
        scb[a.layout == 0 ? c : mma_scale_offset32(row, colc, s_pad4)] = (uint8_t)e4;
    } else if (F == kINT4G32 || F == kINT4G64) {
        const float s = __fdiv_rn(amax, 7.0f);
        const Recip rs = recip_of(s);
        if (!valid) return;
        if (a.layout == 0) {
            const uint32_t b0 = int_x4_quot(v, rs, 7), b1 = int_x4_quot(v + 4, rs, 7);
            const uint32_t b2 = int_x4_quot(v + 8, rs, 7), b3 = int_x4_quot(v + 12, rs, 7);
            *reinterpret_cast<uint2 *>(a.codes + (int64_t)c * 8) =
                make_uint2(nibbles_of_bytes(b0, b1), nibbles_of_bytes(b2, b3));
        } else {   // MMA layout: E4M3 bytes of the integer codes
            *reinterpret_cast<uint4 *>(a.codes + (int64_t)c * 16) =
                make_uint4(int_x4_quot_e4m3(v, rs, 7), int_x4_quot_e4m3(v + 4, rs, 7),
                           int_x4_quot_e4m3(v + 8, rs, 7), int_x4_quot_e4m3(v + 12, rs, 7));
        }
        if ((lane & (G - 1)) == 0) {
            float *sc = reinterpret_cast<float *>(a.scales);
            const uint32_t g = colc / G;
            if (a.layout == 0) sc[row * (cpr / G) + g] = s;
            else sc[g * (uint32_t)a.rows + row] = s;
        }
    } else if (F == kFP8Tensor) {
        if (!valid) return;
        // both ends of the four brackets without branches; one test sends the
        // chunk to e4m3x4_quot (same codes) when any pair disagrees
        const float2 lo2 = make_float2(rt.lo, rt.lo), hi2 = make_float2(rt.hi, rt.hi);
        uint32_t lo[4], hi[4];
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const float2 v01 = make_float2(v[4 * k], v[4 * k + 1]), v23 = make_float2(v[4 * k + 2], v[4 * k + 3]);
            const float2 l01 = __fmul2_rn(v01, lo2), l23 = __fmul2_rn(v23, lo2);
            const float2 h01 = __fmul2_rn(v01, hi2), h23 = __fmul2_rn(v23, hi2);
            lo[k] = cvt_e4m3x4(l01.x, l01.y, l23.x, l23.y);
            hi[k] = cvt_e4m3x4(h01.x, h01.y, h23.x, h23.y);
        }
        uint4 w = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        if (!(rt.fast && lo[0] == hi[0] && lo[1] == hi[1] && lo[2] == hi[2] && lo[3] == hi[3])) {
            w.x = e4m3x4_quot(v, rt);
            w.y = e4m3x4_quot(v + 4, rt);
            w.z = e4m3x4_quot(v + 8, rt);
            w.w = e4m3x4_quot(v + 12, rt);
        }
        *reinterpret_cast<uint4 *>(a.codes + (int64_t)c * 16) = w;
    }
}

template <typename T, int F>
__global__ void __launch_bounds__(kQThreads, 2) k_quantize(const T *__restrict__ x, QuantArgs a) {
    constexpr int kQDepth = 64 / (16 * (int)sizeof(T));   // chunks in flight per thread
    constexpr int BLK = fmt_block(F) ? fmt_block(F) : 16;
    constexpr int G = BLK / 16;   // lanes per quantization block
    const int lane = lane_id();
    // this CTA's chunks [c_begin, c_end), boundaries on multiples of 32 chunks
    const uint32_t total = (uint32_t)a.total_chunks;
    const uint32_t units = (total + 31) >> 5;
    const uint32_t c_begin = (uint32_t)(((uint64_t)blockIdx.x * units / gridDim.x) << 5);
    uint32_t c_end = (uint32_t)(((uint64_t)(blockIdx.x + 1) * units / gridDim.x) << 5);
    c_end = c_end < total ? c_end : total;
    const int steps = (int)((c_end - c_begin + kQThreads - 1) / kQThreads);
    const uint32_t cpr = (uint32_t)(a.cols >> 4);
    const uint32_t s_pad4 = (uint32_t)(a.s_pad >> 2);

    // nothing global is touched before the previous kernel has completed
    pdl_wait();
    pdl_launch_dependents();
    float s_t = 1.0f;
    TensorRecip tr;
    Recip rt;
    if (F == kNVFP4 || F == kFP8Tensor) {
        const float amax_t = a.n_slots > 0 ? cta_max_of<kQThreads>(a.amax_slots, a.n_slots)
                                           : __uint_as_float(*a.amax_word);
        s_t = F == kNVFP4 ? nvfp4_tensor_scale(amax_t) : fp8_tensor_scale(amax_t);
        if (blockIdx.x == 0 && threadIdx.x == 0) *a.tensor_scale = s_t;
        if (F == kNVFP4) tr = tensor_recip_of(s_t);
        else rt = recip_of(s_t);
    }

    const float hnorm = a.hadamard_b ? __frsqrt_rn((float)a.hadamard_b) : 1.0f;   // RN(1/sqrt(b))
    // this thread's chunk c = (row, colc), advanced by kQThreads chunks a step
    uint32_t c = c_begin + threadIdx.x;
    uint32_t row = fdiv(c, a.cpr);
    uint32_t colc = c - row * cpr;
    const uint32_t drow = fdiv((uint32_t)kQThreads, a.cpr);
    const uint32_t dcol = (uint32_t)kQThreads - drow * cpr;

    float tensor_max = 0.0f;
    RawChunk<T> pre[kQDepth];
#pragma unroll
    for (int i = 0; i < kQDepth; i++) {
        const uint32_t ci = c + (uint32_t)i * kQThreads;
        if (ci < c_end) raw_load(pre[i], x + (int64_t)ci * 16);
    }
    // The integer formats keep their register budget for the codes: one
    // chunk per loop turn, the prefetch buffers moved down each turn and the
    // chunk position recomputed.  The others take kQDepth steps a turn with
    // buffer j always holding step it0 + j (no buffer moves) and advance the
    // position incrementally.
    constexpr bool kRotate = F == kINT4G32 || F == kINT4G64;
    constexpr int kTurn = kRotate ? 1 : kQDepth;
#pragma unroll 1
    for (int it0 = 0; it0 < steps; it0 += kTurn) {
#pragma unroll
        for (int j = 0; j < kTurn; j++) {
            if (it0 + j < steps) {
                const bool valid = c < c_end;
                float v[16];
                if (valid) raw_unpack(pre[j], v);
                else {
#pragma unroll
                    for (int i = 0; i < 16; i++) v[i] = 0.0f;
                }
                const uint32_t cn = c + (uint32_t)kQDepth * kQThreads;
                if constexpr (kRotate) {
#pragma unroll
                    for (int i = 0; i + 1 < kQDepth; i++) pre[i] = pre[i + 1];
                    if (cn < c_end) raw_load(pre[kQDepth - 1], x + (int64_t)cn * 16);
                } else {
                    if (cn < c_end) raw_load(pre[j], x + (int64_t)cn * 16);
                }
                if (a.hadamard_b) hadamard_chunk_n(v, a.hadamard_b, lane, hnorm);
                float amax = amax16(v);
                if (F == kNumFmt) {   // tensor-amax pass only
                    tensor_max = fmaxf(tensor_max, amax);
                } else {
                    if (G > 1) amax = group_max<G>(amax);
                    encode_chunk<F>(v, amax, c, row, colc, valid, lane, a, s_pad4, tr, rt);
                }
                c += kQThreads;
                if constexpr (kRotate) {
                    row = fdiv(c, a.cpr);
                    colc = c - row * cpr;
                } else {
                    row += drow;
                    colc += dcol;
                    if (colc >= cpr) {
                        colc -= cpr;
                        row++;
                    }
                }
            }
        }
    }
    if (F == kNumFmt) {
        if (a.amax_out) {   // every CTA writes its slot, so the slots need no clearing
            const float m = cta_reduce_max<kQThreads>(tensor_max);
            if (threadIdx.x == 0) a.amax_out[blockIdx.x] = m;
        } else {
            cta_max_to_word<kQThreads>(tensor_max, const_cast<unsigned int *>(a.amax_word));
        }
        return;
    }
    if (fmt_block(F) && (F == kMXFP8 || F == kMXFP4 || F == kNVFP4) && a.layout == 1) {
        // the MMA layout's padding (columns S .. s_pad - 1 of every row, and
        // every column of the rows up to the next multiple of 128) holds zero
        // scales, which this grid writes: no clearing of the buffer first.
        // Disjoint from the scales written above, so no ordering is needed.
        const uint32_t S = (uint32_t)(a.cols / BLK), sp = (uint32_t)a.s_pad;
        const uint32_t rows = (uint32_t)a.rows, rows_pad = (rows + 127u) & ~127u;
        const uint32_t n1 = rows * (sp - S), n = n1 + (rows_pad - rows) * sp;
        for (uint32_t i = blockIdx.x * kQThreads + threadIdx.x; i < n; i += gridDim.x * kQThreads) {
            uint32_t r, sc;
            if (i < n1) {
                r = i / (sp - S);
                sc = S + (i - r * (sp - S));
            } else {
                r = rows + (i - n1) / sp;
                sc = (i - n1) % sp;
            }
            reinterpret_cast<uint8_t *>(a.scales)[mma_scale_offset32(r, sc, s_pad4)] = 0;
        }
    }
    if (a.tp) {
        // packed low-rank operand, one row per warp, one value per lane:
        // u = t / alpha, hi = bf16(u), lo = bf16(u - hi), zeros past r
        const bool ts = F == kNVFP4 || F == kFP8Tensor;
        const float alpha = ts ? __fmul_rn(s_t, *a.w_ts) : 1.0f;
        const int64_t warp = ((int64_t)blockIdx.x * kQThreads + threadIdx.x) >> 5;
        const int64_t nwarps = ((int64_t)gridDim.x * kQThreads) >> 5;
        for (int64_t r = warp; r < a.rows; r += nwarps) {
            float u = lane < a.r ? a.t[r * a.r + lane] : 0.0f;
            if (ts) u = __fdiv_rn(u, alpha);
            const __nv_bfloat16 hi = __float2bfloat16_rn(u);
            a.tp[r * 64 + lane] = hi;
            a.tp[r * 64 + 32 + lane] = __float2bfloat16_rn(__fsub_rn(u, __bfloat162float(hi)));
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
            if (c < cpr)
                *reinterpret_cast<uint4 *>(a.codes + (row * cpr + c) * 16) =
                    make_uint4(int_x4_quot(v, rs, 127), int_x4_quot(v + 4, rs, 127), int_x4_quot(v + 8, rs, 127),
                               int_x4_quot(v + 12, rs, 127));
        }
        if (lane == 0) reinterpret_cast<float *>(a.scales)[row] = s;
    }
}

// INT8 per row with the whole row in registers (rows of at most 32 * NC
// chunks): one warp per row issues all of its loads at once, reduces the
// row maximum and codes from the registers, so the row is read once.
template <typename T, int NC>
__global__ void __launch_bounds__(kThreads) k_quantize_int8_row_reg(const T *__restrict__ x, QuantArgs a) {
    const int lane = lane_id();
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
    const int cpr = (int)(a.cols >> 4);
    for (int64_t row = warp; row < a.rows; row += nwarps) {
        const T *xr = x + row * a.cols;
        RawChunk<T> raw[NC];
#pragma unroll
        for (int j = 0; j < NC; j++)
            if (lane + 32 * j < cpr) raw_load(raw[j], xr + (int64_t)(lane + 32 * j) * 16);
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < NC; j++) {
            if (lane + 32 * j < cpr) {
                float v[16];
                raw_unpack(raw[j], v);
                m = fmaxf(m, amax16(v));
            }
        }
        m = group_max<32>(m);
        const float s = __fdiv_rn(m, 127.0f);
        const Recip rs = recip_of(s);
#pragma unroll
        for (int j = 0; j < NC; j++) {
            const int c = lane + 32 * j;
            if (c < cpr) {
                float v[16];
                raw_unpack(raw[j], v);
                *reinterpret_cast<uint4 *>(a.codes + (row * cpr + c) * 16) =
                    make_uint4(int_x4_quot(v, rs, 127), int_x4_quot(v + 4, rs, 127), int_x4_quot(v + 8, rs, 127),
                               int_x4_quot(v + 12, rs, 127));
            }
        }
        if (lane == 0) reinterpret_cast<float *>(a.scales)[row] = s;
    }
}

// INT8 per row for bf16 rows of more than 2048 elements, staged in shared
// memory: each CTA walks blocks of kRowBlk consecutive rows; one bulk copy
// brings a block into one of two stages while the CTA codes the one before.
// kI8Parts warps share a row: thread (part, lane) owns the 16-byte words
// part * 32 + lane + 128 j of it (a warp reads 512 consecutive bytes), keeps
// them in registers, forms their maximum, and after the parts' maxima meet
// in shared memory codes them.  The arithmetic is that of
// k_quantize_int8_row_reg; on long rows this kernel keeps more of the input
// in flight than one warp per row can hold in registers.
constexpr int kRowBlk = 4;            // rows per block
constexpr int kI8Parts = 4;           // warps per row
constexpr int kI8RowThreads = 32 * kRowBlk * kI8Parts;
constexpr int kI8CtasPerSm = 2;       // so that one CTA codes while the other waits at a barrier
constexpr int kI8Stages = 2;          // a block is coded while the next one loads
constexpr int kI8SmemCap = 113664;    // dynamic shared memory opt-in per CTA: two CTAs fit on an SM
constexpr unsigned int kErrI8Row = 32u;   // error-word bit of a wait on a block's copy that ran out

__device__ __forceinline__ void bulk_load_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void unpack_bf16x8(const uint4 &w, float v[8]) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; j++) {
        v[2 * j] = __uint_as_float(u[j] << 16);
        v[2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
    }
}

template <int NQ>
__global__ void __launch_bounds__(kI8RowThreads, kI8CtasPerSm)
    k_quantize_int8_row_staged(const __nv_bfloat16 *__restrict__ x, QuantArgs a, unsigned int *err,
                               unsigned long long wait_ns) {
    constexpr int nst = kI8Stages;
    extern __shared__ __align__(128) uint8_t sx[];
    __shared__ float part_max[kRowBlk][kI8Parts];
    __shared__ int abort_flag;
    const int lane = lane_id(), warp = (int)(threadIdx.x >> 5);
    const int rw = warp / kI8Parts, part = warp % kI8Parts;
    const int words = (int)(a.cols >> 3);
    const uint32_t row_bytes = (uint32_t)(a.cols * 2);
    const uint32_t stage_bytes = row_bytes * kRowBlk;
    uint64_t *full = reinterpret_cast<uint64_t *>(sx + (size_t)nst * stage_bytes);
    const int64_t nblk = (a.rows + kRowBlk - 1) / kRowBlk;
    if (threadIdx.x == 0) {
        for (int j = 0; j < nst; j++) mbar_init(full + j, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    auto issue = [&](int64_t b, int st) {
        const int64_t r0 = b * kRowBlk;
        const uint32_t nr = (uint32_t)(a.rows - r0 < kRowBlk ? a.rows - r0 : kRowBlk);
        mbar_arrive_expect_tx(full + st, row_bytes * nr);
        bulk_load_g2s(sx + (size_t)st * stage_bytes, x + r0 * a.cols, row_bytes * nr, full + st);
    };
    int64_t issued = 0;
    if (threadIdx.x == 0) {
        for (int j = 0; j < nst; j++) {
            const int64_t b = blockIdx.x + (int64_t)j * gridDim.x;
            if (b < nblk) {
                issue(b, j);
                issued++;
            }
        }
    }
    int st = 0;
    uint32_t ph = 0;
    int64_t it = 0;
    for (int64_t b = blockIdx.x; b < nblk; b += gridDim.x, it++) {
        if (!mbar_wait(full + st, ph, wait_ns)) {
            if (lane == 0) atomicOr(err, kErrI8Row);
            abort_flag = 1;
        }
        const int64_t row = b * kRowBlk + rw;
        const bool live = row < a.rows;
        const uint4 *src = reinterpret_cast<const uint4 *>(sx + (size_t)st * stage_bytes + (size_t)rw * row_bytes);
        uint4 w[NQ];
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < NQ; j++) {
            const int q = part * 32 + lane + 128 * j;
            w[j] = make_uint4(0u, 0u, 0u, 0u);
            if (live && q < words) w[j] = src[q];
            float v[8];
            unpack_bf16x8(w[j], v);
#pragma unroll
            for (int e = 0; e < 8; e++) m = fmaxf(m, fabsf(v[e]));
        }
        m = group_max<32>(m);
        if (lane == 0) part_max[rw][part] = m;
        __syncthreads();   // the parts' maxima are in; an expired wait anywhere ends every thread here
        if (abort_flag) break;
        if (live) {
            float rm = part_max[rw][0];
#pragma unroll
            for (int j = 1; j < kI8Parts; j++) rm = fmaxf(rm, part_max[rw][j]);
            const float sc = __fdiv_rn(rm, 127.0f);
            const Recip rs = recip_of(sc);
            uint8_t *dst = a.codes + row * a.cols;
#pragma unroll
            for (int j = 0; j < NQ; j++) {
                const int q = part * 32 + lane + 128 * j;
                if (q < words) {
                    float v[8];
                    unpack_bf16x8(w[j], v);
                    *reinterpret_cast<uint2 *>(dst + (int64_t)q * 8) =
                        make_uint2(int_x4_quot_packed(v, rs, 127), int_x4_quot_packed(v + 4, rs, 127));
                }
            }
            if (lane == 0 && part == 0) reinterpret_cast<float *>(a.scales)[row] = sc;
        }
        __syncthreads();   // stage st and part_max are free: thread 0 refills the stage
        if (threadIdx.x == 0) {
            const int64_t b2 = b + (int64_t)nst * gridDim.x;
            if (b2 < nblk) {
                issue(b2, st);
                issued++;
            }
        }
        if (++st == nst) {
            st = 0;
            ph ^= 1u;
        }
    }
    if (threadIdx.x == 0 && abort_flag) {   // let the copies in flight land before the CTA exits
        for (int64_t j = it; j < issued; j++) mbar_wait(full + (int)(j % nst), (uint32_t)((j / nst) & 1), wait_ns);
    }
}

// One launch of k_quantize_int8_row_staged<NQ>, after its one-time opt-in
// to the large shared-memory carve-out on this device.
template <int NQ>
bool launch_int8_row_staged_nq(const __nv_bfloat16 *x, const QuantArgs &a, int grid, size_t smem, unsigned int *err,
                               cudaStream_t s) {
    static PerDeviceOnce opt_in;
    if (opt_in.run([] {
            return cudaFuncSetAttribute(k_quantize_int8_row_staged<NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kI8SmemCap);
        }) != cudaSuccess)
        return false;
    k_quantize_int8_row_staged<NQ><<<grid, kI8RowThreads, smem, s>>>(x, a, err, 2000000000ull);
    return true;
}

// Launches k_quantize_int8_row_staged when it takes the shape (bf16 rows of
// at most 5120 elements, a multiple of 8, starting 16-byte aligned: two
// stages of 4 rows take at most 80 KB); false (nothing launched) otherwise.
bool launch_int8_row_staged(const __nv_bfloat16 *x, const QuantArgs &a, cudaStream_t s) {
    const int64_t words = a.cols >> 3;
    if (a.rows <= 0 || a.cols % 8 || words > 128 * 5 || (reinterpret_cast<uintptr_t>(x) & 15u)) return false;
    const size_t smem = (size_t)kI8Stages * kRowBlk * a.cols * 2 + 8 * kI8Stages;
    unsigned int *err = nullptr;
    if (error_word_address(&err) != cudaSuccess) return false;
    const int64_t nblk = (a.rows + kRowBlk - 1) / kRowBlk;
    const int64_t cap = (int64_t)sm_count() * kI8CtasPerSm;
    const int grid = (int)(nblk < cap ? nblk : cap);
    if (words <= 128 * 4) return launch_int8_row_staged_nq<4>(x, a, grid, smem, err, s);
    return launch_int8_row_staged_nq<5>(x, a, grid, smem, err, s);
}

// ------------------------------------------------------------------ dequantize

struct DequantArgs {
    int64_t rows, cols, total_chunks;
    FastDiv cpr;
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
    const int64_t row = fdiv((uint32_t)c, a.cpr);
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
            // MMA layout: E4M3 byte of the integer code; canonical: two's-complement nibble
            const float q = unpacked_int4 ? dec_e4m3(code[i])
                                          : (float)((code[i] & 8u) ? (int)code[i] - 16 : (int)code[i]);
            out[i] = __fmul_rn(q, s);
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

// ------------------------------------------------------------------ selection over a fixed format set
//
// The same errors for the candidate sets the library is used with -- the
// Chameleon weight set {MXFP4, NVFP4, INT4-g32} and the W8A8 activation set
// {MXFP8, INT8 per row, FP8 per tensor} -- with the formats fixed at compile
// time (MASK, one bit per format), codes taken by the bracketed-reciprocal
// codecs of the quantizer instead of an IEEE division per element, and the
// next chunk of the row prefetched while the current one is scored.  Each
// error term is formed exactly: for the MX formats d = v - q 2^e is exact in
// fp32 (q 2^e has at most 4 significant bits and, unless q = 0 where d = v,
// lies within a few binades of v, so d is a multiple of v's last place below
// 2^24 of them); for the others d = v - q S (S the exact binary64 product of
// the scales) is one binary64 FMA, exact because q S and v are within a few
// binades of each other.  The square is added with one binary64 FMA.  The
// caller's candidate order only decides the reported order and ties.

constexpr uint32_t kSelSetW4 = (1u << kMXFP4) | (1u << kNVFP4) | (1u << kINT4G32);
constexpr uint32_t kSelSetA8 = (1u << kMXFP8) | (1u << kINT8Row) | (1u << kFP8Tensor);
constexpr int kSelThreads = 256;

__host__ __device__ constexpr int sel_slot(uint32_t mask, int f) {
    int n = 0;
    for (int i = 0; i < f; i++) n += (mask >> i) & 1u;
    return n;
}
__host__ __device__ constexpr int sel_count(uint32_t mask) { return sel_slot(mask, kNumFmt); }

struct SelectSetArgs {
    int64_t n, k;
    int ncand;
    int slot[kMaxCandidates];        // slot of caller's candidate j in the kernel's format order
    int cand[kMaxCandidates];
    const float *amax_slots;         // tensor amax = max of n_slots values
    int n_slots;
    uint8_t *choice;
    double *sse;                     // may be null
};

// The eight E2M1 codes packed in a word (element i in nibble i) as fp16
// values (exact: every E2M1 value is an fp16 value), through the hardware
// conversion.
__device__ __forceinline__ void e2m1x8_to_half(uint32_t c, __half (&h)[8]) {
#pragma unroll
    for (int b = 0; b < 4; b++) {
        const __half2_raw r = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)((c >> (8 * b)) & 0xFFu), __NV_E2M1);
        h[2 * b] = __ushort_as_half(r.x);
        h[2 * b + 1] = __ushort_as_half(r.y);
    }
}
__device__ __forceinline__ double half_to_f64(__half h) {
    double d;
    asm("cvt.f64.f16 %0, %1;" : "=d"(d) : "h"(__half_as_ushort(h)));
    return d;
}
// Four E4M3 codes (bytes of c) as fp32 (exact: every E4M3 value is an fp16 value).
__device__ __forceinline__ void e4m3x4_f32(uint32_t c, float *o) {
    uint32_t h0, h1;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, lo;\n\tcvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
        : "=r"(h0), "=r"(h1)
        : "r"(c));
    o[0] = __half2float(__ushort_as_half((unsigned short)(h0 & 0xFFFFu)));
    o[1] = __half2float(__ushort_as_half((unsigned short)(h0 >> 16)));
    o[2] = __half2float(__ushort_as_half((unsigned short)(h1 & 0xFFFFu)));
    o[3] = __half2float(__ushort_as_half((unsigned short)(h1 >> 16)));
}

// acc += sum (v - q 2^e)^2 over one chunk of an MX block with maximum amax.
template <int F>
__device__ __forceinline__ void sel_err_mx(const float (&v)[16], float amax, double &acc) {
    if (!(amax > 0.0f)) return;   // all values are +-0 and all codes zero
    float inv;
    const int e = (int)mx_scale(amax, F == kMXFP8 ? 8 : 2, inv) - 127;
    const float X = exp2i_f32(e);
    float u[16];
    mul8(v, inv, u);
    mul8(v + 8, inv, u + 8);
    if (F == kMXFP4) {
#pragma unroll
        for (int h = 0; h < 2; h++) {
            __half q[8];
            e2m1x8_to_half(cvt_e2m1x8(u[8 * h], u[8 * h + 1], u[8 * h + 2], u[8 * h + 3], u[8 * h + 4],
                                      u[8 * h + 5], u[8 * h + 6], u[8 * h + 7]),
                           q);
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const float d = __fmaf_rn(-__half2float(q[i]), X, v[8 * h + i]);
                const double dd = (double)d;
                acc = __fma_rn(dd, dd, acc);
            }
        }
    } else {
#pragma unroll
        for (int h = 0; h < 4; h++) {
            float q[4];
            e4m3x4_f32(cvt_e4m3x4(u[4 * h], u[4 * h + 1], u[4 * h + 2], u[4 * h + 3]), q);
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const float d = __fmaf_rn(-q[i], X, v[4 * h + i]);
                const double dd = (double)d;
                acc = __fma_rn(dd, dd, acc);
            }
        }
    }
}

// acc += sum (v - q e4 s_t)^2 over one NVFP4 block.
__device__ __forceinline__ void sel_err_nvfp4(const float (&v)[16], const double (&vd)[16], float amax,
                                              const TensorRecip &tr, double st, double &acc) {
    float dsc;
    const uint32_t e4 = nvfp4_block_scale_fast(amax, tr, dsc);
    if (!e4) {   // all codes zero
#pragma unroll
        for (int i = 0; i < 16; i++) acc = __fma_rn(vd[i], vd[i], acc);
        return;
    }
    const Recip r = recip_of(dsc);
    const double S = __dmul_rn((double)e4m3_to_f32(e4), st);   // exact: 4 x 24 significant bits
#pragma unroll
    for (int h = 0; h < 2; h++) {
        __half q[8];
        e2m1x8_to_half(e2m1x8_quot(v + 8 * h, r), q);
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const double d = __fma_rn(-half_to_f64(q[i]), S, vd[8 * h + i]);
            acc = __fma_rn(d, d, acc);
        }
    }
}

// acc += sum (v - q s)^2 for symmetric integer codes with scale s.
__device__ __forceinline__ void sel_err_int(const float (&v)[16], const double (&vd)[16], float s, int qmax,
                                            double &acc) {
    if (s == 0.0f) {   // all codes zero
#pragma unroll
        for (int i = 0; i < 16; i++) acc = __fma_rn(vd[i], vd[i], acc);
        return;
    }
    const Recip r = recip_of(s);
    const double sd = (double)s;
    // the codes as floats: RN(t + 1.5 * 2^23) - 1.5 * 2^23 is RNE(t) for |t| < 2^22 (the quantizer's
    // rounding), taken from both ends of the quotient bracket; any group of four whose ends disagree
    // is coded with exact divisions
    float q[16];
    bool same = r.fast;
#pragma unroll
    for (int i = 0; i < 16; i++) {
        const float lo = __fmaf_rn(v[i], r.lo, kRoundMagic), hi = __fmaf_rn(v[i], r.hi, kRoundMagic);
        same = same && lo == hi;
        q[i] = __fsub_rn(lo, kRoundMagic);
    }
    if (!same) {
#pragma unroll
        for (int i = 0; i < 16; i++) {
            int c = __float2int_rn(__fdiv_rn(v[i], s));
            c = c > qmax ? qmax : (c < -qmax ? -qmax : c);
            q[i] = (float)c;
        }
    }
#pragma unroll
    for (int i = 0; i < 16; i++) {
        const double d = __fma_rn(-(double)q[i], sd, vd[i]);
        acc = __fma_rn(d, d, acc);
    }
}

// acc += sum (v - q s)^2 for E4M3 codes of v / s (FP8 per tensor).
__device__ __forceinline__ void sel_err_fp8t(const float (&v)[16], const double (&vd)[16], const Recip &rt, double sd,
                                             double &acc) {
#pragma unroll
    for (int h = 0; h < 4; h++) {
        float q[4];
        e4m3x4_f32(e4m3x4_quot(v + 4 * h, rt), q);
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const double d = __fma_rn(-(double)q[i], sd, vd[4 * h + i]);
            acc = __fma_rn(d, d, acc);
        }
    }
}

template <typename T, uint32_t MASK>
__global__ void __launch_bounds__(kSelThreads, 3) k_select_set(const T *__restrict__ w, SelectSetArgs a) {
    constexpr int NS = sel_count(MASK);
    constexpr bool kTensor = (MASK & ((1u << kNVFP4) | (1u << kFP8Tensor))) != 0;
    constexpr bool kRow = (MASK & (1u << kINT8Row)) != 0;
    constexpr bool kNeedVd = (MASK & ~((1u << kMXFP4) | (1u << kMXFP8))) != 0;
    const int lane = lane_id();
    const int64_t warp = ((int64_t)blockIdx.x * kSelThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kSelThreads) >> 5;
    const int cpr = (int)(a.k >> 4);
    // launched right after the tensor-amax pass: nothing global is read before it completes
    pdl_wait();
    pdl_launch_dependents();
    float tamax = 0.0f;
    if (kTensor) tamax = cta_max_of<kSelThreads>(a.amax_slots, a.n_slots);
    const float st_nv = nvfp4_tensor_scale(tamax), st_f8 = fp8_tensor_scale(tamax);
    const TensorRecip tr = tensor_recip_of(st_nv);
    const Recip rf8 = recip_of(st_f8);
    for (int64_t row = warp; row < a.n; row += nwarps) {
        const T *wr = w + row * a.k;
        float rowamax = 0.0f;
        if (kRow) {
            for (int c = lane; c < cpr; c += 32) {
                float v[16];
                load16(wr + (int64_t)c * 16, v);
                rowamax = fmaxf(rowamax, amax16(v));
            }
            rowamax = group_max<32>(rowamax);
        }
        const float s_row = __fdiv_rn(rowamax, 127.0f);
        double acc[NS];
#pragma unroll
        for (int j = 0; j < NS; j++) acc[j] = 0.0;
        RawChunk<T> pre;
        if (lane < cpr) raw_load(pre, wr + (int64_t)lane * 16);
        for (int c0 = 0; c0 < cpr; c0 += 32) {
            const int c = c0 + lane;
            float v[16];
            if (c < cpr) raw_unpack(pre, v);
            else {
#pragma unroll
                for (int i = 0; i < 16; i++) v[i] = 0.0f;
            }
            if (c + 32 < cpr) raw_load(pre, wr + (int64_t)(c + 32) * 16);
            // lanes past the row end hold zeros: their blocks (whole groups of
            // lanes, since k % 64 == 0) add nothing
            const float m1 = amax16(v);
            const float m2 = group_max<2>(m1);
            double vd[16];
            if (kNeedVd) {
#pragma unroll
                for (int i = 0; i < 16; i++) vd[i] = (double)v[i];
            }
            if (MASK & (1u << kMXFP8)) sel_err_mx<kMXFP8>(v, m2, acc[sel_slot(MASK, kMXFP8)]);
            if (MASK & (1u << kMXFP4)) sel_err_mx<kMXFP4>(v, m2, acc[sel_slot(MASK, kMXFP4)]);
            if (MASK & (1u << kNVFP4)) sel_err_nvfp4(v, vd, m1, tr, (double)st_nv, acc[sel_slot(MASK, kNVFP4)]);
            if (MASK & (1u << kINT4G32)) sel_err_int(v, vd, __fdiv_rn(m2, 7.0f), 7, acc[sel_slot(MASK, kINT4G32)]);
            if (MASK & (1u << kINT4G64))
                sel_err_int(v, vd, __fdiv_rn(group_max<4>(m2), 7.0f), 7, acc[sel_slot(MASK, kINT4G64)]);
            if (MASK & (1u << kINT8Row)) sel_err_int(v, vd, s_row, 127, acc[sel_slot(MASK, kINT8Row)]);
            if (MASK & (1u << kFP8Tensor)) sel_err_fp8t(v, vd, rf8, (double)st_f8, acc[sel_slot(MASK, kFP8Tensor)]);
        }
#pragma unroll
        for (int j = 0; j < NS; j++) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[j] = __dadd_rn(acc[j], __shfl_xor_sync(0xFFFFFFFFu, acc[j], o));
        }
        if (lane == 0) {
            int best = 0;
            double bestv = 0.0;
#pragma unroll
            for (int j = 0; j < kMaxCandidates; j++) {
                if (j < a.ncand) {
                    double s = 0.0;
#pragma unroll
                    for (int t = 0; t < NS; t++)
                        if (t == a.slot[j]) s = acc[t];
                    if (a.sse) a.sse[row * a.ncand + j] = s;
                    if (j == 0 || s < bestv) {
                        best = j;
                        bestv = s;
                    }
                }
            }
            int fmt = a.cand[0];
#pragma unroll
            for (int j = 1; j < kMaxCandidates; j++)
                if (j == best) fmt = a.cand[j];
            a.choice[row] = (uint8_t)fmt;
        }
    }
}

}  // namespace

// ====================================================================== host

static int sm_count_cached() { return sm_count(); }

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
    a.cpr = make_fastdiv((uint32_t)(cols / 16 > 0 ? cols / 16 : 1));
    a.hadamard_b = hadamard_b;
    a.amax_word = amax_word;
    if (bf16) launch_qf<__nv_bfloat16, kNumFmt>((const __nv_bfloat16 *)x, a, s);
    else launch_qf<float, kNumFmt>((const float *)x, a, s);
    return cudaGetLastError();
}

// The tensor amax of an unrotated tensor as per-CTA maxima: a grid-stride
// stream of 16-byte words, kAmaxWords of them in flight per thread, each
// CTA writing the max |x| of its words to out[blockIdx.x].  The maximum is
// exact and independent of the order it is taken in (fmaxf: a NaN never
// wins), so it is the same value the chunk loop of k_quantize would give.
constexpr int kAmaxWords = 8;   // 128 B in flight per thread, 128 KB per SM
__device__ __forceinline__ float amax_word(const uint4 &w, bool bf16) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; j++) {
        if (bf16) {
            m = fmaxf(m, fabsf(__uint_as_float(u[j] << 16)));
            m = fmaxf(m, fabsf(__uint_as_float(u[j] & 0xFFFF0000u)));
        } else {
            m = fmaxf(m, fabsf(__uint_as_float(u[j])));
        }
    }
    return m;
}
template <bool BF16>
__global__ void __launch_bounds__(kQThreads, 2) k_amax_words(const uint4 *__restrict__ x, int64_t words, float *out) {
    pdl_wait();   // nothing is read before the previous kernel has completed
    pdl_launch_dependents();
    const int64_t stride = (int64_t)gridDim.x * kQThreads;
    int64_t i = (int64_t)blockIdx.x * kQThreads + threadIdx.x;
    float m = 0.0f;
    for (; i + (kAmaxWords - 1) * stride < words; i += kAmaxWords * stride) {
        uint4 w[kAmaxWords];
#pragma unroll
        for (int u = 0; u < kAmaxWords; u++) w[u] = __ldg(x + i + u * stride);
#pragma unroll
        for (int u = 0; u < kAmaxWords; u++) m = fmaxf(m, amax_word(w[u], BF16));
    }
    for (; i < words; i += stride) m = fmaxf(m, amax_word(__ldg(x + i), BF16));
    const float r = cta_reduce_max<kQThreads>(m);
    if (threadIdx.x == 0) out[blockIdx.x] = r;
}

// The tensor amax as per-CTA maxima (no clearing, no atomics): slots must
// hold 2 x SM-count floats; *n_slots gets the count written.
static cudaError_t launch_amax_slots(const void *x, bool bf16, int64_t rows, int64_t cols, int hadamard_b,
                                     float *slots, int *n_slots, cudaStream_t s) {
    *n_slots = 0;
    int64_t chunks = rows * cols / 16;
    if (chunks == 0) return cudaSuccess;
    QuantArgs a;
    memset(&a, 0, sizeof(a));
    a.rows = rows;
    a.cols = cols;
    a.total_chunks = chunks;
    a.cpr = make_fastdiv((uint32_t)(cols / 16 > 0 ? cols / 16 : 1));
    a.hadamard_b = hadamard_b;
    a.amax_out = slots;
    const int64_t cap = (int64_t)sm_count_cached() * 2;
    if (hadamard_b == 0) {
        const int64_t words = chunks * (bf16 ? 2 : 4);
        const int64_t per_cta = (int64_t)kQThreads * kAmaxWords;
        const int64_t want = (words + per_cta - 1) / per_cta;
        const int grid = (int)(want < cap ? want : cap);
        *n_slots = grid;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)grid, 1, 1);
        cfg.blockDim = dim3(kQThreads, 1, 1);
        cfg.stream = s;
        cudaLaunchAttribute attr[1] = {pdl_attribute()};
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (bf16) cudaLaunchKernelEx(&cfg, k_amax_words<true>, (const uint4 *)x, words, slots);
        else cudaLaunchKernelEx(&cfg, k_amax_words<false>, (const uint4 *)x, words, slots);
        return cudaGetLastError();
    }
    const int64_t steps = (chunks + kQThreads - 1) / kQThreads;
    *n_slots = (int)(steps < cap ? steps : cap);
    if (bf16) launch_qf<__nv_bfloat16, kNumFmt>((const __nv_bfloat16 *)x, a, s);
    else launch_qf<float, kNumFmt>((const float *)x, a, s);
    return cudaGetLastError();
}

template <typename T, int F>
static void launch_qf(const T *x, const QuantArgs &a, cudaStream_t s) {
    const int64_t steps = (a.total_chunks + kQThreads - 1) / kQThreads;
    const int64_t cap = (int64_t)sm_count_cached() * 2;   // two 512-thread CTAs per SM
    const int grid = (int)(steps < cap ? steps : cap);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(kQThreads, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1] = {pdl_attribute()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, k_quantize<T, F>, x, a);
}

template <typename T>
static void launch_q(int fmt, const T *x, const QuantArgs &a, cudaStream_t s) {
    switch (fmt) {
    case kMXFP8: launch_qf<T, kMXFP8>(x, a, s); break;
    case kMXFP4: launch_qf<T, kMXFP4>(x, a, s); break;
    case kNVFP4: launch_qf<T, kNVFP4>(x, a, s); break;
    case kINT4G32: launch_qf<T, kINT4G32>(x, a, s); break;
    case kINT4G64: launch_qf<T, kINT4G64>(x, a, s); break;
    case kFP8Tensor: launch_qf<T, kFP8Tensor>(x, a, s); break;
    case kINT8Row: {
        if (sizeof(T) == 2 && a.hadamard_b == 0 && a.cols > 2048 &&
            launch_int8_row_staged(reinterpret_cast<const __nv_bfloat16 *>(x), a, s))
            break;
        int g = grid_for(a.rows, sm_count_cached());
        const int64_t cpr = a.cols >> 4;
        if (a.hadamard_b == 0 && cpr <= 32) k_quantize_int8_row_reg<T, 1><<<g, kThreads, 0, s>>>(x, a);
        else if (a.hadamard_b == 0 && cpr <= 64) k_quantize_int8_row_reg<T, 2><<<g, kThreads, 0, s>>>(x, a);
        else if (a.hadamard_b == 0 && cpr <= 128) k_quantize_int8_row_reg<T, 4><<<g, kThreads, 0, s>>>(x, a);
        else if (a.hadamard_b == 0 && cpr <= 256) k_quantize_int8_row_reg<T, 8><<<g, kThreads, 0, s>>>(x, a);
        else if (a.hadamard_b == 0 && cpr <= 384 && sizeof(T) == 2)   // bf16 rows up to 6144 elements
            k_quantize_int8_row_reg<T, sizeof(T) == 2 ? 12 : 1><<<g, kThreads, 0, s>>>(x, a);
        else k_quantize_int8_row<T><<<g, kThreads, 0, s>>>(x, a);
        break;
    }
    }
}

cudaError_t launch_quantize(const void *x, bool bf16, int64_t rows, int64_t cols, int fmt, int hadamard_b,
                            int layout, void *codes, void *scales, size_t scales_bytes, float *tensor_scale,
                            unsigned int *amax_word, cudaStream_t s, const PackT *pack, bool amax_ready,
                            float mx_grid, const float *amax_slots, int n_slots) {
    cudaError_t e;
    if (fmt_tensor_scaled(fmt) && !amax_ready) {
        // per-CTA maxima in the scratch behind the amax word (kLrHeader bytes)
        float *slots = reinterpret_cast<float *>(reinterpret_cast<char *>(amax_word) + 256);
        e = launch_amax_slots(x, bf16, rows, cols, hadamard_b, slots, &n_slots, s);
        if (e != cudaSuccess) return e;
        amax_slots = slots;
    }
    QuantArgs a;
    a.rows = rows;
    a.cols = cols;
    a.total_chunks = rows * cols / 16;
    a.cpr = make_fastdiv((uint32_t)(cols / 16 > 0 ? cols / 16 : 1));
    a.hadamard_b = hadamard_b;
    a.layout = layout;
    a.s_pad = 0;
    a.codes = (uint8_t *)codes;
    a.scales = scales;
    a.tensor_scale = tensor_scale;
    a.amax_word = amax_word;
    a.amax_slots = amax_slots;
    a.n_slots = n_slots;
    a.mx_grid = mx_grid;
    a.t = pack ? pack->t : nullptr;
    a.r = pack ? pack->r : 0;
    a.w_ts = pack ? pack->w_ts : nullptr;
    a.tp = pack ? (__nv_bfloat16 *)pack->tp : nullptr;
    (void)scales_bytes;   // the whole buffer: k_quantize writes every byte of it, padding included
    if (layout == 1 && fmt_byte_scales(fmt)) {   // k_quantize writes the padding's zero scales itself
        int64_t S = cols / fmt_block(fmt);
        a.s_pad = (S + 15) / 16 * 16;
    }
    if (a.total_chunks == 0) {
        if (fmt_tensor_scaled(fmt)) {   // empty tensor: amax 0 -> scale 1
            static const float one = 1.0f;
            return cudaMemcpyAsync(tensor_scale, &one, sizeof(float), cudaMemcpyHostToDevice, s);
        }
        return cudaSuccess;
    }
    if (bf16) launch_q<__nv_bfloat16>(fmt, (const __nv_bfloat16 *)x, a, s);
    else launch_q<float>(fmt, (const float *)x, a, s);
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
    a.cpr = make_fastdiv((uint32_t)(cols / 16 > 0 ? cols / 16 : 1));
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

// The candidate set as a format mask when it is one of the fixed sets with
// distinct formats (0 otherwise).
static uint32_t select_set_of(const int *cands, int ncand) {
    uint32_t mask = 0;
    for (int j = 0; j < ncand; j++) {
        if (mask & (1u << cands[j])) return 0;   // repeated format
        mask |= 1u << cands[j];
    }
    return (mask == kSelSetW4 || mask == kSelSetA8) ? mask : 0u;
}

template <typename T, uint32_t MASK>
static void launch_select_set(const T *w, const SelectSetArgs &a, cudaStream_t s) {
    const int64_t ctas = (a.n + kSelThreads / 32 - 1) / (kSelThreads / 32);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(ctas < 1 ? 1 : ctas), 1, 1);
    cfg.blockDim = dim3(kSelThreads, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1] = {pdl_attribute()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, k_select_set<T, MASK>, w, a);
}

cudaError_t launch_select_fixed(const void *w, bool bf16, int64_t n, int64_t k, const int *cands, int ncand,
                                uint8_t *choice, double *sse, float *amax_slots, cudaStream_t s) {
    const uint32_t mask = select_set_of(cands, ncand);
    if (!mask || k % 64 || n * (k / 16) >= ((int64_t)1 << 31)) return cudaErrorNotSupported;
    SelectSetArgs a;
    memset(&a, 0, sizeof(a));
    a.n = n;
    a.k = k;
    a.ncand = ncand;
    for (int j = 0; j < ncand; j++) {
        a.cand[j] = cands[j];
        a.slot[j] = sel_slot(mask, cands[j]);
    }
    a.choice = choice;
    a.sse = sse;
    if (mask & ((1u << kNVFP4) | (1u << kFP8Tensor))) {
        // per-CTA maxima of |w| (every slot written, no clearing), read by the
        // selection kernel launched right behind it
        cudaError_t e = launch_amax_slots(w, bf16, n, k, 0, amax_slots, &a.n_slots, s);
        if (e != cudaSuccess) return e;
        a.amax_slots = amax_slots;
    }
    if (n == 0) return cudaSuccess;
    if (mask == kSelSetW4) {
        if (bf16) launch_select_set<__nv_bfloat16, kSelSetW4>((const __nv_bfloat16 *)w, a, s);
        else launch_select_set<float, kSelSetW4>((const float *)w, a, s);
    } else {
        if (bf16) launch_select_set<__nv_bfloat16, kSelSetA8>((const __nv_bfloat16 *)w, a, s);
        else launch_select_set<float, kSelSetA8>((const float *)w, a, s);
    }
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
