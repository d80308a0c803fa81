// mixed.cu -- the linear layer whose weight keeps one format per output
// channel (Chameleon article, section "the format is chosen by the value
// distribution": each output channel takes the format with the least
// reconstruction error among INT4-g32, NVFP4 and MXFP4; the article's note on
// hardware support says such a mix needs native kernels, splitting the GEMM
// into groups or unpacking in the kernel).  Here the channels are split into
// per-format groups, each group runs on the tensor cores in the MMA kind that
// takes it exactly against MXFP8 activations, and the group outputs are
// scattered back to channel order:
//   MXFP4 rows     every E2M1 value is an E4M3 value, so the rows are stored
//                  as E4M3 bytes with their E8M0 scales and multiply the
//                  MXFP8 activation on kind::mxf8f6f4 (block scales applied by
//                  the tensor cores);
//   INT4-g32 rows  the integer codes as E4M3 bytes; the group GEMM forms each
//                  32-element group's product of codes on kind::f8f6f4 and
//                  adds it times (activation block scale 2^e) x (weight group
//                  scale) in fp32;
//   NVFP4 rows     an E2M1 value times its E4M3 block scale has at most 6
//                  significant bits, exact in bf16 but in no 8-bit format, and
//                  the 16-element block scales differ inside a 32-element MX
//                  block, so these rows are stored as those bf16 products and
//                  multiply the activation dequantized to bf16 (exact for
//                  block exponents inside the bf16 range) on kind::f16, the
//                  tensor scale applied in the epilogue.
// This file holds the preparation of the weight groups, the activation-side
// conversions and the scatter; the GEMMs are gemm.cu and gemm_igroup.cu.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "mxq_formats.cuh"
#include "mxq_internal.h"

namespace mxq {

namespace {

constexpr int kMixThreads = 256;

// Group of a format: 0 MXFP4, 1 INT4_G32, 2 NVFP4 (-1 otherwise).
__host__ __device__ __forceinline__ int mixed_group_of(int f) {
    return f == kMXFP4 ? 0 : f == kINT4G32 ? 1 : f == kNVFP4 ? 2 : -1;
}

// E8M0 block scales of an MX tensor in the MMA layout -> fp32 2^(b - 127),
// transposed [blocks][m] (the activation-side group scales of the group GEMM).
__global__ void __launch_bounds__(kMixThreads) k_mx_scales_f32(const uint8_t *__restrict__ sc, uint32_t m,
                                                               uint32_t nblk, uint32_t s_pad4, float *__restrict__ out) {
    const uint64_t total = (uint64_t)m * nblk;
    for (uint64_t i = (uint64_t)blockIdx.x * kMixThreads + threadIdx.x; i < total;
         i += (uint64_t)gridDim.x * kMixThreads) {
        const uint32_t g = (uint32_t)(i / m), r = (uint32_t)(i - (uint64_t)g * m);
        out[i] = dec_e8m0(sc[mma_scale_offset32(r, g, s_pad4)]);
    }
}

struct MixedPrepArgs {
    int64_t n, k;
    const uint8_t *choice;
    const int32_t *gidx;
    const uint8_t *mx_codes_c, *mx_scales_c;   // whole weight, canonical MXFP4
    const uint8_t *i4_codes_c;                 // whole weight, canonical INT4_G32
    const float *i4_scales_c;
    const uint8_t *nv_codes_c, *nv_scales_c;   // whole weight, canonical NVFP4
    uint8_t *mx_codes, *mx_scales;             // [n_mx][k] E4M3 bytes, MMA-layout E8M0 scales
    uint32_t mx_spad4;
    uint8_t *i4_codes;                         // [n_i4][k] E4M3 bytes
    float *i4_scales;                          // [k/32][n_i4]
    int64_t n_i4;
    __nv_bfloat16 *nv_vals;                    // [n_nv][k]
};

// One thread per 16-element chunk of a weight row: the chunk of the row's
// chosen format re-laid into its group's operand.
__global__ void __launch_bounds__(kMixThreads) k_mixed_prep(MixedPrepArgs a) {
    const int64_t cpr = a.k >> 4;
    const int64_t total = a.n * cpr;
    for (int64_t i = (int64_t)blockIdx.x * kMixThreads + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * kMixThreads) {
        const int64_t n = i / cpr, c = i - n * cpr;
        const int f = a.choice[n];
        const int64_t p = a.gidx[n];
        if (f == kMXFP4 || f == kINT4G32) {
            const uint2 raw = *reinterpret_cast<const uint2 *>((f == kMXFP4 ? a.mx_codes_c : a.i4_codes_c) + i * 8);
            const uint32_t w[2] = {raw.x, raw.y};
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; j++) {
                const uint32_t nib = (w[j >> 3] >> (4 * (j & 7))) & 0xFu;
                // E2M1 value, or the two's-complement integer (never -8)
                v[j] = f == kMXFP4 ? dec_e2m1(nib) : (float)((int)(nib << 28) >> 28);
                if (v[j] == 0.0f) v[j] = 0.0f;   // zeros are written as +0
            }
            uint4 o;
            o.x = cvt_e4m3x4(v[0], v[1], v[2], v[3]);
            o.y = cvt_e4m3x4(v[4], v[5], v[6], v[7]);
            o.z = cvt_e4m3x4(v[8], v[9], v[10], v[11]);
            o.w = cvt_e4m3x4(v[12], v[13], v[14], v[15]);
            if (f == kMXFP4) {
                *reinterpret_cast<uint4 *>(a.mx_codes + p * a.k + c * 16) = o;
                if ((c & 1) == 0)
                    a.mx_scales[mma_scale_offset32((uint32_t)p, (uint32_t)(c >> 1), a.mx_spad4)] =
                        a.mx_scales_c[n * (a.k >> 5) + (c >> 1)];
            } else {
                *reinterpret_cast<uint4 *>(a.i4_codes + p * a.k + c * 16) = o;
                if ((c & 1) == 0) a.i4_scales[(c >> 1) * a.n_i4 + p] = a.i4_scales_c[n * (a.k >> 5) + (c >> 1)];
            }
        } else if (f == kNVFP4) {
            const uint2 raw = *reinterpret_cast<const uint2 *>(a.nv_codes_c + i * 8);
            const uint32_t w[2] = {raw.x, raw.y};
            const float e4 = dec_e4m3(a.nv_scales_c[i]);   // the chunk is one 16-element block
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; j++) v[j] = __fmul_rn(dec_e2m1((w[j >> 3] >> (4 * (j & 7))) & 0xFu), e4);   // exact
            store16(a.nv_vals + p * a.k + c * 16, v);   // exact in bf16 (at most 6 significant bits)
        }
    }
}

// y[row][col] = group output of column col's format, at the column's place in its group.
template <typename T>
__global__ void __launch_bounds__(kMixThreads) k_mixed_scatter(const T *__restrict__ y0, const T *__restrict__ y1,
                                                               const T *__restrict__ y2, int64_t n0, int64_t n1,
                                                               int64_t n2, const uint8_t *__restrict__ choice,
                                                               const int32_t *__restrict__ gidx, T *__restrict__ y,
                                                               int64_t m, int64_t n, int rows_per_cta) {
    const int64_t col = (int64_t)blockIdx.x * kMixThreads + threadIdx.x;
    if (col >= n) return;
    const int g = mixed_group_of(choice[col]);
    const T *src = g == 0 ? y0 : g == 1 ? y1 : y2;
    const int64_t pitch = g == 0 ? n0 : g == 1 ? n1 : n2;
    const int64_t p = gidx[col];
    const int64_t r0 = (int64_t)blockIdx.y * rows_per_cta;
    const int64_t r1 = r0 + rows_per_cta < m ? r0 + rows_per_cta : m;
    for (int64_t r = r0; r < r1; r++) y[r * n + col] = src[r * pitch + p];
}

}  // namespace

cudaError_t launch_mx_scales_f32(const void *scales_mma, int64_t m, int64_t k, float *out, cudaStream_t s) {
    const int64_t nblk = k / 32;
    if (m == 0 || nblk == 0) return cudaSuccess;
    const uint32_t s_pad4 = (uint32_t)(((nblk + 15) / 16 * 16) / 4);
    const int64_t total = m * nblk;
    int64_t grid = (total + kMixThreads - 1) / kMixThreads;
    const int64_t cap = (int64_t)sm_count() * 8;
    k_mx_scales_f32<<<(unsigned)(grid < cap ? grid : cap), kMixThreads, 0, s>>>(
        (const uint8_t *)scales_mma, (uint32_t)m, (uint32_t)nblk, s_pad4, out);
    return cudaGetLastError();
}

cudaError_t launch_mixed_prep(const MixedPrep &q, cudaStream_t s) {
    if (q.n == 0) return cudaSuccess;
    if (q.mx_scales_bytes) {   // padding of the MMA scale layout must read as 0
        const cudaError_t e = cudaMemsetAsync(q.mx_scales, 0, q.mx_scales_bytes, s);
        if (e != cudaSuccess) return e;
    }
    MixedPrepArgs a;
    memset(&a, 0, sizeof(a));
    a.n = q.n;
    a.k = q.k;
    a.choice = q.choice;
    a.gidx = q.group_index;
    a.mx_codes_c = (const uint8_t *)q.mx_codes_c;
    a.mx_scales_c = (const uint8_t *)q.mx_scales_c;
    a.i4_codes_c = (const uint8_t *)q.i4_codes_c;
    a.i4_scales_c = q.i4_scales_c;
    a.nv_codes_c = (const uint8_t *)q.nv_codes_c;
    a.nv_scales_c = (const uint8_t *)q.nv_scales_c;
    a.mx_codes = (uint8_t *)q.mx_codes;
    a.mx_scales = (uint8_t *)q.mx_scales;
    a.mx_spad4 = (uint32_t)(((q.k / 32 + 15) / 16 * 16) / 4);
    a.i4_codes = (uint8_t *)q.i4_codes;
    a.i4_scales = q.i4_scales;
    a.n_i4 = q.n_group[1];
    a.nv_vals = (__nv_bfloat16 *)q.nv_vals;
    const int64_t total = q.n * (q.k / 16);
    int64_t grid = (total + kMixThreads - 1) / kMixThreads;
    const int64_t cap = (int64_t)sm_count() * 8;
    k_mixed_prep<<<(unsigned)(grid < cap ? grid : cap), kMixThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_mixed_scatter(const void *const ybuf[3], const int64_t n_group[3], const uint8_t *choice,
                                 const int32_t *group_index, void *y, bool y_bf16, int64_t m, int64_t n,
                                 cudaStream_t s) {
    if (m == 0 || n == 0) return cudaSuccess;
    int rows_per_cta = 32;
    while ((m + rows_per_cta - 1) / rows_per_cta > 65535) rows_per_cta *= 2;
    dim3 grid((unsigned)((n + kMixThreads - 1) / kMixThreads), (unsigned)((m + rows_per_cta - 1) / rows_per_cta));
    if (y_bf16)
        k_mixed_scatter<__nv_bfloat16><<<grid, kMixThreads, 0, s>>>(
            (const __nv_bfloat16 *)ybuf[0], (const __nv_bfloat16 *)ybuf[1], (const __nv_bfloat16 *)ybuf[2],
            n_group[0], n_group[1], n_group[2], choice, group_index, (__nv_bfloat16 *)y, m, n, rows_per_cta);
    else
        k_mixed_scatter<float><<<grid, kMixThreads, 0, s>>>((const float *)ybuf[0], (const float *)ybuf[1],
                                                            (const float *)ybuf[2], n_group[0], n_group[1], n_group[2],
                                                            choice, group_index, (float *)y, m, n, rows_per_cta);
    return cudaGetLastError();
}

}  // namespace mxq
