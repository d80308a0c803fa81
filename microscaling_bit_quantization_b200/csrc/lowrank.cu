// lowrank.cu -- the SVDQuant low-rank branch outside the GEMM: the down
// projection t = bf16(x) . L1 (optionally with the tensor amax of x in the
// same read), and the packing of t and L2 into the operands of the GEMM's
// extra kind::f16 stage (Nunchaku/Diffusers article, "Main explanation": a
// 16-bit low-rank part of each weight is kept beside the 4-bit residual).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "mxq_formats.cuh"
#include "mxq_internal.h"
#include "tc_ptx.cuh"

namespace mxq {

namespace {


// A-fragment pair (two consecutive k) of row `row`, as packed bf16; the
// running max of |x| is updated from the exact input values.
__device__ __forceinline__ uint32_t ld_pair(const __nv_bfloat16 *x, int64_t m, int64_t k, int64_t row, int64_t col,
                                            float &am) {
    if (row >= m) return 0u;
    const uint32_t v = __ldg(reinterpret_cast<const unsigned int *>(x + row * k + col));
    am = fmaxf(am, fmaxf(fabsf(__uint_as_float(v << 16)), fabsf(__uint_as_float(v & 0xFFFF0000u))));
    return v;
}
__device__ __forceinline__ uint32_t ld_pair(const float *x, int64_t m, int64_t k, int64_t row, int64_t col, float &am) {
    if (row >= m) return 0u;
    const float2 f = __ldg(reinterpret_cast<const float2 *>(x + row * k + col));
    am = fmaxf(am, fmaxf(fabsf(f.x), fabsf(f.y)));
    return pack_bf16x2(f.x, f.y);
}

__device__ __forceinline__ void mma_m16n8k16_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

enum LowrankMode : int { kLrT = 0, kLrPacked = 1, kLrTAmax = 2 };
constexpr int kLrWarps = 8, kLrUnroll = 8;

// t = bf16(x) . l1 with fp32 accumulation (mma.sync m16n8k16; the branch is
// a skinny product bound by reading x from HBM).  CTA = 8 warps over a
// 16-row strip; warp w takes the k16 steps w, w+8, ..., loading eight steps
// of A fragments before their MMAs so that enough bytes are in flight.  The
// eight partial tiles are summed in a fixed order through shared memory.
//   kLrT      t (m x r fp32)
//   kLrPacked the GEMM operand tp (m x 64 bf16, [hi | lo] of t / (xs * ws))
//   kLrTAmax  t, and max |x| over the whole tensor: each CTA's maximum into
//             amax_slots[blockIdx.x], or folded into *amax_word
template <typename T, int MODE>
__global__ void __launch_bounds__(kLrWarps * 32) k_lowrank(const T *__restrict__ x, int64_t m, int64_t k,
                                                         const __nv_bfloat16 *__restrict__ l1, int r,
                                                         float *__restrict__ t, const float *xs, const float *ws,
                                                         __nv_bfloat16 *__restrict__ tp, unsigned int *amax_word,
                                                         float *amax_slots) {
    __shared__ float red[kLrWarps][16][33];
    __shared__ float wmax[kLrWarps];
    // launched with programmatic serialization: nothing global is touched
    // before the previous kernel has completed
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq = lane & 3;
    const int64_t row0 = (int64_t)blockIdx.x * 16;
    const int64_t nks = k >> 4;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) acc[i][j] = 0.0f;
    float am = 0.0f;
    const unsigned short *l1u = reinterpret_cast<const unsigned short *>(l1);
    for (int64_t base = warp; base < nks; base += kLrWarps * kLrUnroll) {
        uint32_t a[kLrUnroll][4];
#pragma unroll
        for (int u = 0; u < kLrUnroll; u++) {
            const int64_t ks = base + (int64_t)u * kLrWarps;
            if (ks < nks) {
                const int64_t kk = ks * 16 + tq * 2;
                a[u][0] = ld_pair(x, m, k, row0 + g, kk, am);
                a[u][1] = ld_pair(x, m, k, row0 + g + 8, kk, am);
                a[u][2] = ld_pair(x, m, k, row0 + g, kk + 8, am);
                a[u][3] = ld_pair(x, m, k, row0 + g + 8, kk + 8, am);
            } else {
                a[u][0] = a[u][1] = a[u][2] = a[u][3] = 0u;
            }
        }
#pragma unroll
        for (int u = 0; u < kLrUnroll; u++) {
            const int64_t ks = base + (int64_t)u * kLrWarps;
            if (ks < nks) {
                const int64_t k0 = ks * 16 + tq * 2;
#pragma unroll
                for (int nt = 0; nt < 4; nt++) {
                    const int n = nt * 8 + g;
                    uint32_t b0 = 0, b1 = 0;
                    if (n < r) {
                        b0 = (uint32_t)__ldg(l1u + k0 * r + n) | ((uint32_t)__ldg(l1u + (k0 + 1) * r + n) << 16);
                        b1 = (uint32_t)__ldg(l1u + (k0 + 8) * r + n) | ((uint32_t)__ldg(l1u + (k0 + 9) * r + n) << 16);
                    }
                    mma_m16n8k16_bf16(acc[nt], a[u], b0, b1);
                }
            }
        }
    }
#pragma unroll
    for (int nt = 0; nt < 4; nt++) {
        red[warp][g][nt * 8 + tq * 2] = acc[nt][0];
        red[warp][g][nt * 8 + tq * 2 + 1] = acc[nt][1];
        red[warp][g + 8][nt * 8 + tq * 2] = acc[nt][2];
        red[warp][g + 8][nt * 8 + tq * 2 + 1] = acc[nt][3];
    }
    if (MODE == kLrTAmax) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
        if (lane == 0) wmax[warp] = am;
    }
    __syncthreads();
    if (MODE == kLrTAmax && threadIdx.x == 0) {
        float v = 0.0f;
        for (int w = 0; w < kLrWarps; w++) v = fmaxf(v, wmax[w]);
        if (amax_slots) amax_slots[blockIdx.x] = v;   // every CTA writes its slot: no clearing
        else if (v > 0.0f) atomicMax(amax_word, __float_as_uint(v));
    }
    float alpha = 1.0f;
    if (MODE == kLrPacked && xs) alpha = __fmul_rn(*xs, *ws);
    for (int i = threadIdx.x; i < 16 * 32; i += kLrWarps * 32) {
        const int rr = i >> 5, cc = i & 31;
        const int64_t row = row0 + rr;
        if (row >= m) continue;
        float sum = red[0][rr][cc];
#pragma unroll
        for (int w = 1; w < kLrWarps; w++) sum = __fadd_rn(sum, red[w][rr][cc]);
        if (MODE != kLrPacked) {
            if (cc < r) t[row * r + cc] = sum;
        } else {
            const float u = cc < r ? (xs ? __fdiv_rn(sum, alpha) : sum) : 0.0f;
            const __nv_bfloat16 hi = __float2bfloat16_rn(u);
            tp[row * 64 + cc] = hi;
            tp[row * 64 + 32 + cc] = __float2bfloat16_rn(__fsub_rn(u, __bfloat162float(hi)));
        }
    }
}

// l2p[j][0..31] = l2[0..31][j] (zero past r); l2p[j][32..63] = the same.
__global__ void k_pack_l2(const __nv_bfloat16 *__restrict__ l2, int r, int64_t n, __nv_bfloat16 *__restrict__ l2p) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n * 32) return;
    const int64_t col = i >> 5;
    const int j = (int)(i & 31);
    const __nv_bfloat16 v = j < r ? l2[(int64_t)j * n + col] : __float2bfloat16_rn(0.0f);
    l2p[col * 64 + j] = v;
    l2p[col * 64 + 32 + j] = v;
}

// tp[i][0..31] = bf16(u), tp[i][32..63] = bf16(u - bf16(u)), u = t / alpha,
// alpha = xs * ws (1 when the format has no tensor scales).
__global__ void k_pack_t(const float *__restrict__ t, int r, int64_t m, const float *xs, const float *ws,
                         __nv_bfloat16 *__restrict__ tp) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= m * 32) return;
    const int64_t row = i >> 5;
    const int j = (int)(i & 31);
    float u = 0.0f;
    if (j < r) {
        u = t[row * r + j];
        if (xs) u = __fdiv_rn(u, __fmul_rn(*xs, *ws));
    }
    const __nv_bfloat16 hi = __float2bfloat16_rn(u);
    const __nv_bfloat16 lo = __float2bfloat16_rn(__fsub_rn(u, __bfloat162float(hi)));
    tp[row * 64 + j] = hi;
    tp[row * 64 + 32 + j] = lo;
}

// ---------------------------------------------------------------------------
// Staged variant for bf16 x (k % 64 == 0, r % 8 == 0): a CTA of 4 warps
// owns a 16-row strip and walks K in 64-wide chunks that cp.async stages into
// shared memory, kLsStages chunks in flight; warp w takes the chunk's k16 step
// w.  Fragments come from shared memory through ldmatrix (A) and
// ldmatrix.trans (B, straight from L1's k x r rows); rows are stored with an
// XOR swizzle of their 16-byte pieces so the eight rows an ldmatrix reads hit
// distinct banks.  max |x| comes from each thread's own staged piece.
constexpr int kLsStages = 12, kLsThreads = 128;
constexpr int kLsX = 16 * 128;            // 16 rows x 64 bf16
constexpr int kLsL1 = 64 * 64;            // 64 k-rows x 32 bf16 (zero-padded past r)
constexpr int kLsStage = kLsX + kLsL1;
constexpr int kLsSmem = kLsStages * kLsStage;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    const int n = valid ? 16 : 0;   // zero-fill rows past m
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
// byte offset of 16-byte piece p of row `row` in a 128-byte-row tile (x) / 64-byte-row tile (L1)
__device__ __forceinline__ uint32_t xs_off(int row, int p) { return row * 128 + ((p ^ (row & 7)) << 4); }
__device__ __forceinline__ uint32_t ls_off(int row, int p) { return row * 64 + ((p ^ ((row >> 1) & 3)) << 4); }

template <int MODE>
__global__ void __launch_bounds__(kLsThreads) k_lowrank_staged(const __nv_bfloat16 *__restrict__ x, int64_t m, int64_t k,
                                                              const __nv_bfloat16 *__restrict__ l1, int r,
                                                              float *__restrict__ t, const float *xs, const float *ws,
                                                              __nv_bfloat16 *__restrict__ tp, unsigned int *amax_word,
                                                              float *amax_slots) {
    extern __shared__ __align__(128) uint8_t ls_smem[];
    __shared__ float red[4][16][33];
    __shared__ float wmax[4];
    pdl_wait();   // as in k_lowrank
    pdl_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t row0 = (int64_t)blockIdx.x * 16;
    const int nchunks = (int)(k >> 6);
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(ls_smem);
    const int pieces_l1 = r >> 3;   // 16-byte pieces per L1 row
    // L1 tiles: columns past r stay zero
    for (int i = tid; i < kLsStages * kLsL1 / 16; i += kLsThreads) {
        const int st = i / (kLsL1 / 16), q = i % (kLsL1 / 16);
        *reinterpret_cast<uint4 *>(ls_smem + st * kLsStage + kLsX + q * 16) = make_uint4(0, 0, 0, 0);
    }
    __syncthreads();
    // thread tid stages x piece (row tid / 8, piece tid % 8) and L1 pieces tid, tid + 128
    const int xr = tid >> 3, xp = tid & 7;
    const bool xrow_ok = row0 + xr < m;
    const __nv_bfloat16 *xsrc = x + (row0 + (xrow_ok ? xr : 0)) * k + xp * 8;
    auto issue = [&](int c) {
        const uint32_t st = sbase + (uint32_t)((c % kLsStages) * kLsStage);
        cp_async16(st + xs_off(xr, xp), xsrc + (int64_t)c * 64, xrow_ok);
        for (int i = tid; i < 64 * pieces_l1; i += kLsThreads) {
            const int kr = i / pieces_l1, pc = i % pieces_l1;
            cp_async16(st + kLsX + ls_off(kr, pc), l1 + ((int64_t)c * 64 + kr) * r + pc * 8, true);
        }
    };
#pragma unroll 1
    for (int c = 0; c < kLsStages - 1; c++) {
        if (c < nchunks) issue(c);
        cp_async_commit();
    }
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) acc[i][j] = 0.0f;
    float am = 0.0f;
    // ldmatrix row addresses (lane supplies row lane % 8 of matrix lane / 8)
    const int mi = lane >> 3, mr = lane & 7;
    const int a_row = mr + 8 * (mi & 1), a_piece = 2 * warp + (mi >> 1);
    const int b_row = 16 * warp + mr + 8 * (mi & 1);
#pragma unroll 1
    for (int c = 0; c < nchunks; c++) {
        cp_async_wait<kLsStages - 2>();
        __syncthreads();
        if (c + kLsStages - 1 < nchunks) issue(c + kLsStages - 1);
        cp_async_commit();
        const uint32_t st = sbase + (uint32_t)((c % kLsStages) * kLsStage);
        if (MODE == kLrTAmax) {
            const uint4 v = *reinterpret_cast<const uint4 *>(ls_smem + (c % kLsStages) * kLsStage + xs_off(xr, xp));
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; j++)
                am = fmaxf(am, fmaxf(fabsf(__uint_as_float(w4[j] << 16)), fabsf(__uint_as_float(w4[j] & 0xFFFF0000u))));
        }
        uint32_t a[4], b01[4], b23[4];
        ldsm_x4(st + xs_off(a_row, a_piece), a);
        ldsm_x4_trans(st + kLsX + ls_off(b_row, mi >> 1), b01);
        ldsm_x4_trans(st + kLsX + ls_off(b_row, 2 + (mi >> 1)), b23);
        mma_m16n8k16_bf16(acc[0], a, b01[0], b01[1]);
        mma_m16n8k16_bf16(acc[1], a, b01[2], b01[3]);
        mma_m16n8k16_bf16(acc[2], a, b23[0], b23[1]);
        mma_m16n8k16_bf16(acc[3], a, b23[2], b23[3]);
    }
    cp_async_wait<0>();
    const int g = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 4; nt++) {
        red[warp][g][nt * 8 + tq * 2] = acc[nt][0];
        red[warp][g][nt * 8 + tq * 2 + 1] = acc[nt][1];
        red[warp][g + 8][nt * 8 + tq * 2] = acc[nt][2];
        red[warp][g + 8][nt * 8 + tq * 2 + 1] = acc[nt][3];
    }
    if (MODE == kLrTAmax) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
        if (lane == 0) wmax[warp] = am;
    }
    __syncthreads();
    if (MODE == kLrTAmax && tid == 0) {
        const float v = fmaxf(fmaxf(wmax[0], wmax[1]), fmaxf(wmax[2], wmax[3]));
        if (amax_slots) amax_slots[blockIdx.x] = v;   // every CTA writes its slot: no clearing
        else if (v > 0.0f) atomicMax(amax_word, __float_as_uint(v));
    }
    float alpha = 1.0f;
    if (MODE == kLrPacked && xs) alpha = __fmul_rn(*xs, *ws);
    for (int i = tid; i < 16 * 32; i += kLsThreads) {
        const int rr = i >> 5, cc = i & 31;
        const int64_t row = row0 + rr;
        if (row >= m) continue;
        const float sum = __fadd_rn(__fadd_rn(red[0][rr][cc], red[1][rr][cc]), __fadd_rn(red[2][rr][cc], red[3][rr][cc]));
        if (MODE != kLrPacked) {
            if (cc < r) t[row * r + cc] = sum;
        } else {
            const float u = cc < r ? (xs ? __fdiv_rn(sum, alpha) : sum) : 0.0f;
            const __nv_bfloat16 hi = __float2bfloat16_rn(u);
            tp[row * 64 + cc] = hi;
            tp[row * 64 + 32 + cc] = __float2bfloat16_rn(__fsub_rn(u, __bfloat162float(hi)));
        }
    }
}

}  // namespace

// One launch with the programmatic-serialization attribute.
template <typename... P, typename... A>
static cudaError_t launch_pdl(void (*kern)(P...), int grid, int threads, size_t smem, cudaStream_t s, A... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3((unsigned)threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1] = {pdl_attribute()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <typename T>
static cudaError_t launch_lr(int mode, int grid, const T *x, int64_t m, int64_t k, const __nv_bfloat16 *l1, int r,
                             float *t, const float *xs, const float *ws, __nv_bfloat16 *tp, unsigned int *amax,
                             float *slots, cudaStream_t s) {
    const int threads = kLrWarps * 32;
    auto kern = mode == kLrT ? k_lowrank<T, kLrT> : mode == kLrPacked ? k_lowrank<T, kLrPacked> : k_lowrank<T, kLrTAmax>;
    return launch_pdl(kern, grid, threads, 0, s, x, m, k, l1, r, t, xs, ws, tp, amax, slots);
}

cudaError_t launch_lowrank_down(const void *x, bool bf16, int64_t m, int64_t k, const void *l1, int r, float *t,
                                const float *xs, const float *ws, void *tp, cudaStream_t s, unsigned int *amax_word,
                                float *amax_slots, int *n_slots) {
    if (m == 0) return cudaSuccess;
    if (bf16 && !amax_word && !amax_slots) {   // the tensor-core path when it takes the shape (its amax goes to slots)
        const cudaError_t e = launch_lowrank_tc(x, m, k, l1, r, tp ? nullptr : t, tp, xs, ws, nullptr, nullptr, s);
        if (e != cudaErrorNotSupported) return e;
    }
    const int64_t grid64 = (m + 15) / 16;
    if (amax_slots && (tp || grid64 > kAmaxSlots)) return cudaErrorNotSupported;   // one slot per CTA
    const int grid = (int)grid64;
    const int mode = tp ? kLrPacked : ((amax_word || amax_slots) ? kLrTAmax : kLrT);
    if (amax_slots) *n_slots = grid;
    const __nv_bfloat16 *l = (const __nv_bfloat16 *)l1;
    __nv_bfloat16 *tpb = (__nv_bfloat16 *)tp;
    if (bf16 && k % 64 == 0 && r % 8 == 0 && (reinterpret_cast<uintptr_t>(l1) & 15u) == 0) {
        static PerDeviceOnce smem_opt_in;
        const cudaError_t se = smem_opt_in.run([] {
            cudaError_t e = cudaFuncSetAttribute(k_lowrank_staged<kLrT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kLsSmem);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(k_lowrank_staged<kLrPacked>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kLsSmem);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(k_lowrank_staged<kLrTAmax>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kLsSmem);
            return e;
        });
        if (se != cudaSuccess) return se;
        const __nv_bfloat16 *xb = (const __nv_bfloat16 *)x;
        auto kern = mode == kLrT ? k_lowrank_staged<kLrT>
                  : mode == kLrPacked ? k_lowrank_staged<kLrPacked> : k_lowrank_staged<kLrTAmax>;
        return launch_pdl(kern, grid, kLsThreads, (size_t)kLsSmem, s, xb, m, k, l, r, t, xs, ws, tpb, amax_word,
                          amax_slots);
    }
    if (bf16) return launch_lr(mode, grid, (const __nv_bfloat16 *)x, m, k, l, r, t, xs, ws, tpb, amax_word, amax_slots, s);
    return launch_lr(mode, grid, (const float *)x, m, k, l, r, t, xs, ws, tpb, amax_word, amax_slots, s);
}

cudaError_t launch_pack_l2(const void *l2, int r, int64_t n, void *l2p, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const int64_t total = n * 32;
    k_pack_l2<<<(unsigned)((total + 255) / 256), 256, 0, s>>>((const __nv_bfloat16 *)l2, r, n, (__nv_bfloat16 *)l2p);
    return cudaGetLastError();
}

cudaError_t launch_pack_t(const float *t, int r, int64_t m, const float *xs, const float *ws, void *tp, cudaStream_t s) {
    if (m == 0) return cudaSuccess;
    const int64_t total = m * 32;
    k_pack_t<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(t, r, m, xs, ws, (__nv_bfloat16 *)tp);
    return cudaGetLastError();
}

}  // namespace mxq
