// w4a16.cu -- W4A16 linear on 5th-generation tensor cores: bf16 activations
// against INT4 per-group weights that are dequantized to bf16 in shared
// memory (Nunchaku/Diffusers article, awq_w4a16: 4-bit weights with 16-bit
// activations, the kernel family beside svdq_w4a4).
//
// Y = bf16(X) . W16^T with W16 = bf16(RN32(q s)) (q the signed INT4 code, s
// its group's fp32 scale), products exact in the tensor core, fp32
// accumulation.
//
// Structure.  Persistent CTAs walk 128 x 128 output tiles; K runs in
// 64-column stages through a 6-stage ring.  Per CTA (448 threads):
//   warp 0      TMA producer: the 128 x 64 bf16 tile of X (128B swizzle)
//   warp 1      TMEM allocation (two 128-column accumulators) and the MMA
//               thread: four kind::f16 M=128 N=128 K=16 MMAs per stage
//   warps 2-9   converters: thread t of the 256 owns half h = t / 128 of
//               weight row n0 + t % 128 of the tile; it loads that half's 32
//               codes (16 bytes) and group scale eight stages ahead, writes
//               bf16(RN32(q s)) as four 16-byte units in the 128B-swizzled
//               K-major layout the MMA reads, makes them visible to the
//               tensor cores (fence.proxy.async) and arrives on the stage's
//               B barrier (one arrival per warp); two converter warps per
//               scheduler, so one's fence and loads overlap the other's work
//   warps 10-13 epilogue: TMEM -> registers -> bf16 / fp32 -> global
// Every wait is bounded; one that runs out latches the error word, the CTA
// stops issuing work, lets what is in flight land and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "mxq_formats.cuh"
#include "mxq_internal.h"
#include "tc_ptx.cuh"

namespace mxq {
namespace {

constexpr int WA_STAGES = 6;
constexpr int WA_A = 128 * 128;          // 128 rows x 64 bf16 of X
constexpr int WA_B = 128 * 128;          // 128 weight rows x 64 bf16
constexpr int WA_STAGE = WA_A + WA_B;
constexpr int WA_THREADS = 448;
constexpr int WA_SMEM = WA_STAGES * WA_STAGE + 512 + 1024;
constexpr uint32_t WA_TMEM_COLS = 256;
constexpr unsigned int kErrW4a16 = 128u;
constexpr int WA_DEPTH = 8;              // stages of codes a converter thread keeps in flight

// M = 128, N = 128, bf16 x bf16 -> fp32, K-major A and B.
constexpr uint32_t kWaIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

struct W4a16Params {
    CUtensorMap tma_x;
    const uint8_t *codes;   // n x k/2, two's-complement nibbles, element 2i low
    const float *scales;    // n x k/g
    void *y;
    int m, n, k, g, kb_total, m_tiles, n_tiles, y_bf16, y_vec;   // y_vec: y 16-byte aligned
    unsigned int *err;
    unsigned long long wait_ns;
};

__device__ __forceinline__ void tma_load_a(const CUtensorMap *map, void *dst, uint64_t *bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void mma_wa(uint32_t d, uint64_t a, uint64_t b, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(kWaIdesc), "r"(acc));
}
__device__ __forceinline__ void commit_wa(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// Eight signed 4-bit codes (one word, element 2i in the low nibble of byte i)
// times s, each rounded to fp32 then to bf16, packed two per word in K order.
__device__ __forceinline__ uint4 dequant8(uint32_t w, float s) {
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const uint32_t b = (w >> (8 * i)) & 0xFFu;
        // 2^23 + (q + 8) as fp32 bits, minus 2^23 + 8: q exactly
        const float q0 = __fsub_rn(__uint_as_float(0x4B000000u | ((b & 0xFu) ^ 8u)), 8388616.0f);
        const float q1 = __fsub_rn(__uint_as_float(0x4B000000u | ((b >> 4) ^ 8u)), 8388616.0f);
        const __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(q0, s), __fmul_rn(q1, s));
        out[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

// One converter thread's input for one stage: the 32 codes (16 bytes) of
// half h of its weight row and that half's group scale.
struct CodeRow {
    uint4 c;
    float s;
};
__device__ __forceinline__ CodeRow fetch_row(const W4a16Params &p, int u, int total, int row, int h) {
    CodeRow r;
    r.c = make_uint4(0u, 0u, 0u, 0u);
    r.s = 0.0f;
    if (u >= total) return r;
    const int tile = (int)blockIdx.x + (u / p.kb_total) * (int)gridDim.x, kb = u % p.kb_total;
    const int n = (tile % p.n_tiles) * 128 + row;
    if (n >= p.n) return r;   // rows past N: zero codes
    r.c = __ldg(reinterpret_cast<const uint4 *>(p.codes + (int64_t)n * (p.k >> 1) + kb * 32 + h * 16));
    r.s = __ldg(p.scales + (int64_t)n * (p.k / p.g) + (kb * 64 + h * 32) / p.g);
    return r;
}

__global__ void __launch_bounds__(WA_THREADS, 1) k_w4a16(const __grid_constant__ W4a16Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *afull = reinterpret_cast<uint64_t *>(smem + WA_STAGES * WA_STAGE);
    uint64_t *bfull = afull + WA_STAGES;
    uint64_t *empty = bfull + WA_STAGES;
    uint64_t *accf = empty + WA_STAGES;
    uint64_t *acce = accf + 2;
    uint64_t *drain = acce + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles = p.m_tiles * p.n_tiles;
    const int my_tiles = (int)blockIdx.x < tiles ? (tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
    const int total = my_tiles * p.kb_total;   // stages this CTA runs

    if (threadIdx.x == 0) {
        for (int s = 0; s < WA_STAGES; s++) {
            mbar_init(afull + s, 1);
            mbar_init(bfull + s, 8);   // one arrival per converter warp
            mbar_init(empty + s, 1);   // the MMA commit
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(accf + i, 1);
            mbar_init(acce + i, 4);    // one arrival per epilogue warp
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(WA_TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------- producer (A)
        if (lane == 0) {
            int issued = 0;
            for (int u = 0; u < total && !*abort_flag; u++) {
                const int s = u % WA_STAGES;
                if (!mbar_wait(empty + s, ((u / WA_STAGES) & 1) ^ 1, p.wait_ns)) {
                    atomicOr(p.err, kErrW4a16);
                    *abort_flag = 1;
                    break;
                }
                const int tile = (int)blockIdx.x + (u / p.kb_total) * (int)gridDim.x, kb = u % p.kb_total;
                mbar_arrive_expect_tx(afull + s, WA_A);
                tma_load_a(&p.tma_x, smem + s * WA_STAGE, afull + s, kb * 64, (tile / p.n_tiles) * 128);
                issued = u + 1;
            }
            if (*abort_flag) {   // let the copies in flight land
                for (int i = (issued > WA_STAGES ? issued - WA_STAGES : 0); i < issued; i++)
                    mbar_wait(afull + (i % WA_STAGES), (i / WA_STAGES) & 1, p.wait_ns);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int u = 0;
            bool any = false;
            for (int tc = 0; tc < my_tiles && !*abort_flag; tc++) {
                const uint32_t slot = (uint32_t)(tc & 1);
                bool ok = mbar_wait(acce + slot, ((tc >> 1) & 1) ^ 1, p.wait_ns);
                tc_fence_after();
                for (int kb = 0; ok && kb < p.kb_total; kb++, u++) {
                    const int s = u % WA_STAGES;
                    const uint32_t ph = (u / WA_STAGES) & 1;
                    ok = mbar_wait(afull + s, ph, p.wait_ns) && mbar_wait(bfull + s, ph, p.wait_ns);
                    if (!ok || *abort_flag) break;
                    tc_fence_after();
                    uint8_t *sa = smem + s * WA_STAGE;
#pragma unroll
                    for (int ks = 0; ks < 4; ks++)
                        mma_wa(tmem + slot * 128, sdesc_sw128(sa + ks * 32), sdesc_sw128(sa + WA_A + ks * 32),
                               (kb > 0 || ks > 0) ? 1u : 0u);
                    commit_wa(empty + s);
                    any = true;
                }
                if (!ok || *abort_flag) {
                    if (!ok) atomicOr(p.err, kErrW4a16);
                    *abort_flag = 1;
                    break;
                }
                commit_wa(accf + slot);
            }
            if (*abort_flag && any) {   // nothing may be in flight when TMEM is released
                commit_wa(drain);
                mbar_wait(drain, 0, p.wait_ns);
            }
        }
    } else if (warp < 10) {
        // ---------------------------------------------------------- converters (B)
        const int t = (threadIdx.x - 64) & 127, h = (threadIdx.x - 64) >> 7;   // weight row, half of it
        CodeRow ring[WA_DEPTH];
#pragma unroll
        for (int i = 0; i < WA_DEPTH; i++) ring[i] = fetch_row(p, i, total, t, h);
        // stage u uses buffer u % WA_DEPTH; the turn loop has a fixed trip count
        // (no break inside) so it unrolls and the buffers stay in registers
        bool ok = true;
#pragma unroll 1
        for (int u0 = 0; u0 < total && ok; u0 += WA_DEPTH) {
#pragma unroll
            for (int j = 0; j < WA_DEPTH; j++) {
                const int u = u0 + j;
                if (u < total && ok) {   // uniform over the warp
                    const int s = u % WA_STAGES;
                    bool w_ok = !*abort_flag && mbar_wait(empty + s, ((u / WA_STAGES) & 1) ^ 1, p.wait_ns);
                    w_ok = __all_sync(0xFFFFFFFFu, w_ok);
                    if (w_ok) {
                        const CodeRow cr = ring[j];
                        ring[j] = fetch_row(p, u + WA_DEPTH, total, t, h);
                        const uint32_t words[4] = {cr.c.x, cr.c.y, cr.c.z, cr.c.w};
                        uint8_t *brow = smem + s * WA_STAGE + WA_A + t * 128;
#pragma unroll
                        for (int i = 0; i < 4; i++) {   // 16-byte unit c = 4h + i: elements 8c .. 8c + 7
                            const int c = 4 * h + i;
                            *reinterpret_cast<uint4 *>(brow + ((c ^ (t & 7)) << 4)) = dequant8(words[i], cr.s);
                        }
                        fence_async_smem();   // generic-proxy writes visible to the tensor cores
                        __syncwarp();
                        if (lane == 0) mbar_arrive_local(bfull + s);
                    }
                    ok = w_ok;
                }
            }
        }
        if (!ok) {
            if (lane == 0 && !*abort_flag) atomicOr(p.err, kErrW4a16);
            *abort_flag = 1;
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;   // TMEM lane quarter this warp may access
        for (int tc = 0; tc < my_tiles; tc++) {
            const int tile = (int)blockIdx.x + tc * (int)gridDim.x;
            const int m0 = (tile / p.n_tiles) * 128, n0 = (tile % p.n_tiles) * 128;
            const uint32_t slot = (uint32_t)(tc & 1);
            bool ok = !*abort_flag && mbar_wait(accf + slot, (tc >> 1) & 1, p.wait_ns);
            ok = __all_sync(0xFFFFFFFFu, ok);
            if (!ok) {
                if (lane == 0 && !*abort_flag) atomicOr(p.err, kErrW4a16);
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const int row = m0 + q * 32 + lane;
            for (int c = 0; c < 4; c++) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + slot * 128 + (uint32_t)(c * 32), r);
                if (c == 3) {   // the accumulator is drained
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_local(acce + slot);
                }
                const int nb = n0 + c * 32;
                if (row >= p.m || nb >= p.n) continue;
                if (p.y_bf16) {
                    __nv_bfloat16 *yrow = reinterpret_cast<__nv_bfloat16 *>(p.y) + (int64_t)row * p.n + nb;
                    if (p.y_vec && nb + 32 <= p.n && p.n % 8 == 0) {
#pragma unroll
                        for (int k4 = 0; k4 < 4; k4++)
                            reinterpret_cast<uint4 *>(yrow)[k4] = make_uint4(
                                pack_bf16x2(__uint_as_float(r[8 * k4]), __uint_as_float(r[8 * k4 + 1])),
                                pack_bf16x2(__uint_as_float(r[8 * k4 + 2]), __uint_as_float(r[8 * k4 + 3])),
                                pack_bf16x2(__uint_as_float(r[8 * k4 + 4]), __uint_as_float(r[8 * k4 + 5])),
                                pack_bf16x2(__uint_as_float(r[8 * k4 + 6]), __uint_as_float(r[8 * k4 + 7])));
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; j++)
                            if (nb + j < p.n) yrow[j] = __float2bfloat16_rn(__uint_as_float(r[j]));
                    }
                } else {
                    float *yrow = reinterpret_cast<float *>(p.y) + (int64_t)row * p.n + nb;
                    if (p.y_vec && nb + 32 <= p.n && p.n % 4 == 0) {
#pragma unroll
                        for (int k4 = 0; k4 < 8; k4++)
                            reinterpret_cast<float4 *>(yrow)[k4] =
                                make_float4(__uint_as_float(r[4 * k4]), __uint_as_float(r[4 * k4 + 1]),
                                            __uint_as_float(r[4 * k4 + 2]), __uint_as_float(r[4 * k4 + 3]));
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; j++)
                            if (nb + j < p.n) yrow[j] = __uint_as_float(r[j]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(WA_TMEM_COLS));
    }
}

}  // namespace

cudaError_t launch_w4a16(const void *x, int64_t m, int64_t k, const uint8_t *codes, const float *scales, int64_t n,
                         int g, void *y, bool y_bf16, cudaStream_t s) {
    if (m == 0 || n == 0) return cudaSuccess;
    W4a16Params p;
    memset(&p, 0, sizeof(p));
    if (!encode_2d(&p.tma_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)k, (uint64_t)m, (uint64_t)k * 2, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    p.codes = codes;
    p.scales = scales;
    p.y = y;
    p.m = (int)m;
    p.n = (int)n;
    p.k = (int)k;
    p.g = g;
    p.kb_total = (int)(k / 64);
    p.m_tiles = (int)((m + 127) / 128);
    p.n_tiles = (int)((n + 127) / 128);
    p.y_bf16 = y_bf16 ? 1 : 0;
    p.y_vec = (reinterpret_cast<uintptr_t>(y) & 15u) == 0;
    p.wait_ns = 2000000000ull;   // 2 s
    cudaError_t e = error_word_address(&p.err);
    if (e != cudaSuccess) return e;
    static PerDeviceOnce smem_opt_in;
    e = smem_opt_in.run([] { return cudaFuncSetAttribute(k_w4a16, cudaFuncAttributeMaxDynamicSharedMemorySize, WA_SMEM); });
    if (e != cudaSuccess) return e;
    const int sms = sm_count();
    const int tiles = p.m_tiles * p.n_tiles;
    const int grid = tiles < sms ? tiles : sms;
    k_w4a16<<<grid, WA_THREADS, WA_SMEM, s>>>(p);
    return cudaGetLastError();
}

}  // namespace mxq
