// qlinear.cu -- block-scaled low-bit GEMM on 5th-generation tensor cores
// (tcgen05) with the dequantization epilogue and the SVDQuant low-rank
// branch fused, plus the small kernels that feed the branch.
//
// Sources: Nunchaku/Diffusers article -- svdq_w4a4 runs attention and MLP
// linears with 4-bit weights and activations (INT4 and NVFP4 variants) and
// keeps a 16-bit low-rank part of each weight beside the 4-bit residual
// (sections "Main explanation", "Kernels and supported hardware");
// Chameleon article -- W8A8 formats per layer and timestep interval;
// MixDiT article section 1 -- with shared block exponents a multiply is a
// mantissa multiply plus an exponent add, which the block-scaled MMA does in
// hardware.
//
// Kernel structure (one CTA per 128 x 256 output tile, 6 warps):
//   warp 0      TMA producer: A/B code tiles (128-byte rows, 128B swizzle)
//               and the scale-factor atoms (bulk copies) into a 4-stage ring
//   warp 1      TMEM allocation and the single MMA-issuing thread: copies
//               the stage's scale factors to TMEM (tcgen05.cp) and issues
//               tcgen05.mma into a 128 x 256 fp32 (or s32) accumulator
//   warps 2-5   epilogue: tcgen05.ld of the accumulator, scaling, store
// The low-rank branch is one extra pipeline stage: a bf16 kind::f16 MMA of
// the packed activation [hi | lo] (m x 64) against the packed up-projection
// [L2^T | L2^T] (n x 64) into the same accumulator, the activation having
// been divided by the epilogue scale so that alpha * acc adds t . l2.
// Every mbarrier wait is bounded; a wait that runs out latches the device
// error word (read by mxq_check) and the CTA drains and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "mxq_formats.cuh"
#include "mxq_internal.h"

namespace mxq {

__device__ unsigned int g_error_word;

namespace {

constexpr int BM = 128, BN = 256, BKB = 128, STAGES = 4;
constexpr int A_STAGE = BM * BKB;                          // 16 KB
constexpr int B_STAGE = BN * BKB;                          // 32 KB
constexpr int SF_STAGE = 6144;                             // SFA 2 KB + SFB 2 x 2 KB
constexpr int STAGE_BYTES = A_STAGE + B_STAGE + SF_STAGE;  // 54 KB (multiple of 1 KB)
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 256 + 1024;   // ring + barriers + alignment slack
constexpr int kGemmThreads = 192;
constexpr uint32_t TMEM_COLS = 512;
// TMEM columns: accumulator stage 0 at [0, 256), stage 1 at [192, 448)
// (the stages share 64 columns), scale factors at [448, 512).
constexpr uint32_t ACC_STAGE1 = 192, OVL_COLS = 64;
constexpr uint32_t TMEM_SFA = 448, TMEM_SFB = 464;

enum Kind : int { kKindNVFP4 = 0, kKindMXFP4 = 1, kKindMXFP8 = 2, kKindFP8 = 3, kKindINT8 = 4 };

constexpr unsigned int kErrTimeoutProducer = 1u, kErrTimeoutMma = 2u, kErrTimeoutEpilogue = 4u;

struct GemmParams {
    CUtensorMap tma_a, tma_b, tma_t, tma_l2;
    const uint8_t *sfa, *sfb;
    const float *a_row_scale, *b_row_scale;
    const float *a_ts, *b_ts;
    void *y;
    int m, n, kbytes, num_k_tiles, s4, has_lowrank, y_bf16, m_tiles, n_tiles;
    unsigned long long wait_ns;
};

// ------------------------------------------------------------------ PTX

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Bounded wait for the phase of parity `parity` to complete.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, unsigned long long limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = global_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > limit_ns) return false;
    }
}

__device__ __forceinline__ void tma_load_2d(const CUtensorMap *map, void *dst, uint64_t *bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_cp_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: 8-row x 128 B
// core groups 1024 B apart (stride byte offset), descriptor version 1.
__device__ __forceinline__ uint64_t sdesc_sw128(const void *p) {
    uint64_t a = (smem_u32(p) >> 4) & 0x3FFFu;
    return a | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
// Descriptor of one 512-byte scale-factor atom for tcgen05.cp (no swizzle,
// 8 rows of 16 B per core matrix, core matrices 128 B apart).
__device__ __forceinline__ uint64_t sdesc_sf(const void *p) {
    uint64_t a = (smem_u32(p) >> 4) & 0x3FFFu;
    return a | (8ull << 32) | (1ull << 46);
}

template <int KIND>
__device__ __forceinline__ void mma_block_scaled(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc,
                                                 uint32_t sfa, uint32_t sfb) {
    if (KIND == kKindNVFP4)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
            ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb));
    else if (KIND == kKindMXFP4)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
            ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb));
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
            ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb));
}

template <int KIND>
__device__ __forceinline__ void mma_plain(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    if (KIND == kKindFP8)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
            ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc));
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
            ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_bf16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

// 32 lanes x 32 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Instruction descriptors (M = 128, N = 256, K-major A and B).
__host__ __device__ constexpr uint32_t idesc_common() { return ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24); }
template <int KIND>
__host__ __device__ constexpr uint32_t idesc_main() {
    return KIND == kKindNVFP4 ? idesc_common() | (1u << 7) | (1u << 10)                 // E2M1 x E2M1, UE4M3 scales
         : KIND == kKindMXFP4 ? idesc_common() | (1u << 7) | (1u << 10) | (1u << 23)   // E2M1 x E2M1, UE8M0 scales
         : KIND == kKindMXFP8 ? idesc_common() | (1u << 23)                           // E4M3 x E4M3, UE8M0 scales
         : KIND == kKindFP8   ? idesc_common() | (1u << 4)                            // E4M3 x E4M3 -> f32
                              : idesc_common() | (2u << 4) | (1u << 7) | (1u << 10);  // s8 x s8 -> s32
}
__host__ __device__ constexpr uint32_t idesc_bf16() { return idesc_common() | (1u << 4) | (1u << 7) | (1u << 10); }

// Scale-factor atoms (512 B) per stage for A (128 rows) and per 128-row half of B.
template <int KIND>
__host__ __device__ constexpr int sf_atoms() { return KIND == kKindNVFP4 ? 4 : KIND == kKindMXFP4 ? 2 : KIND == kKindMXFP8 ? 1 : 0; }

__device__ __forceinline__ void latch_error(unsigned int code) { atomicOr(&g_error_word, code); }

// ------------------------------------------------------------------ GEMM

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Epilogue value of accumulator column j of a chunk: alpha * acc (fp32
// accumulators) or acc * sa * sb[n] (s32 accumulators of INT8_ROW).
template <int KIND>
__device__ __forceinline__ void scale_chunk(const uint32_t (&r)[32], float (&v)[32], float alpha, float ra,
                                            const float *sbn, int nvalid) {
    if (KIND == kKindINT8) {
#pragma unroll
        for (int j = 0; j < 32; j++) {
            const float sb = j < nvalid ? __ldg(sbn + j) : 0.0f;
            v[j] = __fmul_rn(__fmul_rn((float)(int)r[j], ra), sb);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; j++) v[j] = __fmul_rn(__uint_as_float(r[j]), alpha);
    }
}

// Persistent GEMM: gridDim.x CTAs (one per SM) walk the output tiles
// blockIdx.x, blockIdx.x + gridDim.x, ...  The TMA ring runs continuously
// across tiles, so the next tile's operands stream in while the current
// tile finishes.  Tiles alternate between two TMEM accumulator stages that
// share 64 columns (512 columns hold two 256-column stages only that way,
// beside the scale factors); the epilogue drains the shared columns first,
// so the next tile's MMAs wait only for those, not for the whole epilogue.
template <int KIND>
__global__ void __launch_bounds__(kGemmThreads, 1) k_gemm(const __grid_constant__ GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
    uint64_t *empty = full + STAGES;
    uint64_t *accf = empty + STAGES;      // [2] accumulator stage full
    uint64_t *acce = accf + 2;            // [2] accumulator stage drained
    uint64_t *ovlf = acce + 2;            // shared 64 columns drained
    uint64_t *drain = ovlf + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int NSF = sf_atoms<KIND>();
    const int num_tiles = p.m_tiles * p.n_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; s++) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(accf + i, 1);
            mbar_init(acce + i, 4);   // one arrival per epilogue warp
        }
        mbar_init(ovlf, 4);
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int nsteps = p.num_k_tiles + p.has_lowrank;

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            int it = 0, issued = 0;
            for (int tile = blockIdx.x; tile < num_tiles && !*abort_flag; tile += gridDim.x) {
                const int m0 = (tile / p.n_tiles) * BM, n0 = (tile % p.n_tiles) * BN;
                const int rt_a = m0 >> 7, rt_b = n0 >> 7;
                const bool b_hi = (n0 + 128) < p.n;
                for (int kt = 0; kt < nsteps; kt++, it++) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(empty + s, ph ^ 1, p.wait_ns)) {
                        latch_error(kErrTimeoutProducer);
                        *abort_flag = 1;
                        break;
                    }
                    if (*abort_flag) break;
                    uint8_t *sa = smem + s * STAGE_BYTES;
                    uint8_t *sb = sa + A_STAGE;
                    uint8_t *sf = sb + B_STAGE;
                    if (kt < p.num_k_tiles) {
                        uint32_t bytes = A_STAGE + B_STAGE;
                        if (NSF) bytes += NSF * 512 * (b_hi ? 3 : 2);
                        mbar_arrive_expect_tx(full + s, bytes);
                        tma_load_2d(&p.tma_a, sa, full + s, kt * BKB, m0);
                        tma_load_2d(&p.tma_b, sb, full + s, kt * BKB, n0);
                        if (NSF) {
                            bulk_load(sf, p.sfa + ((int64_t)rt_a * p.s4 + kt * NSF) * 512, NSF * 512, full + s);
                            bulk_load(sf + 2048, p.sfb + ((int64_t)rt_b * p.s4 + kt * NSF) * 512, NSF * 512, full + s);
                            if (b_hi)
                                bulk_load(sf + 4096, p.sfb + ((int64_t)(rt_b + 1) * p.s4 + kt * NSF) * 512, NSF * 512,
                                          full + s);
                        }
                    } else {
                        mbar_arrive_expect_tx(full + s, A_STAGE + B_STAGE);
                        tma_load_2d(&p.tma_t, sa, full + s, 0, m0);
                        tma_load_2d(&p.tma_l2, sb, full + s, 0, n0);
                    }
                    issued = it + 1;
                }
            }
            if (*abort_flag) {
                // drain: wait (bounded) for the loads this thread may still have in flight
                for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; i++)
                    mbar_wait(full + (i % STAGES), (i / STAGES) & 1, p.wait_ns);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t sfa_addr = tmem + TMEM_SFA, sfb_addr = tmem + TMEM_SFB;
            bool issued_any = false;
            int it = 0, tcount = 0;
            for (int tile = blockIdx.x; tile < num_tiles && !*abort_flag; tile += gridDim.x, tcount++) {
                const int n0 = (tile % p.n_tiles) * BN;
                const bool b_hi = (n0 + 128) < p.n;
                const int st = tcount & 1;
                const uint32_t acc_addr = tmem + (st ? ACC_STAGE1 : 0u);
                // this stage drained by tile tcount-2, shared columns by tile tcount-1
                bool ok = mbar_wait(acce + st, ((tcount >> 1) & 1) ^ 1, p.wait_ns);
                if (ok && tcount > 0) ok = mbar_wait(ovlf, (tcount - 1) & 1, p.wait_ns);
                if (!ok) {
                    latch_error(kErrTimeoutMma);
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                for (int kt = 0; kt < nsteps; kt++, it++) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(full + s, ph, p.wait_ns)) {
                        latch_error(kErrTimeoutMma);
                        *abort_flag = 1;
                        break;
                    }
                    if (*abort_flag) break;
                    tc_fence_after();
                    uint8_t *sa = smem + s * STAGE_BYTES;
                    uint8_t *sb = sa + A_STAGE;
                    uint8_t *sf = sb + B_STAGE;
                    if (kt < p.num_k_tiles) {
                        const int rem = (p.kbytes - kt * BKB) >> 5;
                        const int nks = rem < 4 ? rem : 4;
                        if (NSF) {
#pragma unroll
                            for (int i = 0; i < NSF; i++) {
                                tc_cp_32x128b_warpx4(sfa_addr + 4 * i, sdesc_sf(sf + 512 * i));
                                tc_cp_32x128b_warpx4(sfb_addr + 8 * i, sdesc_sf(sf + 2048 + 512 * i));
                                if (b_hi) tc_cp_32x128b_warpx4(sfb_addr + 8 * i + 4, sdesc_sf(sf + 4096 + 512 * i));
                            }
                        }
                        for (int ks = 0; ks < nks; ks++) {
                            const uint64_t ad = sdesc_sw128(sa + ks * 32), bd = sdesc_sw128(sb + ks * 32);
                            const uint32_t accum = (kt > 0 || ks > 0) ? 1u : 0u;
                            if (KIND == kKindNVFP4) {
                                mma_block_scaled<KIND>(acc_addr, ad, bd, idesc_main<KIND>(), accum, sfa_addr + 4 * ks,
                                                       sfb_addr + 8 * ks);
                            } else if (KIND == kKindMXFP4) {
                                const uint32_t id = (uint32_t)((ks & 1) * 2);
                                mma_block_scaled<KIND>(acc_addr, ad, bd, idesc_main<KIND>() | (id << 29) | (id << 4),
                                                       accum, sfa_addr + 4 * (ks >> 1), sfb_addr + 8 * (ks >> 1));
                            } else if (KIND == kKindMXFP8) {
                                const uint32_t id = (uint32_t)ks;
                                mma_block_scaled<KIND>(acc_addr, ad, bd, idesc_main<KIND>() | (id << 29) | (id << 4),
                                                       accum, sfa_addr, sfb_addr);
                            } else {
                                mma_plain<KIND>(acc_addr, ad, bd, idesc_main<KIND>(), accum);
                            }
                        }
                    } else {
#pragma unroll
                        for (int ks = 0; ks < 4; ks++)
                            mma_bf16(acc_addr, sdesc_sw128(sa + ks * 32), sdesc_sw128(sb + ks * 32), idesc_bf16(), 1u);
                    }
                    issued_any = true;
                    tc_commit(empty + s);
                }
                if (*abort_flag) break;
                tc_commit(accf + st);
            }
            if (*abort_flag && issued_any) {
                tc_commit(drain);
                mbar_wait(drain, 0, p.wait_ns);
            }
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;   // TMEM lane quarter this warp may access
        const bool vec = p.y_bf16 ? (p.n % 8 == 0) : (p.n % 4 == 0);
        int tcount = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, tcount++) {
            const int m0 = (tile / p.n_tiles) * BM, n0 = (tile % p.n_tiles) * BN;
            const int row = m0 + q * 32 + lane;
            const int st = tcount & 1;
            bool ok = !*abort_flag && mbar_wait(accf + st, (tcount >> 1) & 1, p.wait_ns);
            ok = __all_sync(0xFFFFFFFFu, ok);
            if (!ok) {
                if (lane == 0 && !*abort_flag) latch_error(kErrTimeoutEpilogue);
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16) + (st ? ACC_STAGE1 : 0u);
            float alpha = 1.0f, ra = 0.0f;
            if (KIND == kKindNVFP4 || KIND == kKindFP8) alpha = __fmul_rn(__ldg(p.a_ts), __ldg(p.b_ts));
            const bool row_ok = row < p.m;
            if (KIND == kKindINT8 && row_ok) ra = __ldg(p.a_row_scale + row);
            // the 64 shared columns first: the last two chunks of stage 0, the first two of stage 1
#pragma unroll 1
            for (int i = 0; i < BN / 32; i++) {
                const int c = st ? i : (i + 6) & 7;
                uint32_t r[32];
                tmem_ld_32x32b_x32(lane_base + (uint32_t)(c * 32), r);
                if (i == 1 || i == 7) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(i == 1 ? ovlf : acce + st);
                }
                const int nb = n0 + c * 32;
                if (!row_ok || nb >= p.n) continue;
                float v[32];
                scale_chunk<KIND>(r, v, alpha, ra, p.b_row_scale + nb, p.n - nb);
                if (p.y_bf16) {
                    __nv_bfloat16 *yrow = reinterpret_cast<__nv_bfloat16 *>(p.y) + (int64_t)row * p.n;
                    if (vec && nb + 32 <= p.n) {
                        uint4 *dst = reinterpret_cast<uint4 *>(yrow + nb);
#pragma unroll
                        for (int k4 = 0; k4 < 4; k4++)
                            dst[k4] = make_uint4(pack_bf16x2(v[8 * k4], v[8 * k4 + 1]), pack_bf16x2(v[8 * k4 + 2], v[8 * k4 + 3]),
                                                 pack_bf16x2(v[8 * k4 + 4], v[8 * k4 + 5]),
                                                 pack_bf16x2(v[8 * k4 + 6], v[8 * k4 + 7]));
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; j++)
                            if (nb + j < p.n) yrow[nb + j] = __float2bfloat16_rn(v[j]);
                    }
                } else {
                    float *yrow = reinterpret_cast<float *>(p.y) + (int64_t)row * p.n;
                    if (vec && nb + 32 <= p.n) {
                        float4 *dst = reinterpret_cast<float4 *>(yrow + nb);
#pragma unroll
                        for (int k4 = 0; k4 < 8; k4++)
                            dst[k4] = make_float4(v[4 * k4], v[4 * k4 + 1], v[4 * k4 + 2], v[4 * k4 + 3]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; j++)
                            if (nb + j < p.n) yrow[nb + j] = v[j];
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
    }
}

// ------------------------------------------------------------------ low rank

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
//   kLrTAmax  t, and max |x| over the whole tensor into *amax_word
template <typename T, int MODE>
__global__ void __launch_bounds__(kLrWarps * 32) k_lowrank(const T *__restrict__ x, int64_t m, int64_t k,
                                                         const __nv_bfloat16 *__restrict__ l1, int r,
                                                         float *__restrict__ t, const float *xs, const float *ws,
                                                         __nv_bfloat16 *__restrict__ tp, unsigned int *amax_word) {
    __shared__ float red[kLrWarps][16][33];
    __shared__ float wmax[kLrWarps];
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
        if (v > 0.0f) atomicMax(amax_word, __float_as_uint(v));
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

// ------------------------------------------------------------------ host

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

bool encode_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
    auto fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int KIND>
cudaError_t launch_kind(const GemmParams &p, dim3 grid, cudaStream_t s) {
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(k_gemm<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    k_gemm<KIND><<<grid, kGemmThreads, SMEM_BYTES, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

template <typename T>
static void launch_lr(int mode, int grid, const T *x, int64_t m, int64_t k, const __nv_bfloat16 *l1, int r, float *t,
                      const float *xs, const float *ws, __nv_bfloat16 *tp, unsigned int *amax, cudaStream_t s) {
    const int threads = kLrWarps * 32;
    if (mode == kLrT) k_lowrank<T, kLrT><<<grid, threads, 0, s>>>(x, m, k, l1, r, t, xs, ws, tp, amax);
    else if (mode == kLrPacked) k_lowrank<T, kLrPacked><<<grid, threads, 0, s>>>(x, m, k, l1, r, t, xs, ws, tp, amax);
    else k_lowrank<T, kLrTAmax><<<grid, threads, 0, s>>>(x, m, k, l1, r, t, xs, ws, tp, amax);
}

cudaError_t launch_lowrank_down(const void *x, bool bf16, int64_t m, int64_t k, const void *l1, int r, float *t,
                                const float *xs, const float *ws, void *tp, cudaStream_t s, unsigned int *amax_word) {
    if (m == 0) return cudaSuccess;
    const int grid = (int)((m + 15) / 16);
    const int mode = tp ? kLrPacked : (amax_word ? kLrTAmax : kLrT);
    const __nv_bfloat16 *l = (const __nv_bfloat16 *)l1;
    __nv_bfloat16 *tpb = (__nv_bfloat16 *)tp;
    if (bf16) launch_lr(mode, grid, (const __nv_bfloat16 *)x, m, k, l, r, t, xs, ws, tpb, amax_word, s);
    else launch_lr(mode, grid, (const float *)x, m, k, l, r, t, xs, ws, tpb, amax_word, s);
    return cudaGetLastError();
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

cudaError_t launch_qlinear(const GemmOperands &op, cudaStream_t s) {
    if (op.m == 0 || op.n == 0) return cudaSuccess;
    GemmParams p;
    memset(&p, 0, sizeof(p));
    const bool is4 = op.fmt == kMXFP4 || op.fmt == kNVFP4;
    const int64_t kbytes = is4 ? op.k / 2 : op.k;
    if (!encode_2d(&p.tma_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, op.a_codes, kbytes, op.m, kbytes, BKB, BM) ||
        !encode_2d(&p.tma_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, op.b_codes, kbytes, op.n, kbytes, BKB, BN))
        return cudaErrorInvalidValue;
    if (op.tp) {
        if (!encode_2d(&p.tma_t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, op.tp, 64, op.m, 128, 64, BM) ||
            !encode_2d(&p.tma_l2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, op.l2p, 64, op.n, 128, 64, BN))
            return cudaErrorInvalidValue;
    }
    p.sfa = (const uint8_t *)op.a_scales;
    p.sfb = (const uint8_t *)op.b_scales;
    p.a_row_scale = (const float *)op.a_scales;
    p.b_row_scale = (const float *)op.b_scales;
    p.a_ts = op.a_tensor_scale;
    p.b_ts = op.b_tensor_scale;
    p.y = op.y;
    p.m = (int)op.m;
    p.n = (int)op.n;
    p.kbytes = (int)kbytes;
    p.num_k_tiles = (int)((kbytes + BKB - 1) / BKB);
    const int blk = fmt_block(op.fmt);
    p.s4 = blk ? (int)(((op.k / blk) + 15) / 16 * 16 / 4) : 0;
    p.has_lowrank = op.tp != nullptr;
    p.y_bf16 = op.y_bf16;
    p.wait_ns = 2000000000ull;   // 2 s
    p.m_tiles = (int)((op.m + BM - 1) / BM);
    p.n_tiles = (int)((op.n + BN - 1) / BN);
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    const int tiles = p.m_tiles * p.n_tiles;
    dim3 grid((unsigned)(tiles < sms ? tiles : sms));
    switch (op.fmt) {
    case kNVFP4: return launch_kind<kKindNVFP4>(p, grid, s);
    case kMXFP4: return launch_kind<kKindMXFP4>(p, grid, s);
    case kMXFP8: return launch_kind<kKindMXFP8>(p, grid, s);
    case kFP8Tensor: return launch_kind<kKindFP8>(p, grid, s);
    case kINT8Row: return launch_kind<kKindINT8>(p, grid, s);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t read_and_clear_error(unsigned int *value) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(value, g_error_word, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbol(g_error_word, &zero, sizeof(unsigned int));
}

}  // namespace mxq
