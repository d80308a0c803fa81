// gemm.cu -- block-scaled low-bit GEMM on 5th-generation tensor cores
// (tcgen05, CTA pairs) with the dequantization epilogue and the SVDQuant
// low-rank branch fused.
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
// Structure.  Clusters of two CTAs (one per SM) compute 256 x 256 output
// tiles with cta_group::2 MMAs: each CTA stages its own 128 rows of A, its
// 128-row half of B, the scale factors of its A rows and of all 256 B rows,
// and holds its 128 x 256 part of the accumulator in its own TMEM.  Per CTA:
//   warp 0      TMA producer into a 5-stage ring (128-byte rows, 128B
//               swizzle); the second CTA's loads complete on the first
//               CTA's barriers (TMA .cta_group::2, no multicast)
//   warp 1      TMEM allocation; in the first CTA also the single thread
//               that issues the MMAs, committing to both CTAs' barriers
//   warps 2-5   epilogue: TMEM -> registers -> scaling -> swizzled shared
//               staging -> TMA bulk stores
//   warps 6-    in the first CTA, kSfWarps threads that copy each stage's scale
//               factors to TMEM (tcgen05.cp) and signal
//               the MMA thread
// The kernel is persistent: clusters walk the tiles, the TMA ring runs on
// across tiles, and tiles alternate between two TMEM accumulator stages
// that share 96 columns (two 256-column stages fit beside the scale-factor
// ring only that way); the epilogue drains the shared columns first, so the
// next tile's MMAs wait only for those.
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
#include "tc_ptx.cuh"

namespace mxq {

__device__ unsigned int g_error_word;

namespace {

constexpr int BM = 128;                 // accumulator rows per CTA (a pair covers 256)
constexpr int BN = 256;                 // output columns per tile
constexpr int BNH = 128;                // B rows staged per CTA
constexpr int BKB = 128;                // bytes of K per stage row
constexpr int STAGES = 5;
constexpr int A_STAGE = BM * BKB;       // 16 KB
constexpr int B_STAGE = BNH * BKB;      // 16 KB
constexpr int SF_STAGE = 6144;          // SFA (<= 4 atoms) at 0, SFB halves at 2048 and 4096
constexpr int STAGE_BYTES = A_STAGE + B_STAGE + SF_STAGE;   // 38 KB, a multiple of 1 KB
constexpr int EPI_BUF = 4096;           // one 32-row x 128-byte staging buffer
constexpr int EPI_BYTES = 4 * 2 * EPI_BUF;                  // 4 warps x 2 buffers
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 1024;
// Warps that copy scale factors to TMEM (warps 6 .. 6 + kSfWarps - 1), one
// k-step's atoms (SFA and the one or two SFB atoms) per warp in turn: a
// tcgen05.cp stalls the thread that issues it, so a stage's copies are
// spread over several threads (NVFP4, workload 3: 2 warps 95.8 us, 4 warps
// 93.7 us; dealing single copies round-robin instead was slower).
constexpr int kSfWarps = 4;
constexpr int kGemmThreads = 32 * (6 + kSfWarps);
constexpr uint32_t TMEM_COLS = 512;
// TMEM columns: accumulator stage 0 at [0, 256), stage 1 at
// [ACC_STAGE1, ACC_STAGE1 + 256) (the two stages share 256 - ACC_STAGE1
// columns), then SF_GROUPS groups of four 12-column scale-factor slots (SFA 4
// columns, the two SFB halves 4 + 4 per atom) up to column 512.  K-tile i uses
// group i % SF_GROUPS, so the scale factors of k-tile i are copied once the
// MMAs of k-tile i - SF_GROUPS have completed: more groups let the copies run
// further ahead of the MMAs, at the price of more shared accumulator columns
// (which the epilogue drains first, before the next tile's MMAs may start).
#ifndef MXQ_SF_GROUPS
#define MXQ_SF_GROUPS 2
#endif

constexpr uint32_t SF_GROUPS = MXQ_SF_GROUPS;
constexpr uint32_t SF_SLOT_COLS = 12, SF_GROUP_COLS = 48;
constexpr uint32_t TMEM_SF = TMEM_COLS - SF_GROUPS * SF_GROUP_COLS;
constexpr uint32_t ACC_STAGE1 = (TMEM_SF - 256) & ~31u;    // 32-column aligned
constexpr uint32_t OVL_CHUNKS = (256 - ACC_STAGE1) / 32;   // shared 32-column chunks
static_assert(ACC_STAGE1 + 256 <= TMEM_SF && OVL_CHUNKS >= 1 && OVL_CHUNKS <= 8, "TMEM budget");

// kKindBF16: bf16 x bf16 operands on kind::f16 (no block scales), the
// epilogue scale the B operand's tensor scale when it has one.
enum Kind : int { kKindNVFP4 = 0, kKindMXFP4 = 1, kKindMXFP8 = 2, kKindFP8 = 3, kKindINT8 = 4, kKindBF16 = 5 };

constexpr unsigned int kErrTimeoutProducer = 1u, kErrTimeoutMma = 2u, kErrTimeoutEpilogue = 4u;

struct GemmParams {
    CUtensorMap tma_a, tma_b, tma_sfa, tma_sfb, tma_t, tma_l2, tma_y;
    const float *a_row_scale, *b_row_scale;
    const float *a_ts, *b_ts;
    void *y;
    int m, n, kbytes, num_k_tiles, s4, has_lowrank, y_bf16, y_tma;
    int m_tiles, n_tiles;         // 256 x 256 tiles
    int sfa_tiles;                // 128-row scale tiles of A (rows padded to 128)
    unsigned long long wait_ns;
};

// ------------------------------------------------------------------ PTX



// 2-D tiled TMA load into this CTA's shared memory, completing on the
// barrier at cluster address `bar` (either CTA of the pair).
__device__ __forceinline__ void tma_load_pair(const CUtensorMap *map, void *dst, uint32_t bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

// Arrive on the barrier at this offset in both CTAs once the issued MMAs complete.
__device__ __forceinline__ void tc_commit_pair(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"((uint16_t)3)
        : "memory");
}
// Arrive on this CTA's barrier once this thread's issued tcgen05 operations complete.
__device__ __forceinline__ void tc_commit_self(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_cp_pair(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
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
            "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
            ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb));
    else if (KIND == kKindMXFP4)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
            ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb));
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
            ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb));
}

template <int KIND>
__device__ __forceinline__ void mma_plain(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    if (KIND == kKindFP8)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
            ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc));
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}"
            ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_bf16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

// Instruction descriptors (M = 256 over the pair, N = 256, K-major A and B).
__host__ __device__ constexpr uint32_t idesc_common() { return ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(256 >> 4) << 24); }
template <int KIND>
__host__ __device__ constexpr uint32_t idesc_main() {
    return KIND == kKindNVFP4 ? idesc_common() | (1u << 7) | (1u << 10)                 // E2M1 x E2M1, UE4M3 scales
         : KIND == kKindMXFP4 ? idesc_common() | (1u << 7) | (1u << 10) | (1u << 23)   // E2M1 x E2M1, UE8M0 scales
         : KIND == kKindMXFP8 ? idesc_common() | (1u << 23)                           // E4M3 x E4M3, UE8M0 scales
         : KIND == kKindFP8   ? idesc_common() | (1u << 4)                            // E4M3 x E4M3 -> f32
                              : idesc_common() | (2u << 4) | (1u << 7) | (1u << 10);  // s8 x s8 -> s32
}
__host__ __device__ constexpr uint32_t idesc_bf16() { return idesc_common() | (1u << 4) | (1u << 7) | (1u << 10); }

// Scale-factor atoms (512 B) per stage for 128 rows.
template <int KIND>
__host__ __device__ constexpr int sf_atoms() { return KIND == kKindNVFP4 ? 4 : KIND == kKindMXFP4 ? 2 : KIND == kKindMXFP8 ? 1 : 0; }
// Accumulator stage 1 and the columns it shares with stage 0: the kinds
// without block scales leave the scale-factor slots empty, so their two
// stages are disjoint ([0, 256) and [256, 512)) and a tile's MMAs wait only
// for the drain of the tile two before.
template <int KIND>
__host__ __device__ constexpr uint32_t acc_stage1() { return sf_atoms<KIND>() ? ACC_STAGE1 : 256u; }
template <int KIND>
__host__ __device__ constexpr int ovl_chunks() { return sf_atoms<KIND>() ? (int)OVL_CHUNKS : 0; }

__device__ __forceinline__ void latch_error(unsigned int code) { atomicOr(&g_error_word, code); }

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

// One k-step (32 bytes of K) of the main product: an NVFP4 scale atom serves
// one k-step, an MXFP4 atom two, an MXFP8 atom four (the MX kinds select the
// atom's scale column through the instruction descriptor).
template <int KIND>
__device__ __forceinline__ void mma_kstep(uint32_t acc_addr, uint64_t ad, uint64_t bd, uint32_t accum, uint32_t group,
                                          int ks) {
    constexpr int NSF = sf_atoms<KIND>();
    const int a = NSF == 4 ? ks : NSF == 2 ? (ks >> 1) : 0;
    const uint32_t base = group + SF_SLOT_COLS * (uint32_t)a;
    if (KIND == kKindNVFP4) {
        mma_block_scaled<KIND>(acc_addr, ad, bd, idesc_main<KIND>(), accum, base, base + 4);
    } else if (KIND == kKindMXFP4) {
        const uint32_t id = (uint32_t)((ks & 1) * 2);
        mma_block_scaled<KIND>(acc_addr, ad, bd, idesc_main<KIND>() | (id << 29) | (id << 4), accum, base, base + 4);
    } else if (KIND == kKindMXFP8) {
        const uint32_t id = (uint32_t)ks;
        mma_block_scaled<KIND>(acc_addr, ad, bd, idesc_main<KIND>() | (id << 29) | (id << 4), accum, base, base + 4);
    } else if (KIND == kKindBF16) {
        mma_bf16(acc_addr, ad, bd, idesc_bf16(), accum);
    } else {
        mma_plain<KIND>(acc_addr, ad, bd, idesc_main<KIND>(), accum);
    }
}

template <int KIND>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    k_gemm(const __grid_constant__ GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *epi = smem + STAGES * STAGE_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(epi + EPI_BYTES);   // [STAGES] (used in the first CTA)
    uint64_t *empty = full + STAGES;                                   // [STAGES]
    uint64_t *accf = empty + STAGES;                                   // [2] accumulator stage full
    uint64_t *acce = accf + 2;                                         // [2] stage drained (first CTA)
    uint64_t *ovlf = acce + 2;                                         // shared columns drained (first CTA)
    uint64_t *drain = ovlf + 1;
    uint64_t *sfready = drain + 1;                                     // [STAGES] scale factors in TMEM (first CTA)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sfready + STAGES);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int cid = (int)cluster_id(), ncl = (int)cluster_count();
    constexpr int NSF = sf_atoms<KIND>();
    const int num_tiles = p.m_tiles * p.n_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; s++) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(accf + i, 1);
            mbar_init(acce + i, 8);   // 4 epilogue warps x 2 CTAs
        }
        mbar_init(ovlf, 8);
        mbar_init(drain, 1);
        for (int i = 0; i < STAGES; i++) mbar_init(sfready + i, kSfWarps);   // one arrival per scale-factor warp
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int nsteps = p.num_k_tiles + p.has_lowrank;
    // the setup above overlaps the previous kernel (the quantizer); operands
    // are read and Y written only after it has completed
    pdl_wait();
    pdl_launch_dependents();

    if (warp == 0) {
        // ---------------------------------------------------------- producer (both CTAs)
        if (lane == 0) {
            int it = 0, issued = 0;
            for (int tile = cid; tile < num_tiles && !*abort_flag; tile += ncl) {
                const int pm0 = (tile / p.n_tiles) * 256, n0 = (tile % p.n_tiles) * BN;
                const int m0 = pm0 + (int)rank * BM, nb0 = n0 + (int)rank * BNH;
                const int rt_a = (pm0 >> 7) + (int)rank;
                const bool sfa_mine = rt_a < p.sfa_tiles;
                const bool sfa_peer = (pm0 >> 7) + 1 < p.sfa_tiles;
                const bool b_hi = (n0 + 128) < p.n;
                const int rt_b = n0 >> 7;
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
                    const uint32_t bar = map_to_rank(full + s, 0);
                    if (kt < p.num_k_tiles) {
                        if (rank == 0) {
                            uint32_t bytes = 2 * (A_STAGE + B_STAGE);
                            if (NSF) bytes += NSF * 512 * (1 + (sfa_peer ? 1 : 0) + 2 * (b_hi ? 2 : 1));
                            mbar_arrive_expect_tx(full + s, bytes);
                        }
                        tma_load_pair(&p.tma_a, sa, bar, kt * BKB, m0);
                        tma_load_pair(&p.tma_b, sb, bar, kt * BKB, nb0);
                        if (NSF) {
                            if (sfa_mine) tma_load_pair(&p.tma_sfa, sf, bar, 0, rt_a * p.s4 + kt * NSF);
                            tma_load_pair(&p.tma_sfb, sf + 2048, bar, 0, rt_b * p.s4 + kt * NSF);
                            if (b_hi) tma_load_pair(&p.tma_sfb, sf + 4096, bar, 0, (rt_b + 1) * p.s4 + kt * NSF);
                        }
                    } else {
                        if (rank == 0) mbar_arrive_expect_tx(full + s, 2 * (A_STAGE + B_STAGE));
                        tma_load_pair(&p.tma_t, sa, bar, 0, m0);
                        tma_load_pair(&p.tma_l2, sb, bar, 0, nb0);
                    }
                    issued = it + 1;
                }
            }
            if (*abort_flag && rank == 0) {
                // drain: wait (bounded) for the loads that may still be in flight
                for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; i++)
                    mbar_wait(full + (i % STAGES), (i / STAGES) & 1, p.wait_ns);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer (first CTA)
        // This one thread's latency per k-tile (barrier wait, set-up, four MMA
        // issues, commit) is what keeps the tensor pipe fed, so the loop is
        // lean: stage and phase are counters, a stage's descriptors are the
        // stage-0 descriptors plus constants, and a whole k-tile's four
        // k-steps are unrolled.
        if (lane == 0 && rank == 0) {
            bool issued_any = false;
            int it = 0, tcount = 0, s = 0;
            uint32_t ph = 0;
            const uint64_t ad0 = sdesc_sw128(smem), bd0 = sdesc_sw128(smem + A_STAGE);
            const int nk_full = p.kbytes / BKB;   // k-tiles with all four k-steps
            for (int tile = cid; tile < num_tiles && !*abort_flag; tile += ncl, tcount++) {
                const int st = tcount & 1;
                const uint32_t acc_addr = tmem + (st ? acc_stage1<KIND>() : 0u);
                // this stage drained (tile tcount-2) and the shared columns (tile tcount-1), in both CTAs
                bool ok = mbar_wait_spin<true>(acce + st, ((tcount >> 1) & 1) ^ 1, p.wait_ns);
                if (ovl_chunks<KIND>() > 0 && ok && tcount > 0)
                    ok = mbar_wait_spin<true>(ovlf, (tcount - 1) & 1, p.wait_ns);
                if (!ok) {
                    latch_error(kErrTimeoutMma);
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                for (int kt = 0; kt < nsteps; kt++, it++) {
                    // block-scaled kinds: the scale-factor warp has copied this stage's atoms to TMEM
                    // (and seen the stage full); other kinds wait for the stage itself
                    if (!mbar_wait_spin(NSF ? sfready + s : full + s, ph, p.wait_ns)) {
                        latch_error(kErrTimeoutMma);
                        *abort_flag = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t soff = (uint64_t)(s * (STAGE_BYTES >> 4));
                    const uint64_t ad = ad0 + soff, bd = bd0 + soff;   // +2 per 32-byte k-step
                    const uint32_t group = tmem + TMEM_SF + SF_GROUP_COLS * ((uint32_t)it % SF_GROUPS);
                    if (kt < nk_full) {
#pragma unroll
                        for (int ks = 0; ks < 4; ks++)
                            mma_kstep<KIND>(acc_addr, ad + 2 * ks, bd + 2 * ks, (kt | ks) != 0 ? 1u : 0u, group, ks);
                    } else if (kt < p.num_k_tiles) {
                        const int nks = (p.kbytes - kt * BKB) >> 5;   // 1..3 k-steps in the last k-tile
                        for (int ks = 0; ks < nks; ks++)
                            mma_kstep<KIND>(acc_addr, ad + 2 * ks, bd + 2 * ks, (kt | ks) != 0 ? 1u : 0u, group, ks);
                    } else {
#pragma unroll
                        for (int ks = 0; ks < 4; ks++) mma_bf16(acc_addr, ad + 2 * ks, bd + 2 * ks, idesc_bf16(), 1u);
                    }
                    issued_any = true;
                    tc_commit_pair(empty + s);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (*abort_flag) break;
                tc_commit_pair(accf + st);
            }
            if (*abort_flag && issued_any) {
                tc_commit_pair(drain);
                mbar_wait(drain, 0, p.wait_ns);
            }
        }
    } else if (warp >= 6) {
        // ---------------------------------------------------------- scale-factor copies (first CTA)
        // Issued apart from the MMA thread: a tcgen05.cp stalls the thread that
        // issues it, but runs alongside the MMAs in the tensor pipe.  The atoms
        // of a stage are dealt to the kSfWarps warps in turn.
        const int par = warp - 6;
        if (NSF && lane == 0 && rank == 0) {
            int it = 0;
            bool ok = true;
            for (int tile = cid; tile < num_tiles && ok && !*abort_flag; tile += ncl) {
                const int n0 = (tile % p.n_tiles) * BN;
                const bool b_hi = (n0 + 128) < p.n;
                for (int kt = 0; kt < nsteps; kt++, it++) {
                    const int s = it % STAGES;
                    ok = mbar_wait(full + s, (it / STAGES) & 1, p.wait_ns);
                    // slot group it % SF_GROUPS was last read by the MMAs of k-tile it - SF_GROUPS
                    const int prev = it - (int)SF_GROUPS;
                    if (ok && prev >= 0) ok = mbar_wait(empty + (prev % STAGES), (prev / STAGES) & 1, p.wait_ns);
                    if (!ok || *abort_flag) {
                        if (!ok) latch_error(kErrTimeoutMma);
                        *abort_flag = 1;
                        break;
                    }
                    if (kt < p.num_k_tiles) {
                        const int rem = (p.kbytes - kt * BKB) >> 5;
                        const int nks = rem < 4 ? rem : 4;
                        const int natoms = NSF == 4 ? nks : NSF == 2 ? (nks + 1) >> 1 : 1;
                        const uint8_t *sf = smem + s * STAGE_BYTES + A_STAGE + B_STAGE;
                        const uint32_t group = tmem + TMEM_SF + SF_GROUP_COLS * ((uint32_t)it % SF_GROUPS);
                        tc_fence_after();
                        for (int a = par; a < natoms; a += kSfWarps) {
                            const uint32_t base = group + SF_SLOT_COLS * (uint32_t)a;
                            tc_cp_pair(base, sdesc_sf(sf + 512 * a));
                            tc_cp_pair(base + 4, sdesc_sf(sf + 2048 + 512 * a));
                            if (b_hi) tc_cp_pair(base + 8, sdesc_sf(sf + 4096 + 512 * a));
                        }
                        tc_commit_self(sfready + s);
                    } else {
                        mbar_arrive_local(sfready + s);
                    }
                }
            }
            if (*abort_flag) {
                tc_commit_self(drain);
                mbar_wait(drain, 0, p.wait_ns);
            }
        }
    } else {
        // ---------------------------------------------------------- epilogue (both CTAs)
        const int q = warp & 3;   // TMEM lane quarter this warp may access
        const uint32_t ovl_leader = map_to_rank(ovlf, 0);
        const uint32_t acce_leader0 = map_to_rank(acce, 0), acce_leader1 = map_to_rank(acce + 1, 0);
        uint8_t *stage_buf = epi + q * 2 * EPI_BUF;
        const bool vec = p.y_bf16 ? (p.n % 8 == 0) : (p.n % 4 == 0);
        // the tensor scales hold for the whole launch: read once, outside the tile loop
        float alpha = 1.0f;
        if (KIND == kKindNVFP4 || KIND == kKindFP8) alpha = __fmul_rn(__ldg(p.a_ts), __ldg(p.b_ts));
        if (KIND == kKindBF16 && p.b_ts) alpha = __ldg(p.b_ts);
        int tcount = 0, sub = 0;
        for (int tile = cid; tile < num_tiles; tile += ncl, tcount++) {
            const int pm0 = (tile / p.n_tiles) * 256, n0 = (tile % p.n_tiles) * BN;
            const int row0 = pm0 + (int)rank * BM + q * 32;
            const int row = row0 + lane;
            const int st = tcount & 1;
            bool ok = !*abort_flag && mbar_wait(accf + st, (tcount >> 1) & 1, p.wait_ns);
            ok = __all_sync(0xFFFFFFFFu, ok);
            if (!ok) {
                if (lane == 0 && !*abort_flag) latch_error(kErrTimeoutEpilogue);
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16) + (st ? acc_stage1<KIND>() : 0u);
            constexpr int OVL = ovl_chunks<KIND>();
            static_assert(KIND != kKindINT8 || OVL == 0, "the INT8 row scale is read before any chunk");
            float ra = 0.0f;   // INT8 row scale
            const bool row_ok = row < p.m;
            // The shared columns (the last OVL_CHUNKS chunks of stage 0, the first OVL_CHUNKS of
            // stage 1) go to registers first and are released at once, so the next tile's MMAs
            // wait only for these loads; then every chunk is scaled, staged and stored.
            auto process = [&](const int c, const uint32_t (&r)[32]) {
                    const int nb = n0 + c * 32;
                    float v[32];
                    scale_chunk<KIND>(r, v, alpha, ra, p.b_row_scale + nb, p.n - nb);
                    if (p.y_tma) {
                        // swizzled staging of this 32-column chunk, then one TMA store of 32 rows:
                        // bf16 rows of 64 B (64B swizzle: 16-byte unit j of row t at t*64 + (j ^ ((t >> 1) & 3))*16),
                        // fp32 rows of 128 B (128B swizzle: unit j at t*128 + (j ^ (t & 7))*16)
                        uint8_t *buf = stage_buf + (sub & 1) * EPI_BUF;
                        if (lane == 0) bulk_wait_read1();
                        __syncwarp();
                        if (p.y_bf16) {
                            uint4 *rowp = reinterpret_cast<uint4 *>(buf + lane * 64);
#pragma unroll
                            for (int k4 = 0; k4 < 4; k4++)
                                rowp[k4 ^ ((lane >> 1) & 3)] =
                                    make_uint4(pack_bf16x2(v[8 * k4], v[8 * k4 + 1]), pack_bf16x2(v[8 * k4 + 2], v[8 * k4 + 3]),
                                               pack_bf16x2(v[8 * k4 + 4], v[8 * k4 + 5]),
                                               pack_bf16x2(v[8 * k4 + 6], v[8 * k4 + 7]));
                        } else {
                            uint4 *rowp = reinterpret_cast<uint4 *>(buf + lane * 128);
#pragma unroll
                            for (int k4 = 0; k4 < 8; k4++)
                                rowp[k4 ^ (lane & 7)] = make_uint4(__float_as_uint(v[4 * k4]), __float_as_uint(v[4 * k4 + 1]),
                                                                   __float_as_uint(v[4 * k4 + 2]), __float_as_uint(v[4 * k4 + 3]));
                        }
                        fence_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&p.tma_y, buf, nb, row0);
                            bulk_commit();
                        }
                        sub++;
                    } else if (row_ok && nb < p.n) {
                        if (p.y_bf16) {
                            __nv_bfloat16 *yrow = reinterpret_cast<__nv_bfloat16 *>(p.y) + (int64_t)row * p.n;
                            if (vec && nb + 32 <= p.n) {
                                uint4 *dst = reinterpret_cast<uint4 *>(yrow + nb);
#pragma unroll
                                for (int k4 = 0; k4 < 4; k4++)
                                    dst[k4] = make_uint4(pack_bf16x2(v[8 * k4], v[8 * k4 + 1]),
                                                         pack_bf16x2(v[8 * k4 + 2], v[8 * k4 + 3]),
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
            };
            if constexpr (OVL > 0) {
                uint32_t ro[OVL][32];
#pragma unroll
                for (int i = 0; i < OVL; i++)
                    tmem_ld_32x32b_x32_async(lane_base + (uint32_t)((st ? i : 8 - OVL + i) * 32), ro[i]);
                tmem_ld_wait(ro[OVL - 1]);
#pragma unroll
                for (int i = 0; i + 1 < OVL; i++) tmem_reg_tie(ro[i]);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote_relaxed(ovl_leader);
#pragma unroll
                for (int i = 0; i < OVL; i++) process(st ? i : 8 - OVL + i, ro[i]);
            }
            if (KIND == kKindINT8 && row_ok) ra = __ldg(p.a_row_scale + row);   // INT8 has no shared columns
#pragma unroll 1
            for (int i = OVL; i < BN / 32; i++) {
                const int c = st ? i : i - OVL;
                uint32_t r[32];
                tmem_ld_32x32b_x32(lane_base + (uint32_t)(c * 32), r);
                if (i == BN / 32 - 1) {   // the whole stage is drained
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_remote_relaxed(st ? acce_leader1 : acce_leader0);
                }
                process(c, r);
            }
        }
        if (lane == 0) bulk_wait_all();
    }

    tc_fence_before();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
    }
}

// ------------------------------------------------------------------ host

}  // namespace

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
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
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
    auto fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {

template <int KIND>
cudaError_t launch_kind(const GemmParams &p, int grid, cudaStream_t s) {
    static PerDeviceOnce smem_opt_in;
    cudaError_t e = smem_opt_in.run(
        [] { return cudaFuncSetAttribute(k_gemm<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES); });
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);   // clusters of 2 from __cluster_dims__
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1] = {pdl_attribute()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_gemm<KIND>, p);
}

}  // namespace

static cudaError_t launch_gemm_common(const GemmOperands &op, bool bf16_operands, cudaStream_t s) {
    if (op.m == 0 || op.n == 0) return cudaSuccess;
    GemmParams p;
    memset(&p, 0, sizeof(p));
    const bool is4 = !bf16_operands && (op.fmt == kMXFP4 || op.fmt == kNVFP4);
    const int64_t kbytes = bf16_operands ? op.k * 2 : is4 ? op.k / 2 : op.k;
    const auto SW128 = CU_TENSOR_MAP_SWIZZLE_128B, NOSW = CU_TENSOR_MAP_SWIZZLE_NONE;
    if (!encode_2d(&p.tma_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, op.a_codes, kbytes, op.m, kbytes, BKB, BM, SW128) ||
        !encode_2d(&p.tma_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, op.b_codes, kbytes, op.n, kbytes, BKB, BNH, SW128))
        return cudaErrorInvalidValue;
    const int blk = fmt_block(op.fmt);
    const bool byte_sf = !bf16_operands && fmt_byte_scales(op.fmt);
    if (byte_sf) {
        // scale atoms as rows of 64 x 8-byte elements: (row tile, scale-column group) -> atom index
        const int64_t s_pad = ((op.k / blk) + 15) / 16 * 16;
        const int64_t atoms_a = ((op.m + 127) / 128) * (s_pad / 4), atoms_b = ((op.n + 127) / 128) * (s_pad / 4);
        const int nsf = op.fmt == kNVFP4 ? 4 : op.fmt == kMXFP4 ? 2 : 1;
        if (!encode_2d(&p.tma_sfa, CU_TENSOR_MAP_DATA_TYPE_UINT64, op.a_scales, 64, atoms_a, 512, 64, nsf, NOSW) ||
            !encode_2d(&p.tma_sfb, CU_TENSOR_MAP_DATA_TYPE_UINT64, op.b_scales, 64, atoms_b, 512, 64, nsf, NOSW))
            return cudaErrorInvalidValue;
        p.s4 = (int)(s_pad / 4);
    }
    if (op.tp) {
        if (!encode_2d(&p.tma_t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, op.tp, 64, op.m, 128, 64, BM, SW128) ||
            !encode_2d(&p.tma_l2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, op.l2p, 64, op.n, 128, 64, BNH, SW128))
            return cudaErrorInvalidValue;
    }
    const int esz = op.y_bf16 ? 2 : 4;
    p.y_tma = ((op.n * esz) % 16 == 0) && ((reinterpret_cast<uintptr_t>(op.y) & 15u) == 0);
    if (p.y_tma &&
        !encode_2d(&p.tma_y, op.y_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, op.y,
                   op.n, op.m, op.n * esz, 32, 32, op.y_bf16 ? CU_TENSOR_MAP_SWIZZLE_64B : SW128))
        p.y_tma = 0;
    p.a_row_scale = (const float *)op.a_scales;
    p.b_row_scale = (const float *)op.b_scales;
    p.a_ts = op.a_tensor_scale;
    p.b_ts = op.b_tensor_scale;
    p.y = op.y;
    p.m = (int)op.m;
    p.n = (int)op.n;
    p.kbytes = (int)kbytes;
    p.num_k_tiles = (int)((kbytes + BKB - 1) / BKB);
    p.has_lowrank = op.tp != nullptr;
    p.y_bf16 = op.y_bf16;
    p.m_tiles = (int)((op.m + 255) / 256);
    p.n_tiles = (int)((op.n + BN - 1) / BN);
    p.sfa_tiles = (int)((op.m + 127) / 128);
    p.wait_ns = 2000000000ull;   // 2 s
    const int sms = sm_count();
    const int tiles = p.m_tiles * p.n_tiles;
    const int clusters = tiles < sms / 2 ? tiles : sms / 2;
    const int grid = 2 * clusters;
    if (bf16_operands) return launch_kind<kKindBF16>(p, grid, s);
    switch (op.fmt) {
    case kNVFP4: return launch_kind<kKindNVFP4>(p, grid, s);
    case kMXFP4: return launch_kind<kKindMXFP4>(p, grid, s);
    case kMXFP8: return launch_kind<kKindMXFP8>(p, grid, s);
    case kFP8Tensor: return launch_kind<kKindFP8>(p, grid, s);
    case kINT8Row: return launch_kind<kKindINT8>(p, grid, s);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_qlinear(const GemmOperands &op, cudaStream_t s) { return launch_gemm_common(op, false, s); }

cudaError_t launch_gemm_bf16(const GemmOperands &op, cudaStream_t s) { return launch_gemm_common(op, true, s); }

namespace {
constexpr unsigned int kErrSelfTest = 64u;

// Self-test of the bounded waits and the error word: one thread waits on an
// mbarrier that nothing arrives on (its first phase never completes); when
// the bound runs out it latches the error word as every bounded wait of the
// library's kernels does, and the kernel returns.
__global__ void k_wait_selftest(unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    if (!mbar_wait(&bar, 0, limit_ns)) latch_error(kErrSelfTest);
}
}  // namespace

cudaError_t launch_wait_selftest(unsigned long long limit_ns, cudaStream_t s) {
    k_wait_selftest<<<1, 32, 0, s>>>(limit_ns);
    return cudaGetLastError();
}

cudaError_t error_word_address(unsigned int **ptr) {
    static unsigned int *addr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_error_word);
        if (e != cudaSuccess) return e;
        addr[dev] = reinterpret_cast<unsigned int *>(p);
    }
    *ptr = addr[dev];
    return cudaSuccess;
}

cudaError_t read_and_clear_error(unsigned int *value) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(value, g_error_word, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbol(g_error_word, &zero, sizeof(unsigned int));
}

}  // namespace mxq
