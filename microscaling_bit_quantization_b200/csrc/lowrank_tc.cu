// lowrank_tc.cu -- the low-rank down-projection T = bf16(X) . L1 (optionally
// with the tensor amax of X) in one pass over X on 5th-generation tensor
// cores.
//
// Source: Nunchaku/Diffusers article, "Main explanation": SVDQuant keeps a
// 16-bit low-rank branch beside the 4-bit residual, and its down-projection
// X . L1 (rank r <= 32 here) runs on the unquantized activation.
//
// Structure.  Clusters of S CTAs (S in {1, 2, 4, 8}) walk the 128-row tiles
// of X.  CTA j of a cluster owns the k-blocks [j KB / S, (j + 1) KB / S)
// (64 columns each) of every row tile, so its slice of L1 is transposed once
// into K-major, 128-byte-swizzled B tiles (32 rows, zeros past r and K) that
// stay in shared memory.  Per CTA:
//   warp 0      TMA producer: 128 x 64 bf16 tiles of X into a 6-stage ring
//   warp 1      TMEM allocation (two 32-column accumulators) and the MMA
//               thread: four kind::f16 M=128 N=32 K=16 MMAs per tile
//   warps 2-5   the tensor amax from every staged tile (when asked); at the
//               end of a row tile the accumulator rows are reduce-scattered
//               over the cluster through distributed shared memory: CTA i
//               receives rows [i R, (i + 1) R), R = 128 / S, of every CTA's
//               partial, adds them in rank order (so T does not depend on
//               timing) and writes T, or the packed GEMM operand
//               [bf16(u) | bf16(u - bf16(u))], u = T / (s_x s_w).
// All waits are bounded; one that runs out latches the error word and the
// CTA stops issuing work (the cluster still meets at its final barrier).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "mxq_formats.cuh"
#include "mxq_internal.h"
#include "tc_ptx.cuh"

namespace mxq {
namespace {

constexpr int LT_STAGES = 6;
constexpr int LT_X = 128 * 128;         // one 128-row x 64-column bf16 tile of X
constexpr int LT_B = 32 * 128;          // one 32-row x 64-column bf16 tile of L1^T
constexpr int LT_RED = 128 * 32 * 4;    // reduce buffer: 128 rows x 32 fp32
constexpr int LT_BAR = 256;
constexpr int LT_THREADS = 192;
constexpr uint32_t LT_TMEM_COLS = 64;
constexpr int LT_SMEM_MAX = 232448;     // 227 KB per CTA
constexpr unsigned int kErrLt = 16u;

// M = 128, N = 32, bf16 x bf16 -> fp32, K-major A and B; the same with B
// MN-major (bit 16) for B tiles that are L1's own rows.
constexpr uint32_t kLtIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((32u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kLtIdescBmn = kLtIdesc | (1u << 16);

// Shared-memory descriptor of an MN-major operand with 64-byte swizzle: rows
// of 64 B (the 32 columns of L1), 8-row groups 512 B apart.
__device__ __forceinline__ uint64_t sdesc_mn_sw64(const void *p) {
    const uint64_t a = (smem_u32(p) >> 4) & 0x3FFFu;
    return a | (1ull << 16) | (32ull << 32) | (1ull << 46) | (4ull << 61);
}

inline int lt_smem_bytes(int kb_max) { return LT_STAGES * LT_X + kb_max * LT_B + 2 * LT_RED + LT_BAR + 1024; }

struct LrTcParams {
    CUtensorMap tma_x;
    CUtensorMap tma_l1;        // L1 rows (r = 32), 64-row boxes, 64-byte swizzle; used when b_tma
    const __nv_bfloat16 *l1;   // k x r
    float *t;                  // m x r (T output) or null
    __nv_bfloat16 *tp;         // m x 64 (packed output) or null
    const float *xs, *ws;      // packed output divisor s_x * s_w; null: 1
    float *amax_slots;         // null: no amax; else warp w (2-5) of CTA b writes slot 4 b + w - 2
    unsigned int *err;
    int m, k, r, kb_total, kb_max, row_tiles, S, b_tma;
    unsigned long long wait_ns;
};

__device__ __forceinline__ void tma_load_x(const CUtensorMap *map, void *dst, uint64_t *bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void mma_lt(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void commit_lt(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// Asynchronous 16-byte store into a cluster peer's shared memory that counts
// its bytes on the peer's mbarrier (complete_tx): no fence, no separate arrival.
__device__ __forceinline__ void st_async_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                            uint32_t bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                     addr),
                 "r"(a), "r"(b), "r"(c), "r"(d), "r"(bar)
                 : "memory");
}

// Max |x| of eight packed bf16 pairs (exact: it is one of the values).
__device__ __forceinline__ float amax_bf16x8(uint4 a, uint4 b) {
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; i++) {
        m = fmaxf(m, fabsf(__uint_as_float(w[i] << 16)));
        m = fmaxf(m, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
    }
    return m;
}

template <int S>
__global__ void __launch_bounds__(LT_THREADS, 1) k_lowrank_tc(const __grid_constant__ LrTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *xst = smem;
    uint8_t *btile = smem + LT_STAGES * LT_X;
    float *red = reinterpret_cast<float *>(btile + p.kb_max * LT_B);   // [2][128][32]
    uint64_t *full = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(red) + 2 * LT_RED);
    uint64_t *empty = full + LT_STAGES;
    uint64_t *accf = empty + LT_STAGES;
    uint64_t *acce = accf + 2;
    uint64_t *redf = acce + 2;      // my reduce buffer filled (bytes of remote st.async)
    uint64_t *redfree = redf + 2;   // every receiver has consumed buffer (remote arrivals)
    uint64_t *sumdone = redfree + 2;   // the four reducing warps are done with my buffer
    uint64_t *drain = sumdone + 2;
    uint64_t *bfull = drain + 1;    // the B tiles loaded by TMA (b_tma)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bfull + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int R = 128 / S;
    constexpr uint32_t kRedBytes = S * R * 32 * 4;   // bytes each CTA receives per row tile
    const uint32_t rank = cluster_rank();
    const int cid = (int)cluster_id(), ncl = (int)cluster_count();
    const int kb0 = (int)(rank * (uint32_t)p.kb_total / (uint32_t)S);
    const int nkb = (int)((rank + 1) * (uint32_t)p.kb_total / (uint32_t)S) - kb0;
    const int ntiles = cid < p.row_tiles ? (p.row_tiles - cid + ncl - 1) / ncl : 0;
    const int total = ntiles * nkb;
    const bool want_amax = p.amax_slots != nullptr;

    if (threadIdx.x == 0) {
        for (int s = 0; s < LT_STAGES; s++) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, want_amax ? 5 : 1);   // the MMA commit (+ the four amax warps)
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(accf + i, 1);
            mbar_init(acce + i, 4);
            // S > 1: its own expect_tx, completed by the senders' st.async bytes;
            // S == 1: one arrival per warp after plain local stores
            mbar_init(redf + i, S > 1 ? 1 : 4);
            mbar_init(redfree + i, (uint32_t)S);
            mbar_init(sumdone + i, 4);
        }
        mbar_init(drain, 1);
        mbar_init(bfull, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (S > 1) {   // the bytes of the first two row tiles are expected before any sender may start
            mbar_arrive_expect_tx(redf + 0, kRedBytes);
            mbar_arrive_expect_tx(redf + 1, kRedBytes);
        }
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(LT_TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    cluster_sync();   // barriers of every CTA initialized before any remote arrival
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // setup above overlaps the previous kernel; X, L1 and the scales are read,
    // and T and the maxima written, only after it has completed
    pdl_wait();
    pdl_launch_dependents();

    // The first tiles of X are in flight while the B tiles are built; the L1
    // loads of the first round are issued before them, so they are not queued
    // behind the prefetch of X.
    const int pre = total < LT_STAGES ? total : LT_STAGES;
    auto prefetch_x = [&]() {
        if (warp == 0 && lane == 0) {
            for (int u = 0; u < pre; u++) {
                const int rt = cid + (u / nkb) * ncl, kb = kb0 + u % nkb;
                mbar_arrive_expect_tx(full + u, LT_X);
                tma_load_x(&p.tma_x, xst + u * LT_X, full + u, kb * 64, rt * 128);
            }
        }
    };
    if (p.b_tma) {
        // B tile j is rows (kb0 + j) 64 .. + 63 of L1 as they are (MN-major, 64-byte swizzle,
        // zeros past K): no transpose
        if (warp == 0 && lane == 0) {
            mbar_arrive_expect_tx(bfull, (uint32_t)(nkb * LT_B));
            for (int j = 0; j < nkb; j++) tma_load_x(&p.tma_l1, btile + j * LT_B, bfull, 0, (kb0 + j) * 64);
        }
        prefetch_x();
    } else if (p.r % 8 == 0 && (reinterpret_cast<uintptr_t>(p.l1) & 15u) == 0) {
        // B tile j, row n, 16-byte unit c holds L1[(kb0 + j) 64 + 8 c + t][n], t = 0..7 (128B swizzle)
        // 8 x 8 blocks: eight independent 16-byte row loads, a transpose by byte permutes, eight stores
        auto load_block = [&](int idx, uint4 (&rv)[8]) {
            const int j = idx >> 5, c = (idx >> 2) & 7, n0 = 8 * (idx & 3);
            const int kk0 = (kb0 + j) * 64 + 8 * c;
#pragma unroll
            for (int t = 0; t < 8; t++)
                rv[t] = (idx < nkb * 32 && n0 < p.r && kk0 + t < p.k)
                            ? __ldg(reinterpret_cast<const uint4 *>(p.l1 + (int64_t)(kk0 + t) * p.r + n0))
                            : make_uint4(0u, 0u, 0u, 0u);
        };
        auto store_block = [&](int idx, const uint4 (&rv)[8]) {
            if (idx >= nkb * 32) return;
            const int j = idx >> 5, c = (idx >> 2) & 7, n0 = 8 * (idx & 3);
#pragma unroll
            for (int i = 0; i < 4; i++) {   // columns n0 + 2i (low halves) and n0 + 2i + 1 (high halves)
                uint32_t lo[4], hi[4];
#pragma unroll
                for (int jj = 0; jj < 4; jj++) {
                    const uint32_t *wa = reinterpret_cast<const uint32_t *>(&rv[2 * jj]);
                    const uint32_t *wb = reinterpret_cast<const uint32_t *>(&rv[2 * jj + 1]);
                    lo[jj] = __byte_perm(wa[i], wb[i], 0x5410);
                    hi[jj] = __byte_perm(wa[i], wb[i], 0x7632);
                }
                const int na = n0 + 2 * i, nb = na + 1;
                *reinterpret_cast<uint4 *>(btile + j * LT_B + na * 128 + ((c ^ (na & 7)) << 4)) =
                    make_uint4(lo[0], lo[1], lo[2], lo[3]);
                *reinterpret_cast<uint4 *>(btile + j * LT_B + nb * 128 + ((c ^ (nb & 7)) << 4)) =
                    make_uint4(hi[0], hi[1], hi[2], hi[3]);
            }
        };
        // two blocks per thread per round, all sixteen loads in flight before any transpose
        for (int idx = threadIdx.x; idx < nkb * 32; idx += 2 * LT_THREADS) {
            uint4 ra[8], rb[8];
            load_block(idx, ra);
            load_block(idx + LT_THREADS, rb);
            if (idx == (int)threadIdx.x) prefetch_x();
            store_block(idx, ra);
            store_block(idx + LT_THREADS, rb);
        }
        if (nkb * 32 <= (int)threadIdx.x) prefetch_x();   // a thread without blocks
    } else {
        prefetch_x();
        for (int idx = threadIdx.x; idx < nkb * 256; idx += LT_THREADS) {
            const int j = idx >> 8, n = (idx >> 3) & 31, c = idx & 7;
            const int kk0 = (kb0 + j) * 64 + 8 * c;
            uint32_t h[8];
#pragma unroll
            for (int t = 0; t < 8; t++)
                h[t] = (n < p.r && kk0 + t < p.k) ? (uint32_t)__bfloat16_as_ushort(p.l1[(int64_t)(kk0 + t) * p.r + n]) : 0u;
            *reinterpret_cast<uint4 *>(btile + j * LT_B + n * 128 + ((c ^ (n & 7)) << 4)) =
                make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
        }
    }
    fence_async_smem();   // the generic-proxy B tiles become visible to the tensor cores
    __syncthreads();

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            int issued = pre;
            for (int u = pre; u < total && !*abort_flag; u++) {
                const int s = u % LT_STAGES;
                if (!mbar_wait(empty + s, ((u / LT_STAGES) & 1) ^ 1, p.wait_ns)) {
                    atomicOr(p.err, kErrLt);
                    *abort_flag = 1;
                    break;
                }
                const int rt = cid + (u / nkb) * ncl, kb = kb0 + u % nkb;
                mbar_arrive_expect_tx(full + s, LT_X);
                tma_load_x(&p.tma_x, xst + s * LT_X, full + s, kb * 64, rt * 128);
                issued = u + 1;
            }
            if (*abort_flag) {   // let the copies in flight land
                for (int i = (issued > LT_STAGES ? issued - LT_STAGES : 0); i < issued; i++)
                    mbar_wait(full + (i % LT_STAGES), (i / LT_STAGES) & 1, p.wait_ns);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int u = 0;
            bool any = false;
            const bool bmn = p.b_tma != 0;
            const uint32_t idesc = bmn ? kLtIdescBmn : kLtIdesc;
            if (bmn && ntiles > 0 && !mbar_wait(bfull, 0, p.wait_ns)) {
                atomicOr(p.err, kErrLt);
                *abort_flag = 1;
            }
            for (int tc = 0; tc < ntiles && !*abort_flag; tc++) {
                const uint32_t slot = (uint32_t)(tc & 1);
                bool ok = mbar_wait(acce + slot, ((tc >> 1) & 1) ^ 1, p.wait_ns);
                tc_fence_after();
                for (int j = 0; ok && j < nkb; j++, u++) {
                    const int s = u % LT_STAGES;
                    ok = mbar_wait(full + s, (u / LT_STAGES) & 1, p.wait_ns);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < 4; ks++)   // K = 16 per MMA: 32 bytes of a K-major row, 16 rows of an MN-major tile
                        mma_lt(tmem + slot * 32, sdesc_sw128(xst + s * LT_X + ks * 32),
                               bmn ? sdesc_mn_sw64(btile + j * LT_B + ks * 1024) : sdesc_sw128(btile + j * LT_B + ks * 32),
                               idesc, (j > 0 || ks > 0) ? 1u : 0u);
                    commit_lt(empty + s);
                    any = true;
                }
                if (!ok) {
                    atomicOr(p.err, kErrLt);
                    *abort_flag = 1;
                    break;
                }
                commit_lt(accf + slot);
            }
            if (*abort_flag && any) {   // nothing may be in flight when TMEM is released
                commit_lt(drain);
                mbar_wait(drain, 0, p.wait_ns);
            }
        }
    } else {
        // ---------------------------------------------------------- amax + reduce-scatter (warps 2-5)
        const int e = warp - 2, q = warp & 3, te = e * 32 + lane;
        float mx = 0.0f;
        float alpha = 1.0f;
        if (p.tp && p.xs) alpha = __fmul_rn(*p.xs, *p.ws);
        int u = 0;
        bool ok = true;
        for (int tc = 0; tc < ntiles && ok; tc++) {
            const int rt = cid + tc * ncl;
            if (want_amax) {
                for (int j = 0; j < nkb; j++, u++) {
                    const int s = u % LT_STAGES;
                    bool w = !*abort_flag && mbar_wait(full + s, (u / LT_STAGES) & 1, p.wait_ns);
                    if (!__all_sync(0xFFFFFFFFu, w)) {
                        ok = false;
                        break;
                    }
                    const uint4 *src = reinterpret_cast<const uint4 *>(xst + s * LT_X + e * 4096);
#pragma unroll
                    for (int i = 0; i < 8; i += 2) mx = fmaxf(mx, amax_bf16x8(src[lane + 32 * i], src[lane + 32 * (i + 1)]));
                    __syncwarp();
                    if (lane == 0) mbar_arrive_local(empty + s);
                }
                if (!ok) break;
            }
            // the waits of this phase poll: the stream is over, so nothing else needs the issue slots
            const uint32_t slot = (uint32_t)(tc & 1);
            bool w = !*abort_flag && mbar_wait_spin(accf + slot, (tc >> 1) & 1, p.wait_ns);
            if (!__all_sync(0xFFFFFFFFu, w)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t v[32];
            tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + slot * 32, v);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_local(acce + slot);

            // send this thread's row (row q*32 + lane of the tile) to the CTA that owns it
            const uint32_t pb = (uint32_t)(tc & 1);
            w = mbar_wait_spin<true>(redfree + pb, ((tc >> 1) & 1) ^ 1, p.wait_ns);
            if (!__all_sync(0xFFFFFFFFu, w)) {
                ok = false;
                break;
            }
            const int row_t = q * 32 + lane, dst = row_t / R, lr = row_t % R;
            float *mine = red + pb * (128 * 32) + ((int)rank * R + lr) * 32;
            if (S > 1) {
                const uint32_t raddr = map_to_rank(mine, (uint32_t)dst), rbar = map_to_rank(redf + pb, (uint32_t)dst);
#pragma unroll
                for (int i = 0; i < 8; i++)
                    st_async_v4(raddr + 16 * i, v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3], rbar);
            } else {   // the whole tile stays in this CTA
#pragma unroll
                for (int i = 0; i < 8; i++)
                    reinterpret_cast<uint4 *>(mine)[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                __syncwarp();
                if (lane == 0) mbar_arrive_local(redf + pb);
            }

            // receive rows [rank R, rank R + R) from every CTA, add in rank order, write
            w = mbar_wait_spin<true>(redf + pb, (tc >> 1) & 1, p.wait_ns);
            if (!__all_sync(0xFFFFFFFFu, w)) {
                ok = false;
                break;
            }
            const float *buf = red + pb * (128 * 32);
#pragma unroll
            for (int pos = te; pos < R * 32; pos += 128) {
                const int row = pos >> 5, col = pos & 31;
                float part[S];
#pragma unroll
                for (int jj = 0; jj < S; jj++) part[jj] = buf[(jj * R + row) * 32 + col];
                float sum = 0.0f;
#pragma unroll
                for (int jj = 0; jj < S; jj++) sum = __fadd_rn(sum, part[jj]);
                const int64_t grow = (int64_t)rt * 128 + (int)rank * R + row;
                if (grow < p.m) {
                    if (p.t) {
                        if (col < p.r) p.t[grow * p.r + col] = sum;
                    } else {
                        float uu = col < p.r ? sum : 0.0f;
                        if (p.xs && col < p.r) uu = __fdiv_rn(uu, alpha);
                        const __nv_bfloat16 hi = __float2bfloat16_rn(uu);
                        p.tp[grow * 64 + col] = hi;
                        p.tp[grow * 64 + 32 + col] = __float2bfloat16_rn(__fsub_rn(uu, __bfloat162float(hi)));
                    }
                }
            }
            // buffer pb is free again once all four warps are done with it: tell every sender
            // (not after this cluster's last row tile: nothing is sent into it again)
            if (tc + 1 == ntiles) continue;
            __syncwarp();
            if (lane == 0) mbar_arrive_local(sumdone + pb);
            if (te == 0) {
                if (mbar_wait(sumdone + pb, (tc >> 1) & 1, p.wait_ns)) {
                    if (S > 1) mbar_arrive_expect_tx(redf + pb, kRedBytes);   // the bytes of row tile tc + 2
                    for (int d = 0; d < S; d++) mbar_arrive_remote(map_to_rank(redfree + pb, (uint32_t)d));
                } else {
                    ok = false;
                }
            }
            ok = __all_sync(0xFFFFFFFFu, ok);
        }
        if (!ok) {
            if (lane == 0 && !*abort_flag) atomicOr(p.err, kErrLt);
            *abort_flag = 1;
        }
        if (want_amax) {   // every slot is written, so the slots need no clearing
            mx = group_max<32>(mx);
            if (lane == 0) p.amax_slots[4 * blockIdx.x + e] = mx;
        }
    }

    tc_fence_before();
    cluster_sync();   // no CTA leaves while another may still write its shared memory
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(LT_TMEM_COLS));
    }
}

}  // namespace

cudaError_t launch_lowrank_tc(const void *x, int64_t m, int64_t k, const void *l1, int r, float *t, void *tp,
                              const float *xs, const float *ws, float *amax_slots, int *n_slots,
                              cudaStream_t s) {
    if (m <= 0 || k <= 0 || r < 1 || r > 32 || k % 8 || m >= ((int64_t)1 << 31) || k >= ((int64_t)1 << 31) ||
        (reinterpret_cast<uintptr_t>(x) & 15u))
        return cudaErrorNotSupported;
    LrTcParams p;
    memset(&p, 0, sizeof(p));
    p.m = (int)m;
    p.k = (int)k;
    p.r = r;
    p.row_tiles = (int)((m + 127) / 128);
    p.kb_total = (int)((k + 63) / 64);
    static PerDeviceOnce smem_opt_in;
    const cudaError_t se = smem_opt_in.run([] {
        for (auto fn : {k_lowrank_tc<1>, k_lowrank_tc<2>, k_lowrank_tc<4>, k_lowrank_tc<8>}) {
            cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, LT_SMEM_MAX);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    });
    if (se != cudaSuccess) return se;
    const int dev = current_device_index();
    if (dev < 0) return cudaErrorInvalidDevice;
    // cluster size: fewest rounds x k-blocks per CTA, then the smaller cluster; the
    // number of clusters that fit on the GPU at once comes from the occupancy query
    // co-resident clusters per cluster size, per device (0: not yet queried; else the count + 1)
    static std::atomic<int> max_clusters_cache[kMaxDevices][4];
    int best_s = 0, best_clusters = 0;
    int64_t best_cost = 0;
    for (int li = 0, S = 1; S <= 8; li++, S *= 2) {
        if (S > p.kb_total) break;
        const int kb_max = (p.kb_total + S - 1) / S;
        if (lt_smem_bytes(kb_max) > LT_SMEM_MAX) continue;
        int max_clusters = max_clusters_cache[dev][li].load(std::memory_order_relaxed) - 1;
        if (max_clusters < 0) {
            cudaLaunchConfig_t q = {};
            q.gridDim = dim3((unsigned)S, 1, 1);
            q.blockDim = dim3(LT_THREADS, 1, 1);
            q.dynamicSmemBytes = (size_t)LT_SMEM_MAX;
            cudaLaunchAttribute a;
            a.id = cudaLaunchAttributeClusterDimension;
            a.val.clusterDim.x = (unsigned)S;
            a.val.clusterDim.y = 1;
            a.val.clusterDim.z = 1;
            q.attrs = &a;
            q.numAttrs = 1;
            int n = 0;
            const cudaError_t oe = S == 1 ? cudaOccupancyMaxActiveClusters(&n, k_lowrank_tc<1>, &q)
                                 : S == 2 ? cudaOccupancyMaxActiveClusters(&n, k_lowrank_tc<2>, &q)
                                 : S == 4 ? cudaOccupancyMaxActiveClusters(&n, k_lowrank_tc<4>, &q)
                                          : cudaOccupancyMaxActiveClusters(&n, k_lowrank_tc<8>, &q);
            if (oe != cudaSuccess) {
                cudaGetLastError();
                n = 0;
            }
            max_clusters = n;
            max_clusters_cache[dev][li].store(n + 1, std::memory_order_relaxed);
        }
        const int clusters = p.row_tiles < max_clusters ? p.row_tiles : max_clusters;
        if (clusters < 1) continue;
        const int64_t cost = (int64_t)((p.row_tiles + clusters - 1) / clusters) * kb_max;
        if (!best_s || cost < best_cost) {
            best_s = S;
            best_cost = cost;
            best_clusters = clusters;
        }
    }
    if (!best_s) return cudaErrorNotSupported;
    p.S = best_s;
    p.kb_max = (p.kb_total + best_s - 1) / best_s;
    p.l1 = (const __nv_bfloat16 *)l1;
    p.t = t;
    p.tp = (__nv_bfloat16 *)tp;
    p.xs = xs;
    p.ws = ws;
    p.amax_slots = amax_slots;
    if (4 * best_clusters * best_s > kAmaxSlots) return cudaErrorNotSupported;
    if (n_slots) *n_slots = 4 * best_clusters * best_s;
    p.wait_ns = 2000000000ull;
    cudaError_t e = error_word_address(&p.err);
    if (e != cudaSuccess) return e;
    if (!encode_2d(&p.tma_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)k, (uint64_t)m, (uint64_t)k * 2, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    // rank 32: the B tiles are L1's rows loaded as they are (else built by a transpose in the kernel)
    p.b_tma = r == 32 && (reinterpret_cast<uintptr_t>(l1) & 15u) == 0 &&
              encode_2d(&p.tma_l1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, l1, 32, (uint64_t)k, 64, 32, 64,
                        CU_TENSOR_MAP_SWIZZLE_64B);
    const int smem = lt_smem_bytes(p.kb_max);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(best_clusters * best_s), 1, 1);
    cfg.blockDim = dim3(LT_THREADS, 1, 1);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)best_s;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl_attribute();
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    switch (best_s) {
    case 1: return cudaLaunchKernelEx(&cfg, k_lowrank_tc<1>, p);
    case 2: return cudaLaunchKernelEx(&cfg, k_lowrank_tc<2>, p);
    case 4: return cudaLaunchKernelEx(&cfg, k_lowrank_tc<4>, p);
    default: return cudaLaunchKernelEx(&cfg, k_lowrank_tc<8>, p);
    }
}

}  // namespace mxq
