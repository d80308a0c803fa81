// gemm_igroup.cu -- INT4 per-group GEMM (4-bit weights and activations, one
// fp32 scale per group of 32 or 64 along K) on 5th-generation tensor cores,
// with the SVDQuant low-rank branch fused.
//
// Sources: Nunchaku/Diffusers article -- the INT4 variant of svdq_w4a4 keeps
// 4-bit weights and activations with group scales and a 16-bit low-rank
// branch beside the 4-bit residual (sections "Main explanation", "Kernels and
// supported hardware"); Chameleon article -- INT4 with groups of 32 is one of
// the per-channel weight formats.
//
// Y[m,n] = sum_g sx[m,g] sw[n,g] P_g[m,n] + (T . L2)[m,n], where P_g is the
// dot product of the integer codes over group g.  The group scales are
// arbitrary fp32 values that the tensor cores cannot apply, so each P_g is
// formed on its own: the codes are stored as E4M3 bytes (every integer in
// [-7, 7] is an E4M3 value), a kind::f8f6f4 MMA gives P_g exactly in fp32
// (|P_g| <= 64 * 49), and the epilogue folds it into fp32 running sums held
// in registers, acc += P_g * (sx * sw).  The mixed-format linear layer runs
// the same kernel with MXFP8 activations (E4M3 codes, sx = 2^e of the
// 32-element block) against INT4-g32 weights; P_g then sums 32 products of
// E4M3 values and integers, each exact, in fp32.  Those two ALU operations per output
// element and group (one packed fp32x2 multiply and FMA per two columns) and
// the latency of fetching each group's sums from TMEM bound the kernel; the
// MMAs of a group run up to three groups ahead in a ring of four TMEM buffers.
//
// Per CTA (one per SM, persistent over 128 x 128 output tiles):
//   warp 0      TMA producer into a 6-stage ring (A and B tiles of
//               128 rows x 128 B, 128-byte swizzle)
//   warp 1      TMEM allocation (4 group buffers x 128 columns) and the
//               thread that issues the MMAs (cta_group::1)
//   warps 2-17  epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 (its 32
//               rows) and one quarter of the 128 columns ((w - 2) / 4), keeps
//               32 running sums per thread and stores its rows of Y.  Each
//               group's 32 columns are loaded, the buffer released at once,
//               then folded: four epilogue warps per scheduler hide the load
//               latency of one another.  Each warp's group scales arrive by
//               cp.async in a ring of shared-memory slots IG_SCALE_AHEAD
//               groups ahead of their use
// The low-rank branch is one more group with scale 1: a bf16 kind::f16 MMA
// of the packed activation [T_hi | T_lo] against [L2^T | L2^T].
// Every wait is bounded; a wait that runs out latches the error word and
// the CTA drains its in-flight copies and MMAs and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "mxq_formats.cuh"
#include "mxq_internal.h"
#include "tc_ptx.cuh"

namespace mxq {
namespace {

constexpr int IG_BM = 128, IG_BN = 128, IG_BKB = 128;   // tile rows, columns, K bytes per stage
constexpr int IG_STAGES = 6;
constexpr int IG_A = IG_BM * IG_BKB, IG_B = IG_BN * IG_BKB;   // 16 KB each
constexpr int IG_STAGE = IG_A + IG_B;
constexpr int IG_NBUF = 4;                                    // TMEM group buffers
constexpr uint32_t IG_TMEM_COLS = IG_NBUF * IG_BN;            // 512
constexpr int IG_EPI_WARPS = 16;
constexpr int IG_EPI_COLS = IG_BN / (IG_EPI_WARPS / 4);        // 32 columns per epilogue warp
constexpr int IG_THREADS = 64 + 32 * IG_EPI_WARPS;            // 576
constexpr int IG_SCALE_SLOTS = 8, IG_SCALE_AHEAD = 6;          // per-warp scale ring: slots, groups in flight
constexpr int IG_SLOT_FLOATS = 32 + IG_EPI_COLS;              // sx of the warp's 32 rows, sw of its columns
constexpr int IG_WSCALE_BYTES = IG_EPI_WARPS * IG_SCALE_SLOTS * IG_SLOT_FLOATS * 4;
constexpr int IG_BAR_BYTES = 256;
constexpr int IG_SMEM = IG_STAGES * IG_STAGE + IG_WSCALE_BYTES + IG_BAR_BYTES + 1024;

constexpr unsigned int kErrIgProducer = 1u, kErrIgMma = 2u, kErrIgEpilogue = 4u;

// M = 128, N = 128, K-major A and B, fp32 accumulator.
constexpr uint32_t kIdescShape = ((uint32_t)(IG_BN >> 3) << 17) | ((uint32_t)(IG_BM >> 4) << 24);
constexpr uint32_t kIdescE4M3 = kIdescShape | (1u << 4);                           // E4M3 x E4M3
constexpr uint32_t kIdescBF16 = kIdescShape | (1u << 4) | (1u << 7) | (1u << 10);  // bf16 x bf16

struct IGroupParams {
    CUtensorMap tma_a, tma_b, tma_t, tma_l2;
    const float *sx, *sw;   // group scales, transposed: [K/g][M] and [K/g][N]
    void *y;
    unsigned int *err;
    int m, n, k, k_tiles, groups, has_lowrank, y_bf16, y_vec, m_tiles, n_tiles;
    unsigned long long wait_ns;
};

__device__ __forceinline__ void tma_load_2d(const CUtensorMap *map, void *dst, uint64_t *bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void mma_e4m3(uint32_t d, uint64_t a, uint64_t b, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(kIdescE4M3), "r"(acc));
}
__device__ __forceinline__ void mma_bf16_1(uint32_t d, uint64_t a, uint64_t b, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(kIdescBF16), "r"(acc));
}
// 4-byte asynchronous copy global -> shared; src_bytes 0 writes a zero.
__device__ __forceinline__ void cp_async4(void *dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Arrive on this CTA's barrier once this thread's issued MMAs complete.
__device__ __forceinline__ void tc_commit_1(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

template <int GROUP>
__global__ void __launch_bounds__(IG_THREADS, 1) k_gemm_igroup(const __grid_constant__ IGroupParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    float *wscale = reinterpret_cast<float *>(smem + IG_STAGES * IG_STAGE);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + IG_STAGES * IG_STAGE + IG_WSCALE_BYTES);
    uint64_t *empty = full + IG_STAGES;
    uint64_t *bfull = empty + IG_STAGES;   // group buffer written (MMA commit)
    uint64_t *bempty = bfull + IG_NBUF;    // group buffer read (all epilogue warps)
    uint64_t *drain = bempty + IG_NBUF;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_tiles = p.m_tiles * p.n_tiles;
    const int nsteps = p.k_tiles + p.has_lowrank;
    const int ngroups = p.groups + p.has_lowrank;

    if (threadIdx.x == 0) {
        for (int s = 0; s < IG_STAGES; s++) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int b = 0; b < IG_NBUF; b++) {
            mbar_init(bfull + b, 1);
            mbar_init(bempty + b, IG_EPI_WARPS);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(IG_TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            int it = 0, issued = 0;
            for (int tile = blockIdx.x; tile < num_tiles && !*abort_flag; tile += gridDim.x) {
                const int m0 = (tile / p.n_tiles) * IG_BM, n0 = (tile % p.n_tiles) * IG_BN;
                for (int kt = 0; kt < nsteps; kt++, it++) {
                    const int s = it % IG_STAGES;
                    if (!mbar_wait(empty + s, ((it / IG_STAGES) & 1) ^ 1, p.wait_ns)) {
                        atomicOr(p.err, kErrIgProducer);
                        *abort_flag = 1;
                        break;
                    }
                    if (*abort_flag) break;
                    uint8_t *sa = smem + s * IG_STAGE, *sb = sa + IG_A;
                    mbar_arrive_expect_tx(full + s, IG_STAGE);
                    if (kt < p.k_tiles) {
                        tma_load_2d(&p.tma_a, sa, full + s, kt * IG_BKB, m0);
                        tma_load_2d(&p.tma_b, sb, full + s, kt * IG_BKB, n0);
                    } else {
                        tma_load_2d(&p.tma_t, sa, full + s, 0, m0);
                        tma_load_2d(&p.tma_l2, sb, full + s, 0, n0);
                    }
                    issued = it + 1;
                }
            }
            if (*abort_flag) {   // let the copies still in flight land before the CTA exits
                for (int i = (issued > IG_STAGES ? issued - IG_STAGES : 0); i < issued; i++)
                    mbar_wait(full + (i % IG_STAGES), (i / IG_STAGES) & 1, p.wait_ns);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int it = 0;
            uint32_t gc = 0;   // groups issued so far (all tiles)
            bool any = false;
            for (int tile = blockIdx.x; tile < num_tiles && !*abort_flag; tile += gridDim.x) {
                for (int kt = 0; kt < nsteps; kt++, it++) {
                    const int s = it % IG_STAGES;
                    bool ok = mbar_wait(full + s, (it / IG_STAGES) & 1, p.wait_ns);
                    if (ok) {
                        tc_fence_after();
                        const uint8_t *sa = smem + s * IG_STAGE, *sb = sa + IG_A;
                        const bool lr = kt >= p.k_tiles;
                        const int rem = lr ? IG_BKB : (p.k - kt * IG_BKB < IG_BKB ? p.k - kt * IG_BKB : IG_BKB);
                        const int ng = lr ? 1 : rem / GROUP;
                        for (int gi = 0; gi < ng && ok; gi++, gc++) {
                            const uint32_t b = gc % IG_NBUF;
                            ok = mbar_wait(bempty + b, ((gc / IG_NBUF) & 1) ^ 1, p.wait_ns);
                            if (!ok) break;
                            tc_fence_after();
                            const uint32_t d = tmem + b * IG_BN;
                            if (lr) {
#pragma unroll
                                for (int ks = 0; ks < 4; ks++)
                                    mma_bf16_1(d, sdesc_sw128(sa + ks * 32), sdesc_sw128(sb + ks * 32), ks > 0);
                            } else {
#pragma unroll
                                for (int mm = 0; mm < GROUP / 32; mm++) {
                                    const int koff = gi * GROUP + mm * 32;
                                    mma_e4m3(d, sdesc_sw128(sa + koff), sdesc_sw128(sb + koff), mm > 0);
                                }
                            }
                            tc_commit_1(bfull + b);
                            any = true;
                        }
                    }
                    if (!ok || *abort_flag) {
                        if (!ok) atomicOr(p.err, kErrIgMma);
                        *abort_flag = 1;
                        break;
                    }
                    tc_commit_1(empty + s);
                }
            }
            if (*abort_flag && any) {   // no MMA may be in flight when TMEM is released
                tc_commit_1(drain);
                mbar_wait(drain, 0, p.wait_ns);
            }
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int e = warp - 2, q = warp & 3, cq = e >> 2;
        float *ring = wscale + e * IG_SCALE_SLOTS * IG_SLOT_FLOATS;
        const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(cq * IG_EPI_COLS);
        uint32_t gc = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const int m0 = (tile / p.n_tiles) * IG_BM, n0 = (tile % p.n_tiles) * IG_BN;
            const int row = m0 + q * 32 + lane;
            const int col0 = n0 + cq * IG_EPI_COLS;
            const bool row_ok = row < p.m;
            // group g's scales into slot g % IG_SCALE_SLOTS: sx of this lane's row, sw of column
            // col0 + lane (zeros past the matrix); one commit group per group
            auto fetch_scales = [&](int g) {
                if (g < p.groups) {
                    float *slot = ring + (g % IG_SCALE_SLOTS) * IG_SLOT_FLOATS;
                    const int c0 = col0 + lane;
                    cp_async4(slot + lane, p.sx + (int64_t)g * p.m + (row_ok ? row : 0), row_ok ? 4u : 0u);
                    cp_async4(slot + 32 + lane, p.sw + (int64_t)g * p.n + (c0 < p.n ? c0 : 0), c0 < p.n ? 4u : 0u);
                }
                cp_async_commit();
            };
            // acc[j] += P[j] * (sx * sw[j]) over the warp's 32 columns; factor 1 for the branch.
            // Two columns per packed fp32x2 operation, each lane rounded like the scalar operation.
            float2 acc[IG_EPI_COLS / 2];
#pragma unroll
            for (int j = 0; j < IG_EPI_COLS / 2; j++) acc[j] = make_float2(0.0f, 0.0f);
            for (int g = 0; g < IG_SCALE_AHEAD; g++) fetch_scales(g);
            bool ok = true;
#pragma unroll 1
            for (int gi = 0; ok && gi < ngroups; gi++, gc++) {
                const bool lr = gi >= p.groups;
                // slot gi + AHEAD was last read by group gi + AHEAD - SLOTS < gi, before an earlier __syncwarp
                fetch_scales(gi + IG_SCALE_AHEAD);
                const uint32_t b = gc % IG_NBUF;
                ok = !*abort_flag && mbar_wait(bfull + b, (gc / IG_NBUF) & 1, p.wait_ns);
                ok = __all_sync(0xFFFFFFFFu, ok);
                if (!ok) {
                    if (lane == 0 && !*abort_flag) atomicOr(p.err, kErrIgEpilogue);
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                uint32_t r[32];
                tmem_ld_32x32b_x32(lane_base + b * IG_BN, r);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_local_relaxed(bempty + b);   // the MMAs may reuse this buffer
                cp_async_wait<IG_SCALE_AHEAD>();   // this group's copies (all but the newest AHEAD) have landed
                __syncwarp();                      // ... for every lane of the warp
                const float *slot = ring + (gi % IG_SCALE_SLOTS) * IG_SLOT_FLOATS;
                if (lr) {
#pragma unroll
                    for (int j = 0; j < 16; j++)
                        acc[j] = __fadd2_rn(acc[j], make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1])));
                } else {
                    const float sxv = slot[lane];
                    const float2 sx2 = make_float2(sxv, sxv);
                    const float4 *sw4 = reinterpret_cast<const float4 *>(slot + 32);
#pragma unroll
                    for (int jj = 0; jj < 8; jj++) {
                        const float4 w4 = sw4[jj];
                        acc[2 * jj] = __ffma2_rn(make_float2(__uint_as_float(r[4 * jj]), __uint_as_float(r[4 * jj + 1])),
                                                 __fmul2_rn(sx2, make_float2(w4.x, w4.y)), acc[2 * jj]);
                        acc[2 * jj + 1] =
                            __ffma2_rn(make_float2(__uint_as_float(r[4 * jj + 2]), __uint_as_float(r[4 * jj + 3])),
                                       __fmul2_rn(sx2, make_float2(w4.z, w4.w)), acc[2 * jj + 1]);
                    }
                }
            }
            cp_async_wait<0>();
            if (!ok) break;
            if (row_ok) {
                if (p.y_bf16) {
                    __nv_bfloat16 *yr = reinterpret_cast<__nv_bfloat16 *>(p.y) + (int64_t)row * p.n + col0;
#pragma unroll
                    for (int jj = 0; jj < IG_EPI_COLS / 8; jj++) {
                        const int c = col0 + 8 * jj;
                        if (p.y_vec && c + 8 <= p.n) {
                            reinterpret_cast<uint4 *>(yr)[jj] =
                                make_uint4(pack_bf16x2(acc[4 * jj].x, acc[4 * jj].y),
                                           pack_bf16x2(acc[4 * jj + 1].x, acc[4 * jj + 1].y),
                                           pack_bf16x2(acc[4 * jj + 2].x, acc[4 * jj + 2].y),
                                           pack_bf16x2(acc[4 * jj + 3].x, acc[4 * jj + 3].y));
                        } else {
#pragma unroll
                            for (int t = 0; t < 8; t++)
                                if (c + t < p.n)
                                    yr[8 * jj + t] = __float2bfloat16_rn((t & 1) ? acc[4 * jj + (t >> 1)].y
                                                                                  : acc[4 * jj + (t >> 1)].x);
                        }
                    }
                } else {
                    float *yr = reinterpret_cast<float *>(p.y) + (int64_t)row * p.n + col0;
#pragma unroll
                    for (int jj = 0; jj < IG_EPI_COLS / 4; jj++) {
                        const int c = col0 + 4 * jj;
                        if (p.y_vec && c + 4 <= p.n) {
                            reinterpret_cast<float4 *>(yr)[jj] =
                                make_float4(acc[2 * jj].x, acc[2 * jj].y, acc[2 * jj + 1].x, acc[2 * jj + 1].y);
                        } else {
#pragma unroll
                            for (int t = 0; t < 4; t++)
                                if (c + t < p.n) yr[4 * jj + t] = (t & 1) ? acc[2 * jj + (t >> 1)].y : acc[2 * jj + (t >> 1)].x;
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(IG_TMEM_COLS));
    }
}

template <int GROUP>
cudaError_t launch_group(const IGroupParams &p, int grid, cudaStream_t s) {
    static PerDeviceOnce smem_opt_in;
    cudaError_t e = smem_opt_in.run(
        [] { return cudaFuncSetAttribute(k_gemm_igroup<GROUP>, cudaFuncAttributeMaxDynamicSharedMemorySize, IG_SMEM); });
    if (e != cudaSuccess) return e;
    k_gemm_igroup<GROUP><<<grid, IG_THREADS, IG_SMEM, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qlinear_igroup(const GemmOperands &op, cudaStream_t s) {
    if (op.m == 0 || op.n == 0) return cudaSuccess;
    const int g = fmt_block(op.fmt);
    IGroupParams p;
    memset(&p, 0, sizeof(p));
    const auto SW128 = CU_TENSOR_MAP_SWIZZLE_128B;
    if (!encode_2d(&p.tma_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, op.a_codes, op.k, op.m, op.k, IG_BKB, IG_BM, SW128) ||
        !encode_2d(&p.tma_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, op.b_codes, op.k, op.n, op.k, IG_BKB, IG_BN, SW128))
        return cudaErrorInvalidValue;
    if (op.tp) {
        if (!encode_2d(&p.tma_t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, op.tp, 64, op.m, 128, 64, IG_BM, SW128) ||
            !encode_2d(&p.tma_l2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, op.l2p, 64, op.n, 128, 64, IG_BN, SW128))
            return cudaErrorInvalidValue;
    }
    cudaError_t e = error_word_address(&p.err);
    if (e != cudaSuccess) return e;
    p.sx = (const float *)op.a_scales;
    p.sw = (const float *)op.b_scales;
    p.y = op.y;
    p.m = (int)op.m;
    p.n = (int)op.n;
    p.k = (int)op.k;
    p.k_tiles = (int)((op.k + IG_BKB - 1) / IG_BKB);
    p.groups = (int)(op.k / g);
    p.has_lowrank = op.tp != nullptr;
    p.y_bf16 = op.y_bf16;
    p.y_vec = ((op.n * (op.y_bf16 ? 2 : 4)) % 16 == 0) && ((reinterpret_cast<uintptr_t>(op.y) & 15u) == 0);
    p.m_tiles = (int)((op.m + IG_BM - 1) / IG_BM);
    p.n_tiles = (int)((op.n + IG_BN - 1) / IG_BN);
    p.wait_ns = 2000000000ull;   // 2 s
    const int sms = sm_count();
    const int tiles = p.m_tiles * p.n_tiles;
    const int grid = tiles < sms ? tiles : sms;
    return g == 32 ? launch_group<32>(p, grid, s) : launch_group<64>(p, grid, s);
}

}  // namespace mxq
