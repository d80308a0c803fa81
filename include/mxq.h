/*
 * mxq.h -- C ABI of the B200 (sm_100a) microscaling quantized-linear library.
 *
 * The library implements the data-parallel hot path of low-bit diffusion
 * inference described by these pages:
 *   - Chameleon article (rit.work, "Chameleon ... format quantization for
 *     diffusion"): per-output-channel weight format chosen by least
 *     reconstruction error; per-layer, per-timestep-interval activation
 *     format table read at run time; MXFP8 forced where channel ranges reach
 *     163x.
 *   - Nunchaku / Diffusers article (jiti.kz): svdq_w4a4 -- W4A4 linear layers
 *     in INT4 and NVFP4 with a 16-bit low-rank branch (SVDQuant).
 *   - "Bridging the Gap Between Promise and Performance for Microscaling FP4
 *     Quantization": NVFP4 / MXFP4, block-diagonal Hadamard rotation.
 * Bit layouts follow the OCP Microscaling (MX) v1.0 definition and NVIDIA's
 * NVFP4 definition (the pages name the formats without defining them).
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" are caller-owned CUDA device memory; the
 *     library never allocates or frees on any call (TMEM used by the GEMM
 *     is allocated and released inside the kernel).  "host" pointers are
 *     read during the call only.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream) unless stated otherwise.
 *   - Matrices are row-major.  X is M x K, W is N x K (K contiguous, the
 *     torch Linear layout), Y = X . W^T is M x N.  Quantization blocks run
 *     along the contiguous (K) dimension.
 *   - 4-bit codes are packed two per byte, element 2i in the low nibble.
 *   - Errors are returned as mxq_status; nothing aborts or throws.  Argument
 *     errors are detected on the host before any launch.  A device-side
 *     bounded wait that runs out is latched in a device error word and
 *     reported by mxq_check().
 *   - The library keeps state per device for the life of the process: the
 *     device addresses of its own device variables (the error word, the
 *     scratch array of the allocation-free entry point) and the kernels'
 *     shared-memory opt-ins, set up on a device's first use.  A
 *     cudaDeviceReset() discards what that state refers to, so the library
 *     must not be used on a device after the device has been reset.
 *   - Stream order holds as usual.  The kernels of the activation -> GEMM
 *     chain (low-rank down projection, quantizer, GEMM) are launched with
 *     programmatic dependent launch: each may start its setup while the
 *     previous kernel in the stream finishes, and waits for that kernel to
 *     complete before its first global read or write.
 */
#ifndef MXQ_H
#define MXQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mxq_status {
    MXQ_OK = 0,
    MXQ_EINVAL = 1,         /* bad argument (shape, pointer, size, enum)          */
    MXQ_EUNSUPPORTED = 2,   /* valid but unsupported combination, or no sm_100 GPU */
    MXQ_ECUDA = 3,          /* a CUDA runtime/driver call failed                   */
    MXQ_ETIMEOUT = 4,       /* a bounded device wait ran out (see mxq_check)       */
    MXQ_ENOSPACE = 5        /* workspace smaller than the *_workspace_bytes query  */
} mxq_status;

/* Formats.  Block sizes are fixed by the format. */
typedef enum mxq_fmt {
    MXQ_MXFP8 = 0,       /* E4M3 codes, 32-element blocks, E8M0 scale (OCP MX)        */
    MXQ_MXFP4 = 1,       /* E2M1 codes, 32-element blocks, E8M0 scale (OCP MX)        */
    MXQ_NVFP4 = 2,       /* E2M1 codes, 16-element blocks, E4M3 scale, fp32 tensor scale */
    MXQ_INT4_G32 = 3,    /* symmetric int4 [-7,7], fp32 scale per 32 elements          */
    MXQ_INT4_G64 = 4,    /* symmetric int4 [-7,7], fp32 scale per 64 elements          */
    MXQ_INT8_ROW = 5,    /* symmetric int8 [-127,127], fp32 scale per row (per token / per output channel) */
    MXQ_FP8_TENSOR = 6,  /* E4M3 codes, one fp32 scale for the whole tensor            */
    MXQ_NUM_FMT = 7
} mxq_fmt;

typedef enum mxq_dtype { MXQ_F32 = 0, MXQ_BF16 = 1 } mxq_dtype;

/* Layout of the codes and scales a quantizer writes.
 *  CANONICAL: codes as above; scales row-major
 *      MXFP8/MXFP4  uint8 E8M0 [rows][cols/32]
 *      NVFP4        uint8 E4M3 [rows][cols/16]
 *      INT4_G32/64  fp32       [rows][cols/g]
 *      INT8_ROW     fp32       [rows]
 *      FP8_TENSOR   none (the tensor scale only)
 *  MMA: the operand layout the qlinear kernels read.
 *      E8M0/E4M3 scales (MXFP8, MXFP4, NVFP4): rows padded to a multiple of
 *        128 (R'), scale columns padded to a multiple of 16 (S'); byte of
 *        (row r, scale column s) at
 *          ((r/128)*(S'/4) + s/4)*512 + (r%32)*16 + ((r%128)/32)*4 + s%4;
 *        padding bytes are written as 0.
 *      INT4_G32/64: codes one byte per element [rows][cols] holding the
 *        E4M3 encoding of the integer code (every integer in [-7, 7] is an
 *        E4M3 value; zero is encoded +0), so that the tensor cores form the
 *        exact integer products in fp32; scales fp32 transposed [cols/g][rows].
 *      INT8_ROW, FP8_TENSOR: identical to CANONICAL.
 */
typedef enum mxq_layout { MXQ_LAYOUT_CANONICAL = 0, MXQ_LAYOUT_MMA = 1 } mxq_layout;

/* A quantized matrix (descriptor only; all pointers are device memory). */
typedef struct mxq_qtensor {
    int32_t fmt;               /* mxq_fmt                                    */
    int32_t layout;            /* mxq_layout of codes and scales             */
    int64_t rows, cols;        /* logical shape (cols = K)                   */
    const void *codes;         /* device                                     */
    const void *scales;        /* device; NULL for FP8_TENSOR                */
    const float *tensor_scale; /* device fp32 scalar for NVFP4 / FP8_TENSOR  */
} mxq_qtensor;

/* Human-readable name of a status code (static string). */
const char *mxq_status_string(mxq_status st);

/* Text of the CUDA error behind the last MXQ_ECUDA that a call made from
 * this host thread returned ("no error" if none yet); static string. */
const char *mxq_last_cuda_error_string(void);

/* 1 if device `device` is an sm_100-family GPU the kernels were built for. */
int mxq_device_supported(int device);

/* Synchronizes `stream`, then reads and clears the device error word.
 * Returns MXQ_ETIMEOUT if a bounded wait ran out since the last check,
 * MXQ_ECUDA if a CUDA error is pending, else MXQ_OK.  Host-blocking. */
mxq_status mxq_check(void *stream);

/* Diagnostics of the error path: launches one thread that waits, for at
 * most wait_us microseconds (1 .. 1,000,000), on a barrier whose phase never
 * completes; the bound runs out and the thread latches the device error word
 * exactly as a stuck wait in the library's kernels would, then returns, so
 * the next mxq_check returns MXQ_ETIMEOUT and the context stays usable.
 * Asynchronous on `stream`.  Errors: MXQ_EINVAL (wait_us out of range),
 * MXQ_ECUDA. */
mxq_status mxq_selftest_wait_timeout(uint32_t wait_us, void *stream);

/* ---------------------------------------------------------------------- */
/* Sizes (host only).                                                      */
/* ---------------------------------------------------------------------- */

/* Bytes of the codes / scales buffers mxq_quantize writes for a rows x cols
 * input in format `fmt` and `layout`.  MXQ_EINVAL for bad arguments. */
mxq_status mxq_codes_bytes(int32_t fmt, int64_t rows, int64_t cols, int32_t layout, size_t *bytes);
mxq_status mxq_scales_bytes(int32_t fmt, int64_t rows, int64_t cols, int32_t layout, size_t *bytes);

/* Scratch bytes mxq_quantize needs (4096 for NVFP4 and FP8_TENSOR: the
 * per-CTA maxima of the tensor-amax pass; 0 otherwise). */
mxq_status mxq_quantize_workspace_bytes(int32_t fmt, size_t *bytes);

/* ---------------------------------------------------------------------- */
/* a1-a3: tensor amax, optional Hadamard, block-scaled quantization.       */
/* ---------------------------------------------------------------------- */

/* Quantize x (rows x cols, fp32 or bf16, device) into `fmt`.
 * Source: Chameleon article (MXFP8 blocks sharing an exponent; dynamic
 * scales kept for PixArt), Nunchaku/Diffusers article (INT4 / NVFP4
 * svdq_w4a4 variants), "Bridging the Gap ..." (NVFP4 groups, MXFP4
 * power-of-two scales, item 3 Hadamard rotation).  Encodings: OCP MX v1.0,
 * NVFP4.  Per block: amax, scale, round-to-nearest-even codes (saturating);
 * NVFP4 and FP8_TENSOR first reduce the tensor amax.
 *   hadamard_b: 0 (off) or a power of two in [2, 256] dividing cols; the
 *     rows are rotated by the orthonormal block-diagonal Sylvester Hadamard
 *     matrix (fp32 butterflies, then one multiply by RN(1/sqrt(b))) before
 *     quantization.
 *   codes, scales: device, sizes from mxq_codes_bytes / mxq_scales_bytes
 *     (scales may be NULL for FP8_TENSOR).
 *   tensor_scale: device fp32 written for NVFP4 / FP8_TENSOR, else ignored
 *     (may be NULL).
 *   workspace: device scratch of mxq_quantize_workspace_bytes (may be NULL
 *     when that is 0); clobbered.
 * Constraints: cols % 16 == 0 and cols % block == 0; rows >= 0.
 * Errors: MXQ_EINVAL (shape / pointer / hadamard_b), MXQ_ENOSPACE,
 * MXQ_ECUDA (launch failure). */
mxq_status mxq_quantize(const void *x, int32_t xdtype, int64_t rows, int64_t cols, int32_t fmt,
                        int32_t hadamard_b, int32_t layout, void *codes, void *scales,
                        float *tensor_scale, void *workspace, size_t workspace_bytes, void *stream);

/* Dequantize q into y (rows x cols, fp32 or bf16, device).  Each output is
 * the code value times its scale(s) computed in fp32 (NVFP4: the exact
 * E2M1 x E4M3 product, then times the tensor scale), rounded to bf16 (RNE)
 * for bf16 output.  Both layouts are accepted.  MXQ_EINVAL on bad args. */
mxq_status mxq_dequantize(const mxq_qtensor *q, void *y, int32_t ydtype, void *stream);

/* Block-diagonal Hadamard rotation y = x . blockdiag(H_b)/sqrt(b) along
 * the rows ("Bridging the Gap ...", item 3).  x, y: rows x cols device
 * arrays of dtype `dtype` (y may alias x).  bf16 output is the fp32 result
 * rounded once (RNE).  b: power of two in [2, 256], cols % b == 0 and
 * cols % 16 == 0. */
mxq_status mxq_hadamard_block(const void *x, void *y, int32_t dtype, int64_t rows, int64_t cols,
                              int32_t b, void *stream);

/* Element conversion used by the codec tests: out[i] = E4M3 byte (elem 0)
 * or E2M1 code in the low nibble (elem 1) of the fp32 x[i], round to
 * nearest even, saturating.  x, out: device, n elements. */
mxq_status mxq_cast(const float *x, int64_t n, int32_t elem, uint8_t *out, void *stream);

/* ---------------------------------------------------------------------- */
/* a4: per-output-channel weight-format selection.                         */
/* ---------------------------------------------------------------------- */

/* Scratch bytes mxq_select_weight_format needs. */
mxq_status mxq_select_workspace_bytes(const int32_t *candidates, int32_t ncand, size_t *bytes);

/* Chameleon article, section "the format is chosen by the value
 * distribution": each output channel (row of w, n x k, fp32/bf16, device)
 * is quantized under every candidate format (host array of ncand <= 8
 * mxq_fmt values, no Hadamard); its reconstruction error is the binary64
 * sum of squared differences from the exact dequantized values; the
 * channel keeps the candidate with the least error (ties to the lower
 * candidate index).  Tensor-scaled candidates use the tensor scale of the
 * whole w.
 *   fmt_per_channel: device uint8[n], the chosen mxq_fmt.
 *   sse: device double[n][ncand] or NULL.
 *   workspace: device scratch of mxq_select_workspace_bytes.
 * Constraints: k % 64 == 0. */
mxq_status mxq_select_weight_format(const void *w, int32_t wdtype, int64_t n, int64_t k,
                                    const int32_t *candidates, int32_t ncand,
                                    uint8_t *fmt_per_channel, double *sse, void *workspace,
                                    size_t workspace_bytes, void *stream);

/* Scratch bytes mxq_quantize_mse needs for a rows x cols tensor:
 * 256 + 16 * (rows * cols / 16) + 16 * rows + 16 * ceil(rows / 128). */
mxq_status mxq_quantize_mse_workspace_bytes(int64_t rows, int64_t cols, size_t *bytes);

/* NVFP4 quantization with the block and tensor scales fitted to the squared
 * error ("Bridging the Gap Between Promise and Performance for Microscaling
 * FP4 Quantization", MR-GPTQ modification 1: the grid is chosen for the MSE
 * by optimizing the per-block scales and the tensor scale in turn), meant
 * for weights, which are quantized once.
 *   Block step, s_t fixed: per 16-element block the E4M3 codes e0, e0 + 1,
 *     e0 - 1, ..., e0 - 6 (e0 = the usual code; codes in [1, 126]; for
 *     e0 = 0: 0, 1) are scored in that order by the binary64 sum, in element
 *     order, of (v - exact dequantized value)^2 with the elements coded as
 *     usual under each; the first least error wins.
 *   Tensor step, codes fixed: s_t = fp32(A / B), A = sum v u, B = sum u^2,
 *     u = E2M1 value x E4M3 value, binary64 sums within a block in element
 *     order, within a row in block order, over each group of 128
 *     consecutive rows in row order, over the groups in order; B = 0 keeps
 *     s_t.  The total error below is summed in the same order.
 *   Start from the usual s_t; `iters` >= 0 rounds of (block step, tensor
 *   step); a final block step writes codes and scales.
 * The result is the output layout of mxq_quantize for NVFP4 (codes,
 * scales, tensor_scale) and dequantizes with mxq_dequantize / feeds
 * mxq_qlinear unchanged.
 *   w: rows x cols fp32/bf16 device; fmt: MXQ_NVFP4 (others
 *     MXQ_EUNSUPPORTED); layout: MXQ_LAYOUT_CANONICAL or MXQ_LAYOUT_MMA.
 *   sse: device double receiving the total squared error of the result
 *     (same summation order), or NULL.
 *   workspace: device scratch of mxq_quantize_mse_workspace_bytes, 256-byte
 *     aligned; clobbered.
 * Constraints as mxq_quantize (cols % 16 == 0, 16-byte aligned w and
 * codes); rows * cols / 16 < 2^31.  Bit-identical from run to run.
 * Errors: MXQ_EINVAL (shape / pointer / iters < 0 / workspace alignment),
 * MXQ_EUNSUPPORTED (fmt), MXQ_ENOSPACE (workspace), MXQ_ECUDA. */
mxq_status mxq_quantize_mse(const void *w, int32_t wdtype, int64_t rows, int64_t cols, int32_t fmt,
                            int32_t iters, int32_t layout, void *codes, void *scales,
                            float *tensor_scale, double *sse, void *workspace,
                            size_t workspace_bytes, void *stream);

/* MX quantization with a fixed grid scale ("Bridging the Gap Between
 * Promise and Performance for Microscaling FP4 Quantization", MR-GPTQ
 * modification 1: for MXFP4 with Hadamard rotations one fixed grid scale
 * serves every model).  The grid scale g in [1, 2] scales the block amax
 * before the power-of-two exponent is taken: e = floor(log2 amax) +
 * [g m >= 2] - emax, m the significand of amax in [1, 2) (the product
 * exact); g = 1 is mxq_quantize's OCP rule, g = 4/3 the rule under which
 * E2M1 never clips.  Elements, scales and layouts as mxq_quantize.
 *   fmt: MXQ_MXFP4 or MXQ_MXFP8 (others MXQ_EUNSUPPORTED); g outside [1, 2]:
 *     MXQ_EINVAL.  Other arguments and constraints as mxq_quantize.
 * Errors: MXQ_EINVAL, MXQ_EUNSUPPORTED, MXQ_ECUDA. */
mxq_status mxq_quantize_mx_grid(const void *x, int32_t xdtype, int64_t rows, int64_t cols, int32_t fmt,
                                int32_t hadamard_b, float grid_scale, int32_t layout, void *codes,
                                void *scales, void *stream);

/* Scratch bytes mxq_fit_mx_grid needs for n candidates:
 * 256 + 8 * n * (rows * cols / 32) + 8 * rows + 8 * ceil(rows / 128). */
mxq_status mxq_fit_mx_grid_workspace_bytes(int64_t rows, int64_t cols, int32_t n, size_t *bytes);

/* Squared error of w (after the block-diagonal Hadamard rotation when
 * hadamard_b > 0) under mxq_quantize_mx_grid with each candidate grid
 * scale: sse[j] = sum (h - value(code) 2^e)^2 over the rotated tensor h, the
 * dequantized value exact in binary64, summed in binary64 in element order
 * within a block, in block order within a row, over each group of 128
 * consecutive rows in row order and over the groups in order (bit-identical
 * from run to run).  The least entry names the grid scale to fix.
 *   grid_scales: host float[n], 1 <= n <= 8, each in [1, 2].
 *   sse: device double[n].
 *   workspace: device scratch of mxq_fit_mx_grid_workspace_bytes, 256-byte
 *     aligned; clobbered.
 * Other arguments and constraints as mxq_quantize_mx_grid.
 * Errors: MXQ_EINVAL (shape / pointer / candidates / workspace alignment),
 * MXQ_EUNSUPPORTED (fmt), MXQ_ENOSPACE (workspace), MXQ_ECUDA. */
mxq_status mxq_fit_mx_grid(const void *w, int32_t wdtype, int64_t rows, int64_t cols, int32_t fmt,
                           int32_t hadamard_b, const float *grid_scales, int32_t n, double *sse,
                           void *workspace, size_t workspace_bytes, void *stream);

/* Activation-format calibration (Chameleon article, section "the format is
 * chosen by the value distribution": the trajectory is cut into ten
 * intervals, activations are calibrated in advance and the per-layer,
 * per-interval result is the table mxq_route reads).  The page gives no
 * decision rule; this library's reading mirrors its rule for weights: an
 * entry takes the candidate with the least squared quantization error
 * accumulated over the calibration activations of its layer and interval,
 * and the tail moments are accumulated beside it (excess kurtosis
 * n * sum x^4 / (sum x^2)^2 - 3 over n elements).
 *
 * mxq_calibrate_activation adds, for one calibration activation x
 * (rows x cols fp32/bf16, device): to sse_accum[j] (device double[ncand])
 * the squared error of x under candidate j as mxq_select_weight_format
 * measures it per row, the rows summed in binary64 over each group of 128
 * consecutive rows in order and then over the groups in order; to
 * moments_accum[0..1] (device double[2]) sum x^2 and sum x^4 in binary64
 * (element order within 16-element chunks, then chunks, rows, groups as
 * above).  Zero the accumulators before an entry's first activation.
 *   candidates: host array of 1..8 mxq_fmt values; cols % 64 == 0.
 *   workspace: device scratch of mxq_calibrate_workspace_bytes, 256-byte
 *     aligned; clobbered.
 * Errors: MXQ_EINVAL (shape / pointer / candidates / workspace alignment),
 * MXQ_ENOSPACE (workspace), MXQ_ECUDA. */
mxq_status mxq_calibrate_workspace_bytes(int64_t rows, int64_t cols, int32_t ncand, size_t *bytes);
mxq_status mxq_calibrate_activation(const void *x, int32_t xdtype, int64_t rows, int64_t cols,
                                    const int32_t *candidates, int32_t ncand, double *sse_accum,
                                    double *moments_accum, void *workspace, size_t workspace_bytes,
                                    void *stream);

/* Writes one table entry (device uint8): forced_fmt when >= 0 (layers the
 * article pins to MXFP8), else the candidate with the least sse_accum
 * (device double[ncand]), ties to the lower candidate index.
 * Errors: MXQ_EINVAL (pointers / candidates / forced_fmt), MXQ_ECUDA. */
mxq_status mxq_calibrate_pick(const double *sse_accum, const int32_t *candidates, int32_t ncand,
                              int32_t forced_fmt, uint8_t *entry, void *stream);

/* ---------------------------------------------------------------------- */
/* a5-a7: low-rank branch and block-scaled low-bit GEMM.                   */
/* ---------------------------------------------------------------------- */

/* SVDQuant low-rank down projection (Nunchaku/Diffusers article, "Main
 * explanation": a 16-bit low-rank part of the weight is kept beside the
 * 4-bit residual): t = bf16(x) . l1 with fp32 accumulation.
 *   x: m x k fp32/bf16 device; l1: k x r bf16 device; t: m x r fp32 device.
 * Constraints: 1 <= r <= 32, k % 16 == 0. */
mxq_status mxq_lowrank_down(const void *x, int32_t xdtype, int64_t m, int64_t k, const void *l1,
                            int32_t r, float *t, void *stream);

/* Bytes of the packed low-rank activation for m rows (m x 64 bf16). */
mxq_status mxq_lowrank_packed_bytes(int64_t m, size_t *bytes);

/* Packed low-rank activation, the operand mxq_qlinear reads:
 *   tp: m x 64 bf16 device; row i = [hi_0 .. hi_31, lo_0 .. lo_31] with
 *   u_j = t[i][j] / (xs * ws) rounded to fp32, hi_j = bf16(u_j),
 *   lo_j = bf16(u_j - hi_j), and zeros for j >= r.  xs, ws are the device
 *   tensor scales of the quantized activation and weight (NVFP4,
 *   FP8_TENSOR), both NULL for formats without one (then the divisor is 1).
 * The GEMM epilogue multiplies its accumulator by xs * ws, so the split
 * high/low product restores t . l2 to about 2^-16 relative.
 * mxq_lowrank_down_packed computes t as mxq_lowrank_down does and writes
 * tp directly; mxq_lowrank_pack_t packs a given t (m x r fp32 device). */
mxq_status mxq_lowrank_down_packed(const void *x, int32_t xdtype, int64_t m, int64_t k, const void *l1,
                                   int32_t r, const float *x_tensor_scale, const float *w_tensor_scale,
                                   void *tp, void *stream);
mxq_status mxq_lowrank_pack_t(const float *t, int32_t r, int64_t m, const float *x_tensor_scale,
                              const float *w_tensor_scale, void *tp, void *stream);

/* Scratch bytes mxq_quantize_lowrank needs for m rows and rank r. */
mxq_status mxq_quantize_lowrank_workspace_bytes(int64_t m, int32_t r, size_t *bytes);

/* Activation side of one W4A4 + low-rank linear in one call: quantizes x
 * (as mxq_quantize, MMA layout) and writes the packed low-rank operand tp
 * (as mxq_lowrank_down_packed with the new tensor scale of x and
 * w_tensor_scale).  For tensor-scaled formats without rotation the tensor
 * amax and t = bf16(x) . l1 come from one read of x, and the encoding pass
 * re-reads x from L2.
 *   fmt: NVFP4, MXFP4, MXFP8, FP8_TENSOR, INT4_G32 or INT4_G64 (the
 *     formats whose GEMM takes the branch; INT8_ROW gives
 *     MXQ_EUNSUPPORTED); w_tensor_scale: device scalar of the weight
 *     (NVFP4, FP8_TENSOR), else ignored.
 *   workspace: device scratch of mxq_quantize_lowrank_workspace_bytes,
 *     256-byte aligned; clobbered.
 * Other arguments, constraints and errors as mxq_quantize and
 * mxq_lowrank_down. */
mxq_status mxq_quantize_lowrank(const void *x, int32_t xdtype, int64_t m, int64_t k, int32_t fmt,
                                int32_t hadamard_b, const void *l1, int32_t r,
                                const float *w_tensor_scale, void *codes, void *scales,
                                float *tensor_scale, void *tp, void *workspace,
                                size_t workspace_bytes, void *stream);

/* Same as mxq_quantize_lowrank, but without a workspace argument: the
 * scratch it needs (the tensor-amax word and per-CTA maxima, and the m x r
 * fp32 low-rank activation, 4096 + 4*m*r bytes) lives in a 4 MiB array that the library
 * keeps in device memory, one per GPU that loads it, until the process
 * exits.  The pages describe no such call; it exists for callers that
 * cannot allocate device memory themselves: code embedded in a host
 * application that owns every device buffer and hands the library only its
 * inputs and outputs, and latency-bound callers for whom a cudaMalloc,
 * which may synchronize the device, is not acceptable.
 *   Limit: 4096 + 4*m*r <= 4 MiB (m*r <= 1,047,552, e.g. m <= 32,736 rows
 *     at rank 32); larger calls return MXQ_ENOSPACE and launch nothing.
 *   The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *   All calls share the array: calls whose work overlaps on the GPU (other
 *     streams, other host threads) race on it and must be ordered by the
 *     caller.  Every per-CTA maximum a call reads is written by that call,
 *     and a call that folds into the amax word clears it first: nothing in
 *     the array needs to start at zero.
 *   The call itself allocates and frees nothing.
 * Other arguments, results and errors as mxq_quantize_lowrank. */
mxq_status mxq_quantize_lowrank_noalloc(const void *x, int32_t xdtype, int64_t m, int64_t k,
                                        int32_t fmt, int32_t hadamard_b, const void *l1, int32_t r,
                                        const float *w_tensor_scale, void *codes, void *scales,
                                        float *tensor_scale, void *tp, void *stream);

/* Scratch bytes mxq_qlinear_w4a16 can use for an m x k activation and an
 * n x k weight: n * k * 2 (the unpacked bf16 weight) when m >= 512, where
 * unpacking the weight once per call costs less than converting it in
 * every 128-row tile of x; else 0. */
mxq_status mxq_qlinear_w4a16_workspace_bytes(int64_t m, int64_t n, int64_t k, size_t *bytes);

/* W4A16 linear (Nunchaku/Diffusers article, awq_w4a16: 4-bit per-group
 * weights against 16-bit activations): y = bf16(x) . W16^T with
 * W16 = bf16(RN32(q s)), q the signed INT4 code and s its group's fp32
 * scale, fp32 accumulation on tcgen05 tensor cores.  Two routes, the same
 * products:
 *   - workspace of at least mxq_qlinear_w4a16_workspace_bytes (> 0): W16 is
 *     written once into the workspace (mxq_dequantize's kernel) and a bf16
 *     kind::f16 GEMM (the block-scaled GEMM's bf16 variant) multiplies it;
 *   - otherwise (workspace NULL or the query 0): the weights are dequantized
 *     in shared memory, stage by stage, by the converter warps of one fused
 *     kernel, never written out (the memory-light route for small m).
 *   x: m x k bf16 device (16-byte aligned); wq: INT4_G32 or INT4_G64 in the
 *   canonical layout (mxq_quantize), wq->cols == k; y: m x wq->rows device,
 *   ydtype MXQ_BF16 or MXQ_F32; workspace: device, 16-byte aligned, or NULL.
 * Constraints: k % 64 == 0; ceil(m/128) * ceil(n/128) * k/64 < 2^31.
 * Errors: MXQ_EINVAL (shape / layout / pointer / ydtype), MXQ_EUNSUPPORTED
 * (formats other than INT4_G32 / INT4_G64), MXQ_ECUDA; a pipeline wait that
 * runs out is reported by mxq_check(). */
mxq_status mxq_qlinear_w4a16(const void *x, int64_t m, int64_t k, const mxq_qtensor *wq, void *y,
                             int32_t ydtype, void *workspace, size_t workspace_bytes, void *stream);

/* Re-lays the up-projection l2 (r x n bf16, device) as the GEMM operand
 * l2p (n x 64 bf16, device): row j of l2p holds l2[0..r-1][j], zeros up to
 * 32, then the same 32 values again (the operand of the split high/low
 * low-rank product).  Done once per weight. */
mxq_status mxq_lowrank_pack_l2(const void *l2, int32_t r, int64_t n, void *l2p, void *stream);

/* Block-scaled low-bit GEMM with fused dequantization epilogue and
 * low-rank branch (Nunchaku/Diffusers article, svdq_w4a4; Chameleon
 * article, W8A8 formats), one kernel launch:
 *   y[m][n] = sum_k deq(xq)[m][k] * deq(wq)[n][k]  (+ sum_j t[m][j] * l2[j][n])
 * on tcgen05 tensor cores (fp32 accumulation; int32 for INT8_ROW), the
 * per-block scales applied by the tensor cores, tensor / row scales in the
 * epilogue.  INT4_G32 / INT4_G64 (fp32 group scales, which the tensor
 * cores cannot apply) form each group's exact integer dot product on the
 * tensor cores and add it, times sx * sw, to fp32 sums in the epilogue.
 *   xq, wq: same fmt, MMA layout, xq->cols == wq->cols == K.
 *     Supported fmt: NVFP4, MXFP4, MXFP8, FP8_TENSOR, INT8_ROW, INT4_G32,
 *     INT4_G64.
 *   tp: packed low-rank activation (m x 64 bf16, from
 *     mxq_lowrank_down_packed / mxq_lowrank_pack_t with the same tensor
 *     scales as xq, wq) or NULL for no branch; l2p: packed up-projection
 *     (n rows).  The branch is supported for every fmt but INT8_ROW.
 *   y: m x n device, fp32 or bf16 (fp32 result rounded once, RNE).
 * Constraints: K % 64 == 0 (NVFP4, MXFP4), K % g == 0 (INT4_Gg) or
 * K % 32 == 0 (8-bit); K > 0; ceil(m/128) * ceil(n/128) * K/16 < 2^31;
 * device pointers 16-byte aligned.
 * Errors: MXQ_EINVAL, MXQ_EUNSUPPORTED (format pair / branch), MXQ_ECUDA.
 * A pipeline wait that runs out is reported by mxq_check(). */
mxq_status mxq_qlinear(const mxq_qtensor *xq, const mxq_qtensor *wq, const void *tp, const void *l2p,
                       void *y, int32_t ydtype, void *stream);

/* ---------------------------------------------------------------------- */
/* Per-channel mixed weight formats against MXFP8 activations.             */
/* ---------------------------------------------------------------------- */

/* A weight whose output channels keep the formats mxq_select_weight_format
 * chose for them among MXFP4, INT4_G32 and NVFP4 (Chameleon article, section
 * "the format is chosen by the value distribution"), laid out for the
 * tensor cores as three groups of rows -- group 0 MXFP4, group 1 INT4_G32,
 * group 2 NVFP4, each in channel order:
 *   rows, cols: N output channels, K inputs (K % 32 == 0).
 *   n_group[g]: channels in group g.
 *   choice: device uint8[N], each channel's format; group_index: device
 *     int32[N], each channel's row within its group (from mxq_mixed_plan).
 *   mx_codes: device n_group[0] x K bytes, the E4M3 encoding of each E2M1
 *     code (exact; zero as +0); mx_scales: their E8M0 block scales in the MMA
 *     layout of mxq_quantize (n_group[0] rows).
 *   i4_codes: device n_group[1] x K bytes, the E4M3 encoding of each integer
 *     code; i4_scales: device fp32 [K/32][n_group[1]] group scales.
 *   nv_values: device bf16 n_group[2] x K, each E2M1 code value times its
 *     E4M3 block scale (exact in bf16); nv_tensor_scale: device fp32, the
 *     NVFP4 tensor scale, that of the whole weight as in the selection.
 * Buffers with a zero count may be NULL. */
typedef struct mxq_mixed_weight {
    int64_t rows, cols;
    int64_t n_group[3];
    const uint8_t *choice;
    const int32_t *group_index;
    void *mx_codes;
    void *mx_scales;
    void *i4_codes;
    float *i4_scales;
    void *nv_values;
    const float *nv_tensor_scale;
} mxq_mixed_weight;

/* Host only: the grouping of channels by their chosen format.
 *   choice: host uint8[n] of MXQ_MXFP4 / MXQ_INT4_G32 / MXQ_NVFP4.
 *   n_group: host int64[3] receiving the group sizes; group_index: host
 *     int32[n] receiving each channel's row within its group (channels keep
 *     their order inside a group).
 * Errors: MXQ_EINVAL (a format outside the three, n < 0 or >= 2^31, null). */
mxq_status mxq_mixed_plan(const uint8_t *choice, int64_t n, int64_t n_group[3], int32_t *group_index);

/* Host only: bytes of the five group buffers of mxq_mixed_weight, in the
 * order mx_codes, mx_scales, i4_codes, i4_scales, nv_values. */
mxq_status mxq_mixed_weight_bytes(const int64_t n_group[3], int64_t k, size_t bytes[5]);

/* Lays the weight out as mxq_mixed_weight from its quantization in each of
 * the three formats.
 *   w_mxfp4, w_int4, w_nvfp4: the WHOLE weight (N x K) quantized by
 *     mxq_quantize in MXQ_MXFP4, MXQ_INT4_G32 and MXQ_NVFP4, canonical layout.
 *   out: rows, cols, n_group, choice, group_index filled by the caller (from
 *     mxq_mixed_plan, choice and group_index copied to the device), the group
 *     buffers allocated with mxq_mixed_weight_bytes; they are written here
 *     (nv_tensor_scale may point at w_nvfp4->tensor_scale).
 * Errors: MXQ_EINVAL (shapes, formats, layouts, pointers), MXQ_ECUDA. */
mxq_status mxq_mixed_prepare(const mxq_qtensor *w_mxfp4, const mxq_qtensor *w_int4, const mxq_qtensor *w_nvfp4,
                             const mxq_mixed_weight *out, void *stream);

/* Scratch bytes mxq_qlinear_mixed needs for m activation rows: the
 * activation's block scales as fp32 (INT4 group), the activation dequantized
 * to bf16 (NVFP4 group) and one m x n_group[g] output per group (none when
 * one group holds every channel), each at a 256-byte boundary. */
mxq_status mxq_qlinear_mixed_workspace_bytes(int64_t m, const mxq_mixed_weight *w, int32_t ydtype, size_t *bytes);

/* y = deq(xq) . deq_f(W)^T, each output channel n dequantized in its own
 * format f = choice[n]: the MXFP4 group on kind::mxf8f6f4 block-scaled MMAs
 * against the MXFP8 codes, the INT4_G32 group on the group GEMM of
 * mxq_qlinear (each 32-element product of codes times the activation's 2^e
 * and the weight's group scale), the NVFP4 group on bf16 kind::f16 MMAs
 * against the activation dequantized to bf16 (exact while the block
 * exponents stay inside the bf16 range), times the tensor scale; then the
 * group outputs are scattered to channel order (when one group holds every
 * channel, its GEMM writes y directly: channel n is row n of the group, as
 * mxq_mixed_plan numbers them).  fp32 accumulation.
 *   xq: MXQ_MXFP8, MMA layout, cols == w->cols.
 *   y: m x N device, ydtype MXQ_BF16 or MXQ_F32.
 *   workspace: device scratch of mxq_qlinear_mixed_workspace_bytes,
 *     256-byte aligned; clobbered.
 * Errors: MXQ_EINVAL, MXQ_ENOSPACE, MXQ_ECUDA; a pipeline wait that runs out
 * is reported by mxq_check(). */
mxq_status mxq_qlinear_mixed(const mxq_qtensor *xq, const mxq_mixed_weight *w, void *y, int32_t ydtype,
                             void *workspace, size_t workspace_bytes, void *stream);

/* ---------------------------------------------------------------------- */
/* a8: per-layer, per-timestep-interval format table.                      */
/* ---------------------------------------------------------------------- */

/* Chameleon article: the denoising trajectory is cut into intervals and a
 * layer reads its activation format for the current interval from a table
 * at generation time.  table: host uint8[n_layers][n_intervals] of mxq_fmt;
 * interval = floor(step * n_intervals / n_steps).  Returns the format, or
 * -1 for out-of-range arguments.  Host only, no CUDA call. */
int32_t mxq_route(const uint8_t *table, int32_t n_layers, int32_t n_intervals, int32_t layer,
                  int32_t step, int32_t n_steps);

/* One linear layer prepared for routed execution: its weight quantized
 * once, in the MMA layout, in every format its row of the format table can
 * name, and the optional low-rank branch.
 *   w[f]: the weight (N x K) in format f (w[f].fmt == f, layout MMA), or
 *     w[f].codes == NULL when the layer is never routed to f.  All prepared
 *     entries have the same rows (N) and cols (K).
 *   l1: K x r bf16 device, the down projection (NULL: no branch, r = 0);
 *   l2p: the packed up projection (mxq_lowrank_pack_l2, N rows).
 *   hadamard_b: 0, or the block-diagonal rotation size the weights were
 *     quantized with; the activation is rotated the same way. */
typedef struct mxq_layer {
    mxq_qtensor w[MXQ_NUM_FMT];
    const void *l1;
    const void *l2p;
    int32_t r;
    int32_t hadamard_b;
} mxq_layer;

/* Scratch bytes mxq_qlinear_routed needs for an m x k activation and rank
 * r (0 without branch): the quantized activation in the largest format,
 * its scales and tensor scale, the low-rank operands and the tensor-amax
 * words, each at a 256-byte boundary. */
mxq_status mxq_qlinear_routed_workspace_bytes(int64_t m, int64_t k, int32_t r, size_t *bytes);

/* The routed quantized linear layer (Chameleon article, sections "the format
 * is chosen by the value distribution" and "calibration, not acceleration,
 * is planned": the trajectory is cut into intervals, and at generation time
 * each layer reads the activation format of the current interval from a
 * table computed in advance; Nunchaku/Diffusers article: the low-rank
 * branch beside the low-bit residual).  One call:
 *   fmt = fmt_table[layer][floor(step * n_intervals / n_steps)]  (host read,
 *     as mxq_route),
 *   xq  = x quantized in fmt (MMA layout; after the rotation when
 *     layer_w->hadamard_b > 0), into the workspace,
 *   y   = deq(xq) . deq(layer_w->w[fmt])^T (+ (bf16(x) . l1) . l2)
 * with the kernels of mxq_quantize / mxq_quantize_lowrank and mxq_qlinear.
 *   x: m x k fp32/bf16 device, 16-byte aligned; k == the weights' cols.
 *   fmt_table: host uint8[n_layers][n_intervals] of mxq_fmt.
 *   y: m x N device, ydtype MXQ_BF16 or MXQ_F32.
 *   fmt_used: host int32 receiving the routed format, or NULL.
 *   workspace: device scratch of mxq_qlinear_routed_workspace_bytes(m, k,
 *     layer_w->r), 256-byte aligned; clobbered.
 * Errors: MXQ_EINVAL (table arguments out of range, as mxq_route; the
 * weight not prepared in the routed format; shapes, pointers, workspace
 * alignment), MXQ_ENOSPACE (workspace), MXQ_EUNSUPPORTED (a branch with an
 * INT8_ROW entry), MXQ_ECUDA; the argument rules of mxq_quantize and
 * mxq_qlinear apply.  Everything but the table read runs asynchronously on
 * `stream`. */
mxq_status mxq_qlinear_routed(const void *x, int32_t xdtype, int64_t m, int64_t k, const mxq_layer *layer_w,
                              const uint8_t *fmt_table, int32_t n_layers, int32_t n_intervals, int32_t layer,
                              int32_t step, int32_t n_steps, void *y, int32_t ydtype, int32_t *fmt_used,
                              void *workspace, size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MXQ_H */
