/*
 * mxq_oracle.c -- plain, slow, scalar CPU oracle for the microscaling
 * quantized-linear hot path.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The CUDA library
 * never includes, links or calls it, and it includes nothing from the CUDA
 * sources: the two implementations are written independently and compared.
 *
 * What the pages fix, and what this file takes from elsewhere:
 *  - The formats are named by the pages (MXFP8 with small blocks sharing an
 *    exponent: Chameleon article, section "the format is chosen by the value
 *    distribution"; INT4 and NVFP4 variants of svdq_w4a4: Nunchaku/Diffusers
 *    article, section "Kernels and supported hardware"; NVFP4's small groups
 *    and MXFP4's power-of-two scales: "Bridging the Gap Between Promise and
 *    Performance for Microscaling FP4 Quantization", failure modes 1-2).
 *    None of the pages gives the bit layouts, so the element and scale
 *    encodings follow the published OCP Microscaling (MX) v1.0 definition
 *    (E2M1, E4M3 "fn", E8M0, 32-element blocks) and NVIDIA's NVFP4
 *    definition (E2M1 in 16-element blocks, E4M3 block scale, fp32 tensor
 *    scale).
 *  - Every point those definitions leave open is a stated reading; each
 *    function says which one it takes.
 *
 * Arithmetic: C11, IEEE binary32 for every fp32 step (x86-64 SSE, no x87),
 * compiled with -ffp-contract=off so no multiply-add is fused, and without
 * -ffast-math so subnormals are kept.  Mini-float rounding is done by
 * nearest-neighbour search over the decoded code table with exact (binary64)
 * midpoint comparisons, ties going to the code whose least significant bit
 * is 0 (round-half-to-even).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* Format identifiers (must agree, by value, with the library's public enum;
 * the Python test layer maps both by name). */
enum {
    ORC_MXFP8 = 0,      /* E4M3 elements, 32-element blocks, E8M0 scale      */
    ORC_MXFP4 = 1,      /* E2M1 elements, 32-element blocks, E8M0 scale      */
    ORC_NVFP4 = 2,      /* E2M1 elements, 16-element blocks, E4M3 scale + fp32 tensor scale */
    ORC_INT4_G32 = 3,   /* symmetric int4 in [-7,7], fp32 scale per 32      */
    ORC_INT4_G64 = 4,   /* symmetric int4 in [-7,7], fp32 scale per 64      */
    ORC_INT8_ROW = 5,   /* symmetric int8 in [-127,127], fp32 scale per row */
    ORC_FP8_TENSOR = 6, /* E4M3 elements, one fp32 scale for the tensor     */
    ORC_NUM_FMT = 7
};

enum { ORC_OK = 0, ORC_EINVAL = 1 };

static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* ------------------------------------------------------------------ */
/* Element codecs (OCP MX v1.0 element tables).                        */
/* ------------------------------------------------------------------ */

/* E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0; no Inf/NaN.
 * Magnitudes by code 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
double orc_e2m1_value(uint8_t code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* E4M3 ("fn" variant): sign bit 7, exponent bits 6..3 (bias 7), mantissa
 * bits 2..0; exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; there
 * is no infinity.  Largest finite magnitude 448, smallest 2^-9. */
double orc_e4m3_value(uint8_t code)
{
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* E8M0: unsigned power of two 2^(b-127); 0xFF is NaN. */
double orc_e8m0_value(uint8_t b)
{
    return b == 255 ? NAN : ldexp(1.0, (int)b - 127);
}

static double e4m3_mag[127];   /* magnitudes of codes 0x00..0x7E, ascending */
static double e2m1_mag[8];
static int tables_ready = 0;

static void init_tables(void)
{
    if (tables_ready) return;
    for (int c = 0; c < 127; c++) e4m3_mag[c] = orc_e4m3_value((uint8_t)c);
    for (int c = 0; c < 8; c++) e2m1_mag[c] = orc_e2m1_value((uint8_t)c);
    tables_ready = 1;
}

/* Nearest magnitude code to |v| in an ascending table of n magnitudes.
 * Values past the largest magnitude saturate to it (the "satfinite"
 * reading: no overflow to NaN).  Exact ties go to the even code. */
static int nearest_code(double a, const double *mag, int n)
{
    if (a >= mag[n - 1]) return n - 1;
    int lo = 0, hi = n - 1;                 /* mag[lo] <= a < mag[hi] */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (mag[mid] <= a) lo = mid; else hi = mid;
    }
    double midpoint = 0.5 * (mag[lo] + mag[hi]);  /* exact in binary64 */
    if (a < midpoint) return lo;
    if (a > midpoint) return hi;
    return (lo & 1) ? hi : lo;
}

/* fp32 -> E4M3, round-to-nearest-even, saturating to +-448.
 * Reading: the sign of a value that rounds to zero is kept (IEEE style);
 * NaN becomes 0x7F. */
uint8_t orc_to_e4m3(float v)
{
    init_tables();
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0;
    return (uint8_t)(sign | nearest_code(fabs((double)v), e4m3_mag, 127));
}

/* fp32 -> E2M1 (4-bit code in the low nibble), round-to-nearest-even,
 * saturating to +-6, sign of zero kept.  NaN has no E2M1 code; it maps to
 * +6 here (the oracle's callers reject non-finite input beforehand). */
uint8_t orc_to_e2m1(float v)
{
    init_tables();
    if (isnan(v)) return 0x7;
    uint8_t sign = signbit(v) ? 0x8 : 0;
    return (uint8_t)(sign | nearest_code(fabs((double)v), e2m1_mag, 8));
}

/* Round half to even to an integer (|v| < 2^30). */
static int32_t rne_int(float v)
{
    double d = (double)v, f = floor(d), r = d - f;   /* both exact */
    if (r > 0.5 || (r == 0.5 && fmod(f, 2.0) != 0.0)) f += 1.0;
    return (int32_t)f;
}

/* floor(log2(a)) for finite a > 0, read from the binary32 fields
 * (subnormals normalised). */
static int floor_log2_f32(float a)
{
    uint32_t u = f2u(a);
    int e = (int)((u >> 23) & 0xFF);
    uint32_t m = u & 0x7FFFFF;
    if (e != 0) return e - 127;
    int p = 22;
    while (p >= 0 && !((m >> p) & 1u)) p--;
    return p - 149;
}

/* fp32 -> bf16 -> fp32, round-to-nearest-even (finite inputs). */
float orc_round_bf16(float v)
{
    uint32_t u = f2u(v);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return u2f(u & 0xFFFF0000u);
}

/* Bulk conversion of a range of binary32 bit patterns, for the exhaustive
 * codec test.  elem 0: E4M3 byte; elem 1: E2M1 code in the low nibble. */
void orc_cast_range(uint32_t first_bits, int64_t count, int elem, uint8_t *out)
{
    init_tables();
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; i++) {
        float v = u2f(first_bits + (uint32_t)i);
        out[i] = elem == 0 ? orc_to_e4m3(v) : orc_to_e2m1(v);
    }
}

/* ------------------------------------------------------------------ */
/* Block-diagonal Hadamard rotation.                                   */
/* "Bridging the Gap ... Microscaling FP4 Quantization", item 3:       */
/* activations (and, to keep X.W^T unchanged, weights) are rotated by  */
/* block-diagonal Hadamard matrices along K.                           */
/* Reading: orthonormal Sylvester matrix H_b = H_2 (x) ... (x) H_2,    */
/* applied as log2(b) butterfly stages in fp32, stage j pairing        */
/* elements i and i+2^j for every i whose bit j is 0 into (a+c, a-c),  */
/* then one fp32 multiply by RN_f32(1/sqrt(b)).                        */
/* ------------------------------------------------------------------ */

float orc_hadamard_norm(int b)
{
    int lg = 0;
    while ((1 << lg) < b) lg++;
    /* b = 2^lg; 1/sqrt(b) = 2^(-lg/2), times sqrt(1/2) when lg is odd. */
    double v = ldexp(1.0, -(lg / 2));
    if (lg & 1) v *= sqrt(0.5);
    return (float)v;
}

static void fwht_block(float *x, int b, float norm)
{
    for (int h = 1; h < b; h <<= 1)
        for (int i = 0; i < b; i++)
            if (!(i & h)) {
                float a = x[i], c = x[i + h];
                x[i] = a + c;
                x[i + h] = a - c;
            }
    for (int i = 0; i < b; i++) x[i] = x[i] * norm;
}

static int valid_hadamard_b(int b)
{
    return b >= 2 && b <= 256 && (b & (b - 1)) == 0;
}

int orc_hadamard(const float *x, float *y, int64_t rows, int64_t cols, int b)
{
    if (!valid_hadamard_b(b) || cols % b) return ORC_EINVAL;
    float norm = orc_hadamard_norm(b);
    memmove(y, x, (size_t)(rows * cols) * sizeof(float));
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c += b) fwht_block(y + r * cols + c, b, norm);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Quantizers.                                                         */
/* Codes: 4-bit formats pack two per byte, element 2i in the low       */
/* nibble; 8-bit formats one byte per element.  Scales row-major:      */
/*   MXFP8/MXFP4  uint8 E8M0  [rows][cols/32]                          */
/*   NVFP4        uint8 E4M3  [rows][cols/16]  + fp32 tensor scale     */
/*   INT4_G32/64  fp32        [rows][cols/g]                           */
/*   INT8_ROW     fp32        [rows]                                   */
/*   FP8_TENSOR   (none)                   + fp32 tensor scale         */
/* ------------------------------------------------------------------ */

static int fmt_block(int fmt)
{
    switch (fmt) {
    case ORC_MXFP8: case ORC_MXFP4: case ORC_INT4_G32: return 32;
    case ORC_NVFP4: return 16;
    case ORC_INT4_G64: return 64;
    default: return 0;   /* row / tensor scaled */
    }
}

static int fmt_is_4bit(int fmt)
{
    return fmt == ORC_MXFP4 || fmt == ORC_NVFP4 || fmt == ORC_INT4_G32 || fmt == ORC_INT4_G64;
}

static void put_code(uint8_t *codes, int64_t idx, int is4, uint8_t code)
{
    if (!is4) { codes[idx] = code; return; }
    uint8_t *p = codes + idx / 2;
    if (idx & 1) *p = (uint8_t)((*p & 0x0F) | (code << 4));
    else *p = (uint8_t)((*p & 0xF0) | (code & 0x0F));
}

static uint8_t get_code(const uint8_t *codes, int64_t idx, int is4)
{
    if (!is4) return codes[idx];
    uint8_t b = codes[idx / 2];
    return (idx & 1) ? (uint8_t)(b >> 4) : (uint8_t)(b & 0x0F);
}

static float amax_of(const float *v, int64_t n)
{
    float m = 0.0f;
    for (int64_t i = 0; i < n; i++) {
        float a = fabsf(v[i]);
        if (a > m) m = a;
    }
    return m;
}

/* MX block (OCP MX v1.0 shared-scale rule): X = 2^(floor(log2 amax) - emax)
 * with emax the element format's largest exponent (8 for E4M3, 2 for E2M1),
 * clamped to the E8M0 range [-127, 127]; element = RNE_sat(v / X), the
 * division by a power of two done as an fp32 multiply by 2^-e.
 * Reading: an all-zero block gets scale byte 127 (X = 1) and +0 codes. */
/* g: grid scale (see orc_quantize_mx_grid); 1 gives the OCP rule. */
static void quant_mx_block(const float *v, int n, int fp4, float g, uint8_t *codes, int64_t base,
                           uint8_t *scale)
{
    float amax = amax_of(v, n);
    if (amax == 0.0f) {
        *scale = 127;
        for (int i = 0; i < n; i++) put_code(codes, base + i, fp4, 0);
        return;
    }
    int fl = floor_log2_f32(amax);
    double m = ldexp((double)amax, -fl);               /* significand in [1, 2), exact */
    int e = fl + ((double)g * m >= 2.0 ? 1 : 0) - (fp4 ? 2 : 8);   /* product exact */
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    *scale = (uint8_t)(e + 127);
    float inv = (float)ldexp(1.0, -e);          /* 2^-e, exact in binary32 */
    for (int i = 0; i < n; i++) {
        float t = v[i] * inv;
        put_code(codes, base + i, fp4, fp4 ? orc_to_e2m1(t) : orc_to_e4m3(t));
    }
}

/* NVFP4 tensor scale s_t = RN(amax_T / (6 * 448)), so that the largest
 * block scale lands at the top of the E4M3 range.
 * Reading: when amax_T / 2688 is zero in fp32 (all-zero or vanishingly
 * small tensor), s_t = 1. */
static float nvfp4_tensor_scale(float amax_t)
{
    float s = amax_t / 2688.0f;
    return s == 0.0f ? 1.0f : s;
}

/* NVFP4 block: block scale e4 = E4M3(RN(RN(amax_b / 6) / s_t)); decode
 * scale d = RN(value(e4) * s_t); element = E2M1(RN(v / d)).
 * Reading: e4 == 0 gives +0 codes. */
static void quant_nvfp4_block(const float *v, float s_t, uint8_t *codes, int64_t base,
                              uint8_t *scale)
{
    float amax = amax_of(v, 16);
    float raw = (amax / 6.0f) / s_t;
    uint8_t e4 = orc_to_e4m3(raw);
    *scale = e4;
    if (e4 == 0) {
        for (int i = 0; i < 16; i++) put_code(codes, base + i, 1, 0);
        return;
    }
    float d = (float)orc_e4m3_value(e4) * s_t;
    for (int i = 0; i < 16; i++) put_code(codes, base + i, 1, orc_to_e2m1(v[i] / d));
}

/* Symmetric integer block with fp32 scale s = RN(amax / qmax);
 * q = clamp(RNE(RN(v / s)), -qmax, qmax).  Reading: s == 0 gives zero codes.
 * INT4 stores q as a two's-complement nibble (-8 is never produced). */
static void quant_int_block(const float *v, int64_t n, int qmax, int is4, uint8_t *codes,
                            int64_t base, float *scale)
{
    float s = amax_of(v, n) / (float)qmax;
    *scale = s;
    for (int64_t i = 0; i < n; i++) {
        int32_t q = 0;
        if (s != 0.0f) {
            q = rne_int(v[i] / s);
            if (q > qmax) q = qmax;
            if (q < -qmax) q = -qmax;
        }
        put_code(codes, base + i, is4, (uint8_t)(is4 ? (q & 0xF) : (q & 0xFF)));
    }
}

/* FP8 E4M3 with one tensor scale s = RN(amax_T / 448) (dynamic per-tensor
 * scale); element = E4M3(RN(v / s)).  Reading: s == 0 becomes 1. */
static float fp8_tensor_scale(float amax_t)
{
    float s = amax_t / 448.0f;
    return s == 0.0f ? 1.0f : s;
}

static int all_finite(const float *x, int64_t n)
{
    for (int64_t i = 0; i < n; i++)
        if (!isfinite(x[i])) return 0;
    return 1;
}

/* Quantize rows x cols of x (optionally Hadamard-rotated first, b = 0 for
 * none).  See the layout table above. */
int orc_quantize(const float *x, int64_t rows, int64_t cols, int fmt, int hadamard_b,
                 float *work /* rows*cols floats when hadamard_b != 0, else unused */,
                 uint8_t *codes, void *scales, float *tensor_scale)
{
    init_tables();
    if (fmt < 0 || fmt >= ORC_NUM_FMT || rows < 0 || cols < 0) return ORC_EINVAL;
    int blk = fmt_block(fmt);
    if (blk && cols % blk) return ORC_EINVAL;
    if (fmt_is_4bit(fmt) && cols % 2) return ORC_EINVAL;
    if (!all_finite(x, rows * cols)) return ORC_EINVAL;
    const float *src = x;
    if (hadamard_b) {
        if (orc_hadamard(x, work, rows, cols, hadamard_b) != ORC_OK) return ORC_EINVAL;
        src = work;
    }
    int is4 = fmt_is_4bit(fmt);
    if (fmt == ORC_NVFP4 || fmt == ORC_FP8_TENSOR) {
        float amax_t = amax_of(src, rows * cols);
        float s = fmt == ORC_NVFP4 ? nvfp4_tensor_scale(amax_t) : fp8_tensor_scale(amax_t);
        *tensor_scale = s;
        if (fmt == ORC_FP8_TENSOR) {
            for (int64_t i = 0; i < rows * cols; i++) put_code(codes, i, 0, orc_to_e4m3(src[i] / s));
            return ORC_OK;
        }
    }
    for (int64_t r = 0; r < rows; r++) {
        const float *row = src + r * cols;
        int64_t base = r * cols;
        switch (fmt) {
        case ORC_MXFP8:
        case ORC_MXFP4:
            for (int64_t c = 0; c < cols; c += 32)
                quant_mx_block(row + c, 32, fmt == ORC_MXFP4, 1.0f, codes, base + c,
                               (uint8_t *)scales + r * (cols / 32) + c / 32);
            break;
        case ORC_NVFP4:
            for (int64_t c = 0; c < cols; c += 16)
                quant_nvfp4_block(row + c, *tensor_scale, codes, base + c,
                                  (uint8_t *)scales + r * (cols / 16) + c / 16);
            break;
        case ORC_INT4_G32:
        case ORC_INT4_G64:
            for (int64_t c = 0; c < cols; c += blk)
                quant_int_block(row + c, blk, 7, 1, codes, base + c,
                                (float *)scales + r * (cols / blk) + c / blk);
            break;
        case ORC_INT8_ROW:
            quant_int_block(row, cols, 127, 0, codes, base, (float *)scales + r);
            break;
        }
    }
    (void)is4;
    return ORC_OK;
}

/* Exact dequantized values in binary64 (every format's code x scale
 * product is exact in 53 bits). */
int orc_dequantize(const uint8_t *codes, const void *scales, const float *tensor_scale,
                   int64_t rows, int64_t cols, int fmt, double *out)
{
    init_tables();
    if (fmt < 0 || fmt >= ORC_NUM_FMT) return ORC_EINVAL;
    int blk = fmt_block(fmt), is4 = fmt_is_4bit(fmt);
    if (blk && cols % blk) return ORC_EINVAL;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c++) {
            int64_t i = r * cols + c;
            uint8_t q = get_code(codes, i, is4);
            double v = 0.0;
            switch (fmt) {
            case ORC_MXFP8:
                v = orc_e4m3_value(q) * orc_e8m0_value(((const uint8_t *)scales)[r * (cols / 32) + c / 32]);
                break;
            case ORC_MXFP4:
                v = orc_e2m1_value(q) * orc_e8m0_value(((const uint8_t *)scales)[r * (cols / 32) + c / 32]);
                break;
            case ORC_NVFP4:
                v = orc_e2m1_value(q) * orc_e4m3_value(((const uint8_t *)scales)[r * (cols / 16) + c / 16]) *
                    (double)*tensor_scale;
                break;
            case ORC_INT4_G32:
            case ORC_INT4_G64: {
                int qi = (q & 0x8) ? (int)q - 16 : (int)q;
                v = qi * (double)((const float *)scales)[r * (cols / blk) + c / blk];
                break;
            }
            case ORC_INT8_ROW:
                v = (int8_t)q * (double)((const float *)scales)[r];
                break;
            case ORC_FP8_TENSOR:
                v = orc_e4m3_value(q) * (double)*tensor_scale;
                break;
            }
            out[i] = v;
        }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Per-output-channel format choice (Chameleon article, section "the   */
/* format is chosen by the value distribution": weights do not depend  */
/* on the denoising step, so each output channel tries the available   */
/* formats and keeps the one with the least reconstruction error).     */
/* Reading: error = sum over the row of (w - w_hat)^2 in binary64, in  */
/* index order, w_hat the exact dequantized value; formats with tensor */
/* scales take them from the whole W; ties go to the lower candidate   */
/* index.  Output: the chosen format id per row, and optionally the    */
/* row x candidate error matrix.                                       */
/* ------------------------------------------------------------------ */

int orc_select(const float *w, int64_t n, int64_t k, const int *cands, int ncand,
               uint8_t *codes_work /* n*k bytes */, void *scales_work /* n*k*4 bytes */,
               double *deq_work /* n*k doubles */, uint8_t *choice, double *sse)
{
    if (ncand < 1) return ORC_EINVAL;
    for (int ci = 0; ci < ncand; ci++) {
        float ts = 0.0f;
        int st = orc_quantize(w, n, k, cands[ci], 0, 0, codes_work, scales_work, &ts);
        if (st != ORC_OK) return st;
        orc_dequantize(codes_work, scales_work, &ts, n, k, cands[ci], deq_work);
        for (int64_t r = 0; r < n; r++) {
            double acc = 0.0;
            for (int64_t c = 0; c < k; c++) {
                double d = (double)w[r * k + c] - deq_work[r * k + c];
                acc += d * d;
            }
            sse[r * ncand + ci] = acc;
        }
    }
    for (int64_t r = 0; r < n; r++) {
        int best = 0;
        for (int ci = 1; ci < ncand; ci++)
            if (sse[r * ncand + ci] < sse[r * ncand + best]) best = ci;
        choice[r] = (uint8_t)cands[best];
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* NVFP4 scales fitted to the squared error ("Bridging the Gap Between */
/* Promise and Performance for Microscaling FP4 Quantization", MR-GPTQ */
/* modification 1: the quantization grid is chosen for the MSE by      */
/* optimizing the per-block scales and the tensor scale in turn; the   */
/* page reports the gain for NVFP4 without rotations).  The page gives */
/* no candidate set, round count or summation order; the readings:     */
/*  - Block step (tensor scale s_t fixed).  e0 = the usual block code   */
/*    (quant_nvfp4_block).  Candidates, scored in this order: e0, then  */
/*    e0 + 1, e0 - 1, e0 - 2, ..., e0 - 6, keeping codes in [1, 126]    */
/*    (for e0 = 0: 0 then 1).  A candidate e codes the block as usual   */
/*    under it: d = RN(value(e) s_t), q_i = E2M1(RN(v_i / d)) (e = 0:   */
/*    all +0).  Its error is sum_i (v_i - value(q_i) value(e) s_t)^2    */
/*    with the dequantized value exact in binary64 and the sum taken    */
/*    in binary64 in element order.  The first least error wins.        */
/*  - Tensor step (block codes fixed).  Least squares for the common    */
/*    factor: s_t = RN32(RN64(A / B)), A = sum v_i u_i, B = sum u_i^2,  */
/*    u_i = value(q_i) value(e); binary64 sums within a block in        */
/*    element order, within a row in block order, over each group of    */
/*    128 consecutive rows in row order, then over the groups in order  */
/*    (a fixed order whose longest chain of additions is short enough   */
/*    to run in parallel).  B = 0 keeps s_t.                            */
/*  - Start from the usual tensor scale; `iters` rounds of (block step, */
/*    tensor step); a final block step gives codes and scales.  The     */
/*    total error of the result (same summation order) goes to *sse.    */
/* Output layout as orc_quantize's canonical NVFP4.                     */
/* ------------------------------------------------------------------ */

#define ORC_MSE_GROUP 128   /* rows per group of the tensor-level sums */

/* error of block v under block code e (codes into q[16] when q != NULL) */
static double mse_block_error(const float *v, float s_t, uint8_t e, uint8_t *q)
{
    double err = 0.0;
    float d = e ? (float)orc_e4m3_value(e) * s_t : 0.0f;
    for (int i = 0; i < 16; i++) {
        uint8_t c = e ? orc_to_e2m1(v[i] / d) : 0;
        if (q) q[i] = c;
        double w_hat = orc_e2m1_value(c) * orc_e4m3_value(e) * (double)s_t;
        double diff = (double)v[i] - w_hat;
        err += diff * diff;
    }
    return err;
}

/* block step for one block: chosen code, its element codes and error */
static uint8_t mse_block_choose(const float *v, float s_t, uint8_t *q, double *err_out)
{
    float raw = (amax_of(v, 16) / 6.0f) / s_t;
    int e0 = orc_to_e4m3(raw);
    int order[8];
    int n = 0;
    order[n++] = e0;
    if (e0 == 0) {
        order[n++] = 1;
    } else {
        if (e0 + 1 <= 126) order[n++] = e0 + 1;
        for (int j = 1; j <= 6; j++)
            if (e0 - j >= 1) order[n++] = e0 - j;
    }
    int best = order[0];
    double best_err = mse_block_error(v, s_t, (uint8_t)best, NULL);
    for (int i = 1; i < n; i++) {
        double err = mse_block_error(v, s_t, (uint8_t)order[i], NULL);
        if (err < best_err) {
            best_err = err;
            best = order[i];
        }
    }
    mse_block_error(v, s_t, (uint8_t)best, q);
    *err_out = best_err;
    return (uint8_t)best;
}

/* The block step alone under a given tensor scale (the last step of       */
/* orc_quantize_mse_nvfp4): codes, scale bytes, and each row's error       */
/* summed in block order.                                                   */
int orc_mse_nvfp4_blocks(const float *x, int64_t rows, int64_t cols, float s_t, uint8_t *codes,
                         uint8_t *scales, double *row_err)
{
    if (rows < 0 || cols < 0 || cols % 16) return ORC_EINVAL;
    int64_t nb = cols / 16;
    uint8_t q[16];
    double err;
    for (int64_t r = 0; r < rows; r++) {
        double acc = 0.0;
        for (int64_t b = 0; b < nb; b++) {
            uint8_t e = mse_block_choose(x + r * cols + b * 16, s_t, q, &err);
            scales[r * nb + b] = e;
            for (int i = 0; i < 16; i++) put_code(codes, r * cols + b * 16 + i, 1, q[i]);
            acc += err;
        }
        row_err[r] = acc;
    }
    return ORC_OK;
}

int orc_quantize_mse_nvfp4(const float *x, int64_t rows, int64_t cols, int iters, uint8_t *codes,
                           uint8_t *scales, float *tensor_scale, double *sse)
{
    if (rows < 0 || cols < 0 || cols % 16 || iters < 0) return ORC_EINVAL;
    float amax_t = amax_of(x, rows * cols);
    float s_t = nvfp4_tensor_scale(amax_t);
    int64_t nb = cols / 16;
    uint8_t q[16];
    double err;
    for (int it = 0; it < iters; it++) {
        double a_sum = 0.0, b_sum = 0.0;
        for (int64_t g0 = 0; g0 < rows; g0 += ORC_MSE_GROUP) {
            double a_grp = 0.0, b_grp = 0.0;
            for (int64_t r = g0; r < rows && r < g0 + ORC_MSE_GROUP; r++) {
                double a_row = 0.0, b_row = 0.0;
                for (int64_t b = 0; b < nb; b++) {
                    const float *v = x + r * cols + b * 16;
                    uint8_t e = mse_block_choose(v, s_t, q, &err);
                    double a_blk = 0.0, b_blk = 0.0;
                    for (int i = 0; i < 16; i++) {
                        double u = orc_e2m1_value(q[i]) * orc_e4m3_value(e);
                        a_blk += (double)v[i] * u;
                        b_blk += u * u;
                    }
                    a_row += a_blk;
                    b_row += b_blk;
                }
                a_grp += a_row;
                b_grp += b_row;
            }
            a_sum += a_grp;
            b_sum += b_grp;
        }
        if (b_sum > 0.0) s_t = (float)(a_sum / b_sum);
    }
    *tensor_scale = s_t;
    double total = 0.0;
    for (int64_t g0 = 0; g0 < rows; g0 += ORC_MSE_GROUP) {
        double grp = 0.0;
        for (int64_t r = g0; r < rows && r < g0 + ORC_MSE_GROUP; r++) {
            double row_err;
            orc_mse_nvfp4_blocks(x + r * cols, 1, cols, s_t, codes + r * (cols / 2), scales + r * nb, &row_err);
            grp += row_err;
        }
        total += grp;
    }
    if (sse) *sse = total;
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Fixed grid scale for MX formats after rotation ("Bridging the Gap   */
/* Between Promise and Performance for Microscaling FP4 Quantization", */
/* MR-GPTQ modification 1: for MXFP4 with Hadamard rotations one fixed */
/* grid scale serves every model).  Readings: the grid scale g in      */
/* [1, 2] scales the block amax before the power-of-two exponent is    */
/* taken: e = floor(log2(g amax)) - emax, computed exactly as           */
/* floor(log2 amax) + [g m >= 2] - emax with m the significand of amax  */
/* in [1, 2) (g = 1: the OCP rule; g = 4/3: the exponent rises exactly */
/* when amax / 2^e would land in [6, 8), so E2M1 never clips; g and 2g */
/* differ by one exponent step, so [1, 2] spans every such rule); the   */
/* block is rotated first when hadamard_b > 0.  The                    */
/* fit scores each candidate g by the squared error of the rotated     */
/* tensor, sum (h - value(code) 2^e)^2 with the dequantized value exact */
/* in binary64, summed in binary64 in element order within a block, in */
/* block order within a row, over each group of 128 consecutive rows   */
/* in row order, and over the groups in order; the caller keeps the    */
/* least (a constant of the method, found once).                       */
/* ------------------------------------------------------------------ */

int orc_quantize_mx_grid(const float *x, int64_t rows, int64_t cols, int fmt, int hadamard_b, float g,
                         float *work, uint8_t *codes, uint8_t *scales)
{
    if ((fmt != ORC_MXFP4 && fmt != ORC_MXFP8) || rows < 0 || cols < 0 || cols % 32) return ORC_EINVAL;
    if (!(g >= 1.0f && g <= 2.0f)) return ORC_EINVAL;
    if (!all_finite(x, rows * cols)) return ORC_EINVAL;
    const float *src = x;
    if (hadamard_b) {
        if (orc_hadamard(x, work, rows, cols, hadamard_b) != ORC_OK) return ORC_EINVAL;
        src = work;
    }
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c += 32)
            quant_mx_block(src + r * cols + c, 32, fmt == ORC_MXFP4, g, codes, r * cols + c,
                           scales + r * (cols / 32) + c / 32);
    return ORC_OK;
}

int orc_mx_grid_sse(const float *x, int64_t rows, int64_t cols, int fmt, int hadamard_b, const float *gs, int n,
                    float *work, uint8_t *codes, uint8_t *scales, double *sse)
{
    int fp4 = fmt == ORC_MXFP4;
    for (int j = 0; j < n; j++) {
        int st = orc_quantize_mx_grid(x, rows, cols, fmt, hadamard_b, gs[j], work, codes, scales);
        if (st != ORC_OK) return st;
        const float *h = hadamard_b ? work : x;
        double total = 0.0;
        for (int64_t g0 = 0; g0 < rows; g0 += ORC_MSE_GROUP) {
            double grp = 0.0;
            for (int64_t r = g0; r < rows && r < g0 + ORC_MSE_GROUP; r++) {
                double row_err = 0.0;
                for (int64_t b = 0; b < cols / 32; b++) {
                    double scale = ldexp(1.0, (int)scales[r * (cols / 32) + b] - 127);
                    double err = 0.0;
                    for (int i = 0; i < 32; i++) {
                        int64_t idx = r * cols + b * 32 + i;
                        uint8_t c = fp4 ? (uint8_t)((codes[idx >> 1] >> (4 * (idx & 1))) & 0xF) : codes[idx];
                        double w_hat = (fp4 ? orc_e2m1_value(c) : orc_e4m3_value(c)) * scale;
                        double diff = (double)h[idx] - w_hat;
                        err += diff * diff;
                    }
                    row_err += err;
                }
                grp += row_err;
            }
            total += grp;
        }
        sse[j] = total;
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Activation-format calibration (Chameleon article, section "the      */
/* format is chosen by the value distribution": per layer and per      */
/* interval of the trajectory, activations are calibrated in advance   */
/* into the table read at generation time).  The page gives no         */
/* decision rule; the reading mirrors its rule for weights: an entry   */
/* takes the candidate with the least squared quantization error       */
/* accumulated over its calibration activations (orc_select's per-row  */
/* errors, rows summed over each group of 128 consecutive rows in      */
/* order, then the groups in order, then added to the accumulator);   */
/* the tail moments sum x^2 and sum x^4 are accumulated beside it      */
/* (binary64, element order within 16-element chunks, chunks in order  */
/* within a row, rows and groups as above).                            */
/* ------------------------------------------------------------------ */

int orc_calibrate_activation(const float *x, int64_t rows, int64_t cols, const int *cands, int ncand,
                             uint8_t *codes_work, void *scales_work, double *deq_work, uint8_t *choice_work,
                             double *sse_rows, double *sse_accum, double *moments_accum)
{
    if (rows < 0 || cols < 0 || cols % 16) return ORC_EINVAL;
    if (rows == 0 || cols == 0) return ORC_OK;
    int st = orc_select(x, rows, cols, cands, ncand, codes_work, scales_work, deq_work, choice_work, sse_rows);
    if (st != ORC_OK) return st;
    for (int j = 0; j < ncand; j++) {
        double total = 0.0;
        for (int64_t g0 = 0; g0 < rows; g0 += ORC_MSE_GROUP) {
            double grp = 0.0;
            for (int64_t r = g0; r < rows && r < g0 + ORC_MSE_GROUP; r++) grp += sse_rows[r * ncand + j];
            total += grp;
        }
        sse_accum[j] += total;
    }
    double t2 = 0.0, t4 = 0.0;
    for (int64_t g0 = 0; g0 < rows; g0 += ORC_MSE_GROUP) {
        double g2 = 0.0, g4 = 0.0;
        for (int64_t r = g0; r < rows && r < g0 + ORC_MSE_GROUP; r++) {
            double r2 = 0.0, r4 = 0.0;
            for (int64_t c = 0; c < cols; c += 16) {
                double c2 = 0.0, c4 = 0.0;
                for (int i = 0; i < 16; i++) {
                    double q = (double)x[r * cols + c + i] * (double)x[r * cols + c + i];
                    c2 += q;
                    c4 += q * q;
                }
                r2 += c2;
                r4 += c4;
            }
            g2 += r2;
            g4 += r4;
        }
        t2 += g2;
        t4 += g4;
    }
    moments_accum[0] += t2;
    moments_accum[1] += t4;
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* W4A16 weights (Nunchaku/Diffusers article, awq_w4a16: 4-bit         */
/* per-group weights against 16-bit activations).  Reading: a weight   */
/* is dequantized the way a kernel feeding 16-bit tensor cores does    */
/* it, w = bf16(RN32(q * s)) with q the signed INT4 code and s the     */
/* group's fp32 scale (canonical INT4 layout); the product with        */
/* bf16(x) is then summed (binary64 here, by the caller).               */
/* ------------------------------------------------------------------ */

int orc_w4a16_weights(const uint8_t *codes, const float *scales, int64_t n, int64_t k, int g, float *w)
{
    if (n < 0 || k < 0 || (g != 32 && g != 64) || k % g) return ORC_EINVAL;
    for (int64_t r = 0; r < n; r++)
        for (int64_t c = 0; c < k; c++) {
            int64_t idx = r * k + c;
            int q = get_code(codes, idx, 1);
            if (q & 8) q -= 16;
            float prod = (float)q * scales[r * (k / g) + c / g];
            w[idx] = orc_round_bf16(prod);
        }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* SVDQuant low-rank branch, down projection (Nunchaku/Diffusers       */
/* article, section "Main explanation": a 16-bit low-rank part of the  */
/* weight is kept beside the 4-bit residual).                          */
/* T[m][j] = sum_k bf16(x[m][k]) * L1[k][j], summed in binary64.       */
/* L1 values are given as fp32 (exact copies of bf16).                 */
/* ------------------------------------------------------------------ */

int orc_lowrank_down(const float *x, const float *l1, int64_t m, int64_t k, int r, double *t)
{
    for (int64_t i = 0; i < m; i++)
        for (int j = 0; j < r; j++) {
            double acc = 0.0;
            for (int64_t c = 0; c < k; c++)
                acc += (double)orc_round_bf16(x[i * k + c]) * (double)l1[c * r + j];
            t[i * r + j] = acc;
        }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Per-layer, per-timestep-interval format table (Chameleon article:   */
/* the trajectory is cut into ten intervals and, at generation time, a */
/* layer reads its format for the current stage from the table).       */
/* Reading: interval = floor(step * n_intervals / n_steps).            */
/* Returns the format id, or -1 for out-of-range arguments.            */
/* ------------------------------------------------------------------ */

int orc_route(const uint8_t *table, int n_layers, int n_intervals, int layer, int step, int n_steps)
{
    if (n_layers <= 0 || n_intervals <= 0 || n_steps <= 0) return -1;
    if (layer < 0 || layer >= n_layers || step < 0 || step >= n_steps) return -1;
    int interval = (int)((int64_t)step * n_intervals / n_steps);
    return table[(int64_t)layer * n_intervals + interval];
}
