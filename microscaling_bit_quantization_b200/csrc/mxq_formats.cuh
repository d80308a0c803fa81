// mxq_formats.cuh -- device-side element codecs and per-block scale rules.
//
// Encodings follow the OCP Microscaling (MX) v1.0 definition (E2M1, E4M3
// "fn", E8M0, 32-element blocks) and NVIDIA's NVFP4 definition (E2M1 in
// 16-element blocks with an E4M3 block scale and an fp32 tensor scale); the
// pages name these formats (Chameleon article: MXFP8 blocks sharing an
// exponent; Nunchaku/Diffusers article: INT4 and NVFP4 svdq_w4a4 variants;
// "Bridging the Gap ... Microscaling FP4 Quantization": NVFP4 groups, MXFP4
// power-of-two scales) but do not define them.
//
// Encoding uses the hardware conversions (cvt.rn.satfinite.{e4m3x2,e2m1x2})
// through the CUDA intrinsics; every fp32 division or multiply that feeds a
// code uses the IEEE round-to-nearest intrinsics so no contraction or
// approximate division can change a code.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace mxq {

enum Fmt : int {
    kMXFP8 = 0, kMXFP4 = 1, kNVFP4 = 2, kINT4G32 = 3, kINT4G64 = 4, kINT8Row = 5, kFP8Tensor = 6,
    kNumFmt = 7
};

__host__ __device__ constexpr int fmt_block(int f) {
    return (f == kMXFP8 || f == kMXFP4 || f == kINT4G32) ? 32 : f == kNVFP4 ? 16 : f == kINT4G64 ? 64 : 0;
}
__host__ __device__ constexpr bool fmt_is4(int f) {
    return f == kMXFP4 || f == kNVFP4 || f == kINT4G32 || f == kINT4G64;
}
__host__ __device__ constexpr bool fmt_tensor_scaled(int f) { return f == kNVFP4 || f == kFP8Tensor; }
__host__ __device__ constexpr bool fmt_byte_scales(int f) { return f == kMXFP8 || f == kMXFP4 || f == kNVFP4; }

// ----------------------------------------------------------------- encode

__device__ __forceinline__ uint8_t enc_e4m3(float v) {
    return (uint8_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

// Two E2M1 codes in one byte: `lo` in bits 0..3, `hi` in bits 4..7.
__device__ __forceinline__ uint8_t enc_e2m1x2(float lo, float hi) {
    return (uint8_t)__nv_cvt_float2_to_fp4x2(make_float2(lo, hi), __NV_E2M1, cudaRoundNearest);
}

// ----------------------------------------------------------------- decode

// E4M3: exponent field e (bias 7), mantissa m; e == 0 is subnormal m * 2^-9;
// S.1111.111 is NaN.
__device__ __forceinline__ float dec_e4m3(uint32_t c) {
    uint32_t e = (c >> 3) & 15u, m = c & 7u;
    float mag;
    if ((c & 0x7Fu) == 0x7Fu) mag = __int_as_float(0x7FC00000);
    else if (e == 0) mag = __fmul_rn((float)m, 0.001953125f);          // m * 2^-9, exact
    else mag = __int_as_float((int)(((e + 120u) << 23) | (m << 20)));  // (1 + m/8) * 2^(e-7)
    return (c & 0x80u) ? -mag : mag;
}

// E2M1: exponent field e (bias 1), mantissa bit m; e == 0 is m * 0.5.
__device__ __forceinline__ float dec_e2m1(uint32_t c) {
    uint32_t e = (c >> 1) & 3u, m = c & 1u;
    float mag = e == 0 ? (m ? 0.5f : 0.0f) : __int_as_float((int)(((e + 126u) << 23) | (m << 22)));
    return (c & 8u) ? -mag : mag;
}

// 2^n as fp32 for n in [-127, 127] (2^-127 is the subnormal 0x00400000).
__device__ __forceinline__ float exp2i_f32(int n) {
    return n >= -126 ? __int_as_float((n + 127) << 23) : __int_as_float(0x00400000);
}

// E8M0 scale byte b -> 2^(b - 127); 0xFF is NaN.
__device__ __forceinline__ float dec_e8m0(uint32_t b) {
    return b == 255u ? __int_as_float(0x7FC00000) : exp2i_f32((int)b - 127);
}

__device__ __forceinline__ double exp2i_f64(int n) {   // n in [-1022, 1023]
    return __longlong_as_double((long long)(n + 1023) << 52);
}

// floor(log2(a)) for finite a > 0, from the binary32 fields.
__device__ __forceinline__ int floor_log2_pos(float a) {
    uint32_t u = __float_as_uint(a);
    int e = (int)((u >> 23) & 0xFFu);
    if (e) return e - 127;
    return (31 - __clz((int)(u & 0x7FFFFFu))) - 149;
}

// ----------------------------------------------------------------- integer division

// floor(n / d) for n < 2^31 and 1 <= d < 2^31 by one multiply-high
// (Granlund & Montgomery, "Division by invariant integers using
// multiplication", 1994): with l = ceil(log2 d) and m = floor(2^(31+l)/d) + 1,
// m*d - 2^(31+l) <= 2^l, so floor(n/d) = floor(m n / 2^(31+l)) for all 31-bit
// n; m fits 32 bits when d is not a power of two (powers of two shift).
struct FastDiv {
    uint32_t d, m;
    int l;
};
inline FastDiv make_fastdiv(uint32_t d) {
    FastDiv f;
    f.d = d;
    f.l = 0;
    while ((1u << f.l) < d) f.l++;
    f.m = (d & (d - 1)) == 0 ? 0u : (uint32_t)((((uint64_t)1) << (31 + f.l)) / d + 1);
    return f;
}
__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv &f) {
    return f.m == 0 ? (n >> f.l) : (__umulhi(n, f.m) >> (f.l - 1));
}

// ----------------------------------------------------------------- scale rules

// OCP MX shared scale: e = floor(log2 amax) - emax_elem, clamped to [-127,127];
// scale byte e + 127.  Returns the byte; `inv` gets 2^-e.  amax must be > 0.
__device__ __forceinline__ uint32_t mx_scale(float amax, int emax_elem, float &inv) {
    int e = floor_log2_pos(amax) - emax_elem;
    e = e < -127 ? -127 : (e > 127 ? 127 : e);
    inv = exp2i_f32(-e);
    return (uint32_t)(e + 127);
}

// MX shared scale with a fixed grid scale g in [1, 2] ("Bridging the Gap
// ...", MR-GPTQ modification 1: one fixed grid scale for rotated MXFP4): the
// exponent of g * amax, e = floor(log2 amax) + [g m >= 2] - emax_elem with m
// the significand of amax in [1, 2), the product exact in binary64; g = 1
// gives mx_scale.  amax must be > 0.
__device__ __forceinline__ uint32_t mx_scale_grid(float amax, int emax_elem, float g, float &inv) {
    const int fl = floor_log2_pos(amax);
    const double m = __dmul_rn((double)amax, exp2i_f64(-fl));   // exact
    int e = fl + (__dmul_rn((double)g, m) >= 2.0 ? 1 : 0) - emax_elem;
    e = e < -127 ? -127 : (e > 127 ? 127 : e);
    inv = exp2i_f32(-e);
    return (uint32_t)(e + 127);
}

// NVFP4 tensor scale s_t = RN(amax_T / (6 * 448)); 1 when that is 0.
__device__ __forceinline__ float nvfp4_tensor_scale(float amax_t) {
    float s = __fdiv_rn(amax_t, 2688.0f);
    return s == 0.0f ? 1.0f : s;
}

// FP8 per-tensor scale s = RN(amax_T / 448); 1 when that is 0.
__device__ __forceinline__ float fp8_tensor_scale(float amax_t) {
    float s = __fdiv_rn(amax_t, 448.0f);
    return s == 0.0f ? 1.0f : s;
}

// NVFP4 block: E4M3 block scale of RN(RN(amax_b / 6) / s_t); decode scale
// d = RN(value(e4) * s_t) (0 when e4 == 0).
__device__ __forceinline__ uint32_t nvfp4_block_scale(float amax_b, float s_t, float &d) {
    float raw = __fdiv_rn(__fdiv_rn(amax_b, 6.0f), s_t);
    uint32_t e4 = enc_e4m3(raw);
    d = e4 ? __fmul_rn(dec_e4m3(e4), s_t) : 0.0f;
    return e4;
}

// Symmetric integer code: clamp(RNE(RN(v / s)), -qmax, qmax); 0 when s == 0.
__device__ __forceinline__ int int_code(float v, float s, int qmax) {
    if (s == 0.0f) return 0;
    int q = __float2int_rn(__fdiv_rn(v, s));
    return q > qmax ? qmax : (q < -qmax ? -qmax : q);
}

// ----------------------------------------------------------------- packed conversions

// E2M1 codes of eight fp32 values (RN, satfinite), two per byte, element
// 2i in the low nibble of byte i.  The conversion keeps the sign of zero.
__device__ __forceinline__ uint32_t cvt_e2m1x8(float v0, float v1, float v2, float v3, float v4, float v5,
                                               float v6, float v7) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
    return r;
}

// E4M3 codes of four fp32 values (RN, satfinite), element i in byte i.
__device__ __forceinline__ uint32_t cvt_e4m3x4(float v0, float v1, float v2, float v3) {
    uint32_t r;
    asm("{\n\t.reg .b16 h0, h1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 h0, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 h1, %4, %3;\n\t"
        "mov.b32 %0, {h0, h1};\n\t}"
        : "=r"(r)
        : "f"(v0), "f"(v1), "f"(v2), "f"(v3));
    return r;
}

// Value of a positive E4M3 code (exact: every E4M3 value is an fp16 value).
// The code is placed in both bytes, so either half of the result holds it.
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
    uint32_t h2;
    asm("{\n\t.reg .b16 c;\n\tcvt.u16.u32 c, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, c;\n\t}" : "=r"(h2) : "r"(code * 0x101u));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// ----------------------------------------------------------------- codes of quotients
//
// Codes of RN(v / d) for many v and one divisor d, without an IEEE division
// per element.  With y within one ulp of 1/d (rcp.approx.ftz.f32, whose
// maximum error the PTX ISA gives as 1 ulp over the full range) and the
// bracket multipliers y_lo = RN(y (1 - 2^-20)), y_hi = RN(y (1 + 2^-20)), the
// products L = v y_lo and H = v y_hi (exact reals, or rounded once) satisfy
// |L| < |v/d|(1 - 11 * 2^-24) and |H| > |v/d|(1 + 11 * 2^-24), so RN(v/d),
// which is within 2^-24 of v/d, lies strictly between them.  Every code
// function used here (E2M1, E4M3, round-to-integer) is monotone, so when the
// codes of L and H agree the code of RN(v/d) is that code; otherwise a code
// boundary or an exact tie lies inside the bracket and that group of values
// is coded from exact divisions.  Signs need no special handling: the codes
// are odd functions and the bracket ends keep the sign of v.  When products
// fall into the fp32 subnormal range the relative bound fails, but the ends
// and the true quotient are then far below the smallest nonzero code.
struct Recip {
    float d, lo, hi;
    bool fast;   // d in [2^-120, 2^120]: y finite and normal, no overflow in the products
};
constexpr float kBracketLo = 0.99999904632568359375f;   // 1 - 2^-20
constexpr float kBracketHi = 1.00000095367431640625f;   // 1 + 2^-20
__device__ __forceinline__ Recip recip_of(float d) {
    Recip r;
    r.d = d;
    r.fast = d >= 7.52316384526264e-37f && d <= 1.329227995784916e36f;
    float y = 0.0f;
    if (r.fast) asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(d));
    r.lo = __fmul_rn(y, kBracketLo);
    r.hi = __fmul_rn(y, kBracketHi);
    return r;
}

// Products of eight values with one factor, as four packed two-wide multiplies
// (each lane of a pair rounded exactly like __fmul_rn).
__device__ __forceinline__ void mul8(const float *v, float f, float *o) {
    const float2 ff = make_float2(f, f);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const float2 p = __fmul2_rn(make_float2(v[2 * i], v[2 * i + 1]), ff);
        o[2 * i] = p.x;
        o[2 * i + 1] = p.y;
    }
}

// E2M1 codes of RN(v[i] / d) for eight values, packed like cvt_e2m1x8.
__device__ __forceinline__ uint32_t e2m1x8_quot(const float *v, const Recip &r) {
    if (r.fast) {
        float l[8], h[8];
        mul8(v, r.lo, l);
        mul8(v, r.hi, h);
        const uint32_t lo = cvt_e2m1x8(l[0], l[1], l[2], l[3], l[4], l[5], l[6], l[7]);
        const uint32_t hi = cvt_e2m1x8(h[0], h[1], h[2], h[3], h[4], h[5], h[6], h[7]);
        if (lo == hi) return lo;
    }
    return cvt_e2m1x8(__fdiv_rn(v[0], r.d), __fdiv_rn(v[1], r.d), __fdiv_rn(v[2], r.d), __fdiv_rn(v[3], r.d),
                      __fdiv_rn(v[4], r.d), __fdiv_rn(v[5], r.d), __fdiv_rn(v[6], r.d), __fdiv_rn(v[7], r.d));
}

// E4M3 codes of RN(v[i] / d) for four values, packed like cvt_e4m3x4.
__device__ __forceinline__ uint32_t e4m3x4_quot(const float *v, const Recip &r) {
    if (r.fast) {
        // packed two-wide products, each lane rounded like __fmul_rn
        const float2 v01 = make_float2(v[0], v[1]), v23 = make_float2(v[2], v[3]);
        const float2 lo2 = make_float2(r.lo, r.lo), hi2 = make_float2(r.hi, r.hi);
        const float2 l01 = __fmul2_rn(v01, lo2), l23 = __fmul2_rn(v23, lo2);
        const float2 h01 = __fmul2_rn(v01, hi2), h23 = __fmul2_rn(v23, hi2);
        const uint32_t lo = cvt_e4m3x4(l01.x, l01.y, l23.x, l23.y);
        const uint32_t hi = cvt_e4m3x4(h01.x, h01.y, h23.x, h23.y);
        if (lo == hi) return lo;
    }
    return cvt_e4m3x4(__fdiv_rn(v[0], r.d), __fdiv_rn(v[1], r.d), __fdiv_rn(v[2], r.d), __fdiv_rn(v[3], r.d));
}

// Symmetric integer codes clamp(RNE(RN(v[i]/s)), -qmax, qmax) of four values,
// as bytes (two's complement, element i in byte i); all 0 when s == 0.
// Rounding to an integer is one FMA: for |t| < 2^22, RN(t + 1.5 * 2^23) is
// 1.5 * 2^23 + RNE(t) with no intermediate rounding of t, and the low byte of
// its bit pattern is RNE(t) in two's complement.  The fast path needs no
// clamp when s comes from the block's own maximum: |v| <= amax and
// s = RN(amax / qmax) give |v/s| <= qmax (1 + 2^-23), which rounds to qmax.
constexpr float kRoundMagic = 12582912.0f;   // 1.5 * 2^23
__device__ __forceinline__ uint32_t int_x4_quot(const float *v, const Recip &r, int qmax) {
    if (r.d == 0.0f) return 0u;
    if (r.fast) {
        uint32_t b[4];
        bool same = true;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float l = __fmaf_rn(v[i], r.lo, kRoundMagic), h = __fmaf_rn(v[i], r.hi, kRoundMagic);
            same = same && l == h;
            b[i] = __float_as_uint(l);
        }
        if (same) return __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
    }
    uint32_t out = 0;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        int q = __float2int_rn(__fdiv_rn(v[i], r.d));
        q = q > qmax ? qmax : (q < -qmax ? -qmax : q);
        out |= ((uint32_t)q & 0xFFu) << (8 * i);
    }
    return out;
}

// int_x4_quot with the bracket FMAs packed two-wide (each lane rounded like
// __fmaf_rn): fewer instructions, two more live registers, so it is used
// where registers are not the limit (the staged INT8 per-row kernel).
__device__ __forceinline__ uint32_t int_x4_quot_packed(const float *v, const Recip &r, int qmax) {
    if (r.d == 0.0f) return 0u;
    if (r.fast) {
        const float2 lo2 = make_float2(r.lo, r.lo), hi2 = make_float2(r.hi, r.hi);
        const float2 mg = make_float2(kRoundMagic, kRoundMagic);
        const float2 v01 = make_float2(v[0], v[1]), v23 = make_float2(v[2], v[3]);
        const float2 l01 = __ffma2_rn(v01, lo2, mg), l23 = __ffma2_rn(v23, lo2, mg);
        const float2 h01 = __ffma2_rn(v01, hi2, mg), h23 = __ffma2_rn(v23, hi2, mg);
        if (l01.x == h01.x && l01.y == h01.y && l23.x == h23.x && l23.y == h23.y)
            return __byte_perm(__byte_perm(__float_as_uint(l01.x), __float_as_uint(l01.y), 0x0040),
                               __byte_perm(__float_as_uint(l23.x), __float_as_uint(l23.y), 0x0040), 0x5410);
    }
    return int_x4_quot(v, Recip{r.d, r.lo, r.hi, false}, qmax);   // exact divisions
}

// The same integer codes as E4M3 bytes (element i in byte i).  Every integer
// of magnitude <= 7 is an E4M3 value, so the conversion is exact; a zero code
// is +0 (RN(1.5 * 2^23 - 1.5 * 2^23) = +0).
__device__ __forceinline__ uint32_t int_x4_quot_e4m3(const float *v, const Recip &r, int qmax) {
    if (r.d == 0.0f) return 0u;
    if (r.fast) {
        float q[4];
        bool same = true;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float l = __fmaf_rn(v[i], r.lo, kRoundMagic), h = __fmaf_rn(v[i], r.hi, kRoundMagic);
            same = same && l == h;
            q[i] = __fsub_rn(l, kRoundMagic);
        }
        if (same) return cvt_e4m3x4(q[0], q[1], q[2], q[3]);
    }
    float q[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        int c = __float2int_rn(__fdiv_rn(v[i], r.d));
        c = c > qmax ? qmax : (c < -qmax ? -qmax : c);
        q[i] = (float)c;
    }
    return cvt_e4m3x4(q[0], q[1], q[2], q[3]);
}

// Low nibbles of the four bytes of two words, as eight packed nibbles
// (byte i of w0 -> nibble i, byte i of w1 -> nibble 4 + i).
__device__ __forceinline__ uint32_t nibbles_of_bytes(uint32_t w0, uint32_t w1) {
    uint32_t t0 = w0 & 0x0F0F0F0Fu, t1 = w1 & 0x0F0F0F0Fu;
    t0 |= t0 >> 4;   // byte 0: n0 | n1 << 4, byte 2: n2 | n3 << 4
    t1 |= t1 >> 4;
    return __byte_perm(t0, t1, 0x6420);
}

// ----------------------------------------------------------------- NVFP4 block scale

// Reciprocal of the tensor scale, for the division-free block-scale path.
struct TensorRecip {
    float s, inv;
    bool fast;   // s in [2^-100, 2^100]
};
__device__ __forceinline__ TensorRecip tensor_recip_of(float s) {
    TensorRecip t;
    t.s = s;
    t.fast = s >= 7.888609052210118e-31f && s <= 1.2676506002282294e30f;
    t.inv = t.fast ? __frcp_rn(s) : 0.0f;
    return t;
}

// The NVFP4 block scale of nvfp4_block_scale without the two divisions in
// the common case.  q = RN(RN(amax_b c6) inv), c6 = RN(1/6), is within
// 4 * 2^-24 of amax_b / (6 s_t) and the exact RN(RN(amax_b / 6) / s_t) within
// 2 * 2^-24, so the E4M3 codes of RN(q (1 -+ 2^-20)) enclose the exact code
// (the argument of the quotient codes above); on disagreement, divide.  With
// s_t in [2^-100, 2^100] a subnormal RN(amax_b c6) only occurs when both ends
// and the exact value are below 2^-26, where every code is 0.
constexpr float kInvSix = 0.16666667163372039794921875f;   // RN(1/6)
__device__ __forceinline__ uint32_t nvfp4_block_scale_fast(float amax_b, const TensorRecip &t, float &d) {
    uint32_t e4 = 0;
    bool done = false;
    if (t.fast) {
        const float q = __fmul_rn(__fmul_rn(amax_b, kInvSix), t.inv);
        const uint32_t two = cvt_e4m3x4(__fmul_rn(q, kBracketLo), __fmul_rn(q, kBracketHi), 0.0f, 0.0f);
        e4 = two & 0xFFu;
        done = e4 == ((two >> 8) & 0xFFu);
    }
    if (!done) e4 = enc_e4m3(__fdiv_rn(__fdiv_rn(amax_b, 6.0f), t.s));
    d = e4 ? __fmul_rn(e4m3_to_f32(e4), t.s) : 0.0f;
    return e4;
}

// ----------------------------------------------------------------- loads

// 16 consecutive elements as fp32 (bf16 widened exactly).
__device__ __forceinline__ void load16(const float *p, float v[16]) {
    const float4 *q = reinterpret_cast<const float4 *>(p);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        float4 t = __ldg(q + i);
        v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
    }
}
__device__ __forceinline__ void load16(const __nv_bfloat16 *p, float v[16]) {
    const uint4 *q = reinterpret_cast<const uint4 *>(p);
#pragma unroll
    for (int i = 0; i < 2; i++) {
        uint4 t = __ldg(q + i);
        uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
            v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
            v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    }
}

__device__ __forceinline__ void store16(float *p, const float v[16]) {
    float4 *q = reinterpret_cast<float4 *>(p);
#pragma unroll
    for (int i = 0; i < 4; i++) q[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);   // RNE; .x (low half) = lo
    return *reinterpret_cast<uint32_t *>(&t);
}
__device__ __forceinline__ void store16(__nv_bfloat16 *p, const float v[16]) {
    uint4 *q = reinterpret_cast<uint4 *>(p);
#pragma unroll
    for (int i = 0; i < 2; i++)
        q[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                          pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
}

__device__ __forceinline__ float amax16(const float v[16]) {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; i++) m = fmaxf(m, fabsf(v[i]));
    return m;
}

// Max over aligned groups of G lanes (G a power of two <= 32).
template <int G>
__device__ __forceinline__ float group_max(float a) {
#pragma unroll
    for (int o = 1; o < G; o <<= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
    return a;
}

// ----------------------------------------------------------------- Hadamard

// Block-diagonal Hadamard rotation of size b (a power of two in [2, 256]:
// the callers check it) ("Bridging the Gap ...", item 3) over 16-element
// chunks, one chunk per lane, consecutive chunks of
// a row in consecutive lanes.  Butterfly stage h pairs elements i and i+h
// (bit h of i clear) into (a+c, a-c); stages h < 16 stay inside the lane,
// stages h >= 16 pair lanes that differ in bit h/16.  Then every element is
// multiplied by norm = RN(1/sqrt(b)) (hadamard_chunk computes it; a loop over
// many chunks passes it in).  All lanes of the warp must call this.
__device__ __forceinline__ void hadamard_chunk_n(float v[16], int b, int lane, float norm) {
    // stage h = 1 inside the lane, element pairs (i, i + 1)
    if (b > 1) {
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            const float a = v[i], c = v[i + 1];
            v[i] = __fadd_rn(a, c);
            v[i + 1] = __fsub_rn(a, c);
        }
    }
    // stages h = 2, 4, 8 inside the lane on adjacent pairs, two-wide: a + c,
    // and a - c as the FMA c * (-1) + a (exact product, one rounding: the
    // same value as the subtraction)
#pragma unroll
    for (int h = 2; h < 16; h <<= 1) {
        if (h < b) {
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
                if (!(i & h)) {
                    const float2 a = make_float2(v[i], v[i + 1]), c = make_float2(v[i + h], v[i + h + 1]);
                    const float2 sum = __fadd2_rn(a, c), dif = __ffma2_rn(c, make_float2(-1.0f, -1.0f), a);
                    v[i] = sum.x;
                    v[i + 1] = sum.y;
                    v[i + h] = dif.x;
                    v[i + h + 1] = dif.y;
                }
            }
        }
    }
    // stages h = 16 lm across lanes that differ in bit lm: the lower lane
    // keeps v + p, the upper p - v, both as the FMA (+-1) * v + p
#pragma unroll
    for (int lm = 1; lm < 16; lm <<= 1) {
        if (16 * lm < b) {
            const float sg = (lane & lm) ? -1.0f : 1.0f;
            const float2 sg2 = make_float2(sg, sg);
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
                const float p0 = __shfl_xor_sync(0xFFFFFFFFu, v[i], lm);
                const float p1 = __shfl_xor_sync(0xFFFFFFFFu, v[i + 1], lm);
                const float2 r = __ffma2_rn(sg2, make_float2(v[i], v[i + 1]), make_float2(p0, p1));
                v[i] = r.x;
                v[i + 1] = r.y;
            }
        }
    }
    const float2 n2 = make_float2(norm, norm);
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
        const float2 r = __fmul2_rn(make_float2(v[i], v[i + 1]), n2);
        v[i] = r.x;
        v[i + 1] = r.y;
    }
}
__device__ __forceinline__ void hadamard_chunk(float v[16], int b, int lane) {
    hadamard_chunk_n(v, b, lane, __frsqrt_rn((float)b));
}

// Byte offset of scale (row r, scale column s) in the MMA scale layout:
// 128-row x 4-column atoms of 512 bytes, row r%32 at 16-byte pitch, the four
// 32-row quarters side by side in each 16-byte line.
__host__ __device__ __forceinline__ int64_t mma_scale_offset(int64_t r, int64_t s, int64_t s_pad) {
    return ((r >> 7) * (s_pad >> 2) + (s >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (s & 3);
}
// The same offset in 32-bit arithmetic (scale arrays below 2^32 bytes);
// s_pad4 = s_pad / 4.
__device__ __forceinline__ uint32_t mma_scale_offset32(uint32_t r, uint32_t s, uint32_t s_pad4) {
    return ((r >> 7) * s_pad4 + (s >> 2)) * 512u + (r & 31u) * 16u + ((r >> 5) & 3u) * 4u + (s & 3u);
}

}  // namespace mxq
