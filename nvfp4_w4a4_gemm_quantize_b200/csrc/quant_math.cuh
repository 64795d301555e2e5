// quant_math.cuh -- per-block NVFP4 arithmetic shared by the quantize kernel
// and the NVFP4-emitting GEMM epilogue, so both produce identical codes.
//
// "NVFP4-DiT ..." README, Methodology 1, Definition III.1 with the
// "[RFC]: NVFP4 Quantization Support for Diffusion Models" two-level scaling:
//   sf = E4M3_rne_satfinite(a_b / d),  d = 6 g,  s = e4m3(sf) * g
//   code = E2M1_rne_satfinite(rn(x / s)), sign of x kept; s == 0 gives 0.
#pragma once
#include "ptx.cuh"

namespace nvfp4 {

// True when r is within 8 ulps of a value whose low 19 fraction bits are zero:
// every E4M3 rounding midpoint (4 significant bits, normal or subnormal) is
// such a value.
__device__ __forceinline__ bool near_e4m3_midpoint(float r) {
    return ((__float_as_uint(r) + 8u) & 0x7FFF0u) == 0u;
}

// Hardware reciprocal approximation (at most 1 ulp from 1/s for normal s).
__device__ __forceinline__ float rcp_approx(float s) {
    float r;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(s));
    return r;
}

// Per-tensor constants of the block-scale step: d = 6 g and rd = rn(1/d).
struct ScaleConsts {
    float g, d, rd;
    bool fast;          // d in the range where ab * rd is within 1.5 ulps of ab / d
};

__device__ __forceinline__ ScaleConsts scale_consts(float g) {
    ScaleConsts c;
    c.g = g;
    c.d = __fmul_rn(6.0f, g);
    c.fast = c.d >= 0x1p-125f && c.d <= 0x1p125f;
    c.rd = c.fast ? __frcp_rn(c.d) : 0.0f;
    return c;
}

// E4M3 block-scale code for block max `ab`: E4M3_rne_satfinite(rn(ab / d)).
// The product ab * rd differs from the IEEE quotient by at most 2 ulps, and
// E4M3 rounding can only differ near a midpoint, where the exact quotient is
// taken instead.
__device__ __forceinline__ uint32_t block_scale_code(float ab, const ScaleConsts& c) {
    if (!(c.d > 0.0f)) return 0u;
    float r;
    if (c.fast) {
        r = __fmul_rn(ab, c.rd);
        if (near_e4m3_midpoint(r)) r = __fdiv_rn(ab, c.d);
    } else {
        r = __fdiv_rn(ab, c.d);
    }
    return cvt_e4m3(r);
}

// Pack four E2M1 pairs (each in the low byte of a word) into one word.
__device__ __forceinline__ uint32_t pack4(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
    uint32_t lo, hi, r;
    asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(lo) : "r"(b0), "r"(b1));
    asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(hi) : "r"(b2), "r"(b3));
    asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(r) : "r"(lo), "r"(hi));
    return r;
}

// Two FP32 values in one 64-bit register (low word first) for the packed
// FP32 instructions of sm_100.
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// E2M1 codes of four packed FP32 pairs (satfinite, RNE) in one word: byte j
// holds pair j, its low word's code in the low nibble.
__device__ __forceinline__ uint32_t cvt_e2m1x8(uint64_t p0, uint64_t p1, uint64_t p2, uint64_t p3) {
    uint32_t r;
    asm("{\n\t.reg .b8 t0, t1, t2, t3;\n\t.reg .f32 a0, a1, a2, a3, a4, a5, a6, a7;\n\t"
        "mov.b64 {a0, a1}, %1;\n\t"
        "mov.b64 {a2, a3}, %2;\n\t"
        "mov.b64 {a4, a5}, %3;\n\t"
        "mov.b64 {a6, a7}, %4;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t0, a1, a0;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t1, a3, a2;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t2, a5, a4;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t3, a7, a6;\n\t"
        "mov.b32 %0, {t0, t1, t2, t3};\n\t}"
        : "=r"(r)
        : "l"(p0), "l"(p1), "l"(p2), "l"(p3));
    return r;
}

// Reciprocal bracket of s: rl <= 1/s <= rh, four ulps either side of the
// hardware approximation (which is within one ulp of 1/s for normal s).
struct RcpBracket {
    uint64_t lo, hi;
};

__device__ __forceinline__ RcpBracket rcp_bracket(float s) {
    const uint32_t rb = __float_as_uint(rcp_approx(s));
    const float rl = __uint_as_float(rb - 4u), rh = __uint_as_float(rb + 4u);
    return {f32x2(rl, rl), f32x2(rh, rh)};
}

// E2M1 codes of eight values given as four packed pairs, divided by the
// decoded block scale s (IEEE single quotient, then RNE to E2M1, saturating).
// The quotient is bracketed: |x * rl| <= |x / s| <= |x * rh| for the
// reciprocal bracket of s, and both rounding to single precision and the
// E2M1 rounding are monotone in magnitude, so where the codes of the two
// bounds agree they are the code of the exact quotient.  Returns the codes
// of the lower bound (element 2j in the low nibble of byte j) and, in `d`,
// the nibbles where the bounds disagree (a rounding boundary lies inside the
// bracket: about 1 value in 2000, because quotients a unit in the last place
// from an E2M1 midpoint are common); those values must be divided exactly.
__device__ __forceinline__ uint32_t bracket_codes8(const uint64_t (&x)[4], float s, uint32_t& d) {
    const RcpBracket rb = rcp_bracket(s);
    const uint32_t w = cvt_e2m1x8(mul_f32x2(x[0], rb.lo), mul_f32x2(x[1], rb.lo), mul_f32x2(x[2], rb.lo),
                                  mul_f32x2(x[3], rb.lo));
    d = w ^ cvt_e2m1x8(mul_f32x2(x[0], rb.hi), mul_f32x2(x[1], rb.hi), mul_f32x2(x[2], rb.hi),
                       mul_f32x2(x[3], rb.hi));
    return w;
}

// Replace nibble j of w by the E2M1 code of v / s (exact IEEE quotient).
__device__ __forceinline__ uint32_t patch_exact(uint32_t w, int j, float v, float s) {
    const uint32_t c = cvt_e2m1x2(__fdiv_rn(v, s), 0.0f) & 0xFu;
    return (w & ~(0xFu << (4 * j))) | (c << (4 * j));
}

// s in the range where the reciprocal bracket is valid (normal reciprocal).
__device__ __forceinline__ bool bracket_ok(float s) { return s >= 0x1p-125f && s <= 0x1p125f; }

// Eight FP32 values (element 2j in the low nibble of byte j).  Blocks whose s
// is outside the bracket range are divided exactly throughout.
__device__ __forceinline__ uint32_t quantize8(const float (&f)[8], float s) {
    if (s == 0.0f) return 0u;
    uint32_t w = 0u;
    if (bracket_ok(s)) {
        const uint64_t x[4] = {f32x2(f[0], f[1]), f32x2(f[2], f[3]), f32x2(f[4], f[5]), f32x2(f[6], f[7])};
        uint32_t d;
        w = bracket_codes8(x, s, d);
        // rare: the disagreeing values, by an unrolled scan (a register array
        // indexed at run time would live in local memory)
        if (d != 0u) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if ((d >> (4 * j)) & 0xFu) w = patch_exact(w, j, f[j], s);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) w = patch_exact(w, j, f[j], s);
    }
    return w;
}

// bf16 value j (0..7) of four words, the lower half of each word first, as FP32.
__device__ __forceinline__ float bf16_at(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, int j) {
    const uint32_t w = j < 2 ? w0 : j < 4 ? w1 : j < 6 ? w2 : w3;
    return __uint_as_float((j & 1) ? (w & 0xFFFF0000u) : (w << 16));
}

// Eight bf16 values in four words (the lower half of each word first).
__device__ __forceinline__ uint32_t quantize8_bf16(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, float s) {
    if (s == 0.0f) return 0u;
    uint32_t w = 0u;
    if (bracket_ok(s)) {
        const uint64_t x[4] = {f32x2(__uint_as_float(w0 << 16), __uint_as_float(w0 & 0xFFFF0000u)),
                               f32x2(__uint_as_float(w1 << 16), __uint_as_float(w1 & 0xFFFF0000u)),
                               f32x2(__uint_as_float(w2 << 16), __uint_as_float(w2 & 0xFFFF0000u)),
                               f32x2(__uint_as_float(w3 << 16), __uint_as_float(w3 & 0xFFFF0000u))};
        uint32_t d;
        w = bracket_codes8(x, s, d);
        while (d != 0u) {                       // rare: one pass per disagreeing value
            const int j = (31 - __clz(d)) >> 2;
            w = patch_exact(w, j, bf16_at(w0, w1, w2, w3, j), s);
            d &= ~(0xFu << (4 * j));
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) w = patch_exact(w, j, bf16_at(w0, w1, w2, w3, j), s);
    }
    return w;
}

// Largest magnitude of two packed bf16 pairs, per half (sign bits are the
// XOR of the inputs' and are cleared by the caller).  NaN operands are
// ignored when the other operand is a number.
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// |x| pattern (sign cleared) of the largest-magnitude value among 16 bf16
// values in eight words.
__device__ __forceinline__ uint32_t block_absmax16(const uint32_t (&w)[8]) {
    const uint32_t m = absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(w[0], w[1]), absmax_bf16x2(w[2], w[3])),
                                     absmax_bf16x2(absmax_bf16x2(w[4], w[5]), absmax_bf16x2(w[6], w[7])));
    const uint32_t lo = m & 0x7FFFu, hi = (m >> 16) & 0x7FFFu;
    return lo > hi ? lo : hi;
}

}  // namespace nvfp4
