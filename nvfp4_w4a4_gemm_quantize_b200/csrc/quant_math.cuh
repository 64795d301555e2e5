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

// True when q is within 8 ulps of a value whose low 21 fraction bits are
// zero: every E2M1 rounding midpoint and grid point is such a value.
__device__ __forceinline__ bool near_grid(float q) {
    return ((__float_as_uint(q) + 8u) & 0x1FFFF0u) == 0u;
}

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

// Eight values with decoded block scale s -> four packed bytes (element 2j in
// the low nibble of byte j).  The quotient is the IEEE single quotient: the
// product with the approximate reciprocal lies within 3 ulps of it, and E2M1
// rounding can only differ near a midpoint or grid point (a value whose low 21
// fraction bits are zero), where the exact division is used.  The test maps
// (bits + 8) mod 2^21 to the top of a word with one multiply-add, so "within
// 8 ulps" is one unsigned comparison of the minimum.  Blocks whose s is
// outside [2^-125, 2^125] use the exact division throughout.
__device__ __forceinline__ uint32_t quantize8(const float (&f)[8], float s) {
    if (s == 0.0f) return 0u;
    float q[8];
    if (s >= 0x1p-125f && s <= 0x1p125f) {
        const float rcp = rcp_approx(s);
        uint32_t mn = 0xFFFFFFFFu;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            q[j] = __fmul_rn(f[j], rcp);
            mn = min(mn, __float_as_uint(q[j]) * 2048u + 16384u);
        }
        if (mn < 32768u) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (near_grid(q[j])) q[j] = __fdiv_rn(f[j], s);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) q[j] = __fdiv_rn(f[j], s);
    }
    return pack4(cvt_e2m1x2(q[0], q[1]), cvt_e2m1x2(q[2], q[3]), cvt_e2m1x2(q[4], q[5]), cvt_e2m1x2(q[6], q[7]));
}

}  // namespace nvfp4
