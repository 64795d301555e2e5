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

// True when q is within 4 ulps of a value whose low 21 fraction bits are zero:
// every E2M1 rounding midpoint and grid point is such a value.
__device__ __forceinline__ bool near_grid(float q) {
    return ((__float_as_uint(q) + 4u) & 0x1FFFFFu) <= 8u;
}

// E4M3 block-scale code for block max `ab` (d = 6 g).
__device__ __forceinline__ uint32_t block_scale_code(float ab, float d) {
    return d > 0.0f ? cvt_e4m3(__fdiv_rn(ab, d)) : 0u;
}

// Eight values with decoded block scale s -> four packed bytes (element 2j in
// the low nibble of byte j).  The quotient is the IEEE single quotient: the
// reciprocal product is used where it provably rounds the same way, the exact
// division elsewhere (see near_grid).
__device__ __forceinline__ uint32_t quantize8(const float (&f)[8], float s) {
    if (s == 0.0f) return 0u;
    float q[8];
    if (s >= 0x1p-125f && s <= 0x1p125f) {
        const float rcp = __frcp_rn(s);
        bool redo = false;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            q[j] = __fmul_rn(f[j], rcp);
            redo |= near_grid(q[j]);
        }
        if (redo) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (near_grid(q[j])) q[j] = __fdiv_rn(f[j], s);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) q[j] = __fdiv_rn(f[j], s);
    }
    uint32_t packed = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) packed |= cvt_e2m1x2(q[2 * j], q[2 * j + 1]) << (8 * j);
    return packed;
}

}  // namespace nvfp4
