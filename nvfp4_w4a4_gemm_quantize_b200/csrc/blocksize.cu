// blocksize.cu -- the measurement behind the per-layer block-size choice of
// "NVFP4-DiT ..." README, Algorithmic framework, Algorithm 1 / Eq. 9:
//   BlockSize(l) = argmin_{b in {1,2,4,8,16,32,64}} Error(l, b) + lambda Memory(b) / Memory_max.
// One pass over a bf16 tensor gives, for every candidate b, the squared error
// sum_j (x_j - Q_b(x)_j)^2 of the two-level NVFP4 quantization with the block
// maximum taken over b values (Q_b(x)_j = e2m1(code_j) * e4m3(sf) * g, codes
// of the IEEE quotient x / s as in the quantize kernel, found through the same
// reciprocal bracket), and sum_j x_j^2; the host then applies Eq. 9
// (nvfp4_select_block_size).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"
#include "quant_math.cuh"
#include "internal.h"

namespace nvfp4 {

constexpr int kBsThreads = 256;

// Scale code -> the exact e4m3 value and the decoded scale s = e4m3(sfc) * g.
struct BlockScale {
    float dec, s;
};

__device__ __forceinline__ BlockScale block_scale(uint32_t sfc, float g) {
    const float dec = e4m3_to_f32(sfc);
    return {dec, __fmul_rn(dec, g)};
}

// E2M1 code of the IEEE quotient x / s (0 when s is 0): the rare exact path,
// kept out of line so that the unrolled pair loops stay small.
__device__ __noinline__ uint32_t exact_code(float x, float s) {
    return s == 0.0f ? 0u : cvt_e2m1x2(__fdiv_rn(x, s), 0.0f) & 0x0Fu;
}

// E2M1 codes of the IEEE quotients x0 / s0 and x1 / s1 (x0 in bits 0-3, x1 in
// bits 4-7; 0 where s is 0).  The reciprocal bracket of the quantize kernel
// gives lower and upper bounds of each quotient; where their codes agree that
// is the code of the quotient (rounding is monotone in magnitude), elsewhere,
// and for s outside the bracket's range, the quotient is formed exactly.
__device__ __forceinline__ uint32_t codes2(float x0, float x1, float s0, float s1) {
    if (!(bracket_ok(s0) && bracket_ok(s1))) return exact_code(x0, s0) | (exact_code(x1, s1) << 4);
    const uint32_t r0 = __float_as_uint(rcp_approx(s0)), r1 = __float_as_uint(rcp_approx(s1));
    uint32_t c = cvt_e2m1x2(__fmul_rn(x0, __uint_as_float(r0 - 4u)), __fmul_rn(x1, __uint_as_float(r1 - 4u))) & 0xFFu;
    const uint32_t ch =
        cvt_e2m1x2(__fmul_rn(x0, __uint_as_float(r0 + 4u)), __fmul_rn(x1, __uint_as_float(r1 + 4u))) & 0xFFu;
    if (c != ch) {
        if ((c ^ ch) & 0x0Fu) c = (c & 0xF0u) | exact_code(x0, s0);
        if ((c ^ ch) & 0xF0u) c = (c & 0x0Fu) | (exact_code(x1, s1) << 4);
    }
    return c;
}

// (x0 - Q(x0))^2 + (x1 - Q(x1))^2 in FP32 for one pair: Q(x) = e2m1(code) *
// e4m3 * g, the first product exact, x - Q(x) rounded once (FMA).  The two
// codes are decoded exactly through the packed f16 conversion.
__device__ __forceinline__ float sq_err2(float x0, float x1, const BlockScale& b0, const BlockScale& b1, float g) {
    const uint32_t c = codes2(x0, x1, b0.s, b1.s);
    uint32_t h2;
    asm("{\n\t.reg .b8 cb;\n\tcvt.u8.u32 cb, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, cb;\n\t}" : "=r"(h2) : "r"(c));
    const float v0 = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu))) * b0.dec;   // exact
    const float v1 = __half2float(__ushort_as_half((unsigned short)(h2 >> 16))) * b1.dec;
    const float d0 = __fmaf_rn(-v0, g, x0), d1 = __fmaf_rn(-v1, g, x1);
    return __fmaf_rn(d0, d0, d1 * d1);
}

// One lane per 16-value block of a row (consecutive lanes: consecutive blocks,
// k / 16 a multiple of 4), so the 32- and 64-value maxima come from lane
// shuffles; grid-stride over whole warps so every lane joins the shuffles.
// Per lane and block size the 16 squared errors are summed in FP32 (relative
// rounding below 1e-6), then added in double.
// errors[0..6]: the squared errors for b = 1 .. 64, errors[7]: sum x^2
// (accumulated: the caller zeroes them).
__global__ void __launch_bounds__(kBsThreads)
block_size_errors_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t k, int64_t ld,
                         const float* __restrict__ tensor_scale, double* __restrict__ errors) {
    const ScaleConsts sc = scale_consts(*tensor_scale);
    const float g = sc.g;
    const int lane = threadIdx.x & 31;
    const int64_t kb = k >> 4;
    const int64_t total = rows * kb;
    double acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t t0 = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); t0 < total; t0 += stride) {
        const int64_t t = t0 + lane;
        const bool ok = t < total;
        const int64_t r = ok ? t / kb : 0, c = ok ? t - r * kb : 0;
        uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
        if (ok) {
            const uint4* p = reinterpret_cast<const uint4*>(x + r * ld + c * 16);
            v0 = __ldcs(p);
            v1 = __ldcs(p + 1);
        }
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        float xs[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            xs[2 * j] = __uint_as_float(w[j] << 16);
            xs[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
        const float m16 = __uint_as_float(block_absmax16(w) << 16);
        const float m32 = fmaxf(m16, __shfl_xor_sync(0xffffffffu, m16, 1));
        const float m64 = fmaxf(m32, __shfl_xor_sync(0xffffffffu, m32, 2));
        if (!ok) continue;
        const BlockScale b16 = block_scale(block_scale_code(m16, sc), g);
        const BlockScale b32 = block_scale(block_scale_code(m32, sc), g);
        const BlockScale b64 = block_scale(block_scale_code(m64, sc), g);
        float e[7] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
        double ss = 0.0;
#pragma unroll
        for (int q = 0; q < 2; ++q) {                    // 8-value halves
            float a8 = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j) a8 = fmaxf(a8, fabsf(xs[8 * q + j]));
            const BlockScale b8 = block_scale(block_scale_code(a8, sc), g);
#pragma unroll
            for (int h = 0; h < 2; ++h) {                // 4-value quarters
                const int i4 = 8 * q + 4 * h;
                const float a4 = fmaxf(fmaxf(fabsf(xs[i4]), fabsf(xs[i4 + 1])), fmaxf(fabsf(xs[i4 + 2]), fabsf(xs[i4 + 3])));
                const BlockScale b4 = block_scale(block_scale_code(a4, sc), g);
#pragma unroll
                for (int pp = 0; pp < 2; ++pp) {         // pairs
                    const int i2 = i4 + 2 * pp;
                    const float x0 = xs[i2], x1 = xs[i2 + 1];
                    const BlockScale b2 = block_scale(block_scale_code(fmaxf(fabsf(x0), fabsf(x1)), sc), g);
                    const BlockScale e0 = block_scale(block_scale_code(fabsf(x0), sc), g);
                    const BlockScale e1 = block_scale(block_scale_code(fabsf(x1), sc), g);
                    e[0] += sq_err2(x0, x1, e0, e1, g);
                    e[1] += sq_err2(x0, x1, b2, b2, g);
                    e[2] += sq_err2(x0, x1, b4, b4, g);
                    e[3] += sq_err2(x0, x1, b8, b8, g);
                    e[4] += sq_err2(x0, x1, b16, b16, g);
                    e[5] += sq_err2(x0, x1, b32, b32, g);
                    e[6] += sq_err2(x0, x1, b64, b64, g);
                    ss = fma((double)x0, (double)x0, fma((double)x1, (double)x1, ss));
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 7; ++i) acc[i] += (double)e[i];
        acc[7] += ss;
    }
    // warp sums, then one atomic per warp and quantity
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        double v = acc[i];
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) atomicAdd(errors + i, v);
    }
}

cudaError_t launch_block_size_errors(const uint16_t* x, int64_t rows, int64_t k, int64_t ld,
                                     const float* tensor_scale, double* errors, int num_sms, cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(errors, 0, 8 * sizeof(double), stream);
    if (e != cudaSuccess) return e;
    const int64_t total = rows * (k / 16);
    int64_t g = (total + kBsThreads - 1) / kBsThreads;
    if (g > (int64_t)num_sms * 8) g = (int64_t)num_sms * 8;
    if (g < 1) g = 1;
    block_size_errors_kernel<<<(unsigned)g, kBsThreads, 0, stream>>>(x, rows, k, ld, tensor_scale, errors);
    count_launch(1);
    return cudaGetLastError();
}

}  // namespace nvfp4
