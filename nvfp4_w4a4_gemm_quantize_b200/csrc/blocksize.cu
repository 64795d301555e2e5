// blocksize.cu -- the measurement behind the per-layer block-size choice of
// "NVFP4-DiT ..." README, Algorithmic framework, Algorithm 1 / Eq. 9:
//   BlockSize(l) = argmin_{b in {1,2,4,8,16,32,64}} Error(l, b) + lambda Memory(b) / Memory_max.
// One pass over a bf16 tensor gives, for every candidate b, the squared error
// sum_j (x_j - Q_b(x)_j)^2 of the two-level NVFP4 quantization with the block
// maximum taken over b values (Q_b(x)_j = e2m1(code_j) * e4m3(sf) * g, codes
// of the IEEE quotient x / s as in the quantize kernel), and sum_j x_j^2; the
// host then applies Eq. 9 (nvfp4_select_block_size).
#include <cuda_runtime.h>

#include "ptx.cuh"
#include "quant_math.cuh"
#include "internal.h"

namespace nvfp4 {

constexpr int kBsThreads = 256;

// E2M1 code -> value (exact): 0.5 m for exponent field 0, else (1 + m/2) 2^(e-1).
__device__ __forceinline__ float e2m1_value(uint32_t c) {
    const uint32_t e = (c >> 1) & 3u, m = c & 1u;
    const float mag = e == 0u ? 0.5f * (float)m : __uint_as_float(((e + 126u) << 23) | (m << 22));
    return (c & 8u) ? -mag : mag;
}

// (x - Q(x))^2 for one element with block scale code sfc: the element's code
// is that of the IEEE quotient x / s; the difference x - e2m1 * dec * g is
// rounded once (FMA) and squared exactly in double.
__device__ __forceinline__ double sq_err(float x, uint32_t sfc, float g) {
    const float dec = e4m3_to_f32(sfc);
    const float s = __fmul_rn(dec, g);
    float v = 0.0f;
    if (s != 0.0f) v = e2m1_value(cvt_e2m1x2(__fdiv_rn(x, s), 0.0f) & 0xFu) * dec;   // exact product
    const float d = __fmaf_rn(-v, g, x);
    return (double)d * (double)d;
}

// One lane per 16-value block of a row (consecutive lanes: consecutive blocks,
// k / 16 a multiple of 4), so the 32- and 64-value maxima come from lane
// shuffles; grid-stride over whole warps so every lane joins the shuffles.
// errors[0..6]: the squared errors for b = 1 .. 64, errors[7]: sum x^2
// (accumulated: the caller zeroes them).
__global__ void __launch_bounds__(kBsThreads)
block_size_errors_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t k, int64_t ld,
                         const float* __restrict__ tensor_scale, double* __restrict__ errors) {
    const ScaleConsts sc = scale_consts(*tensor_scale);
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
        const uint32_t s16 = block_scale_code(m16, sc), s32 = block_scale_code(m32, sc);
        const uint32_t s64 = block_scale_code(m64, sc);
#pragma unroll
        for (int q = 0; q < 2; ++q) {                    // 8-value halves
            float a8 = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j) a8 = fmaxf(a8, fabsf(xs[8 * q + j]));
            const uint32_t s8 = block_scale_code(a8, sc);
#pragma unroll
            for (int h = 0; h < 2; ++h) {                // 4-value quarters
                const int b4 = 8 * q + 4 * h;
                const float a4 = fmaxf(fmaxf(fabsf(xs[b4]), fabsf(xs[b4 + 1])), fmaxf(fabsf(xs[b4 + 2]), fabsf(xs[b4 + 3])));
                const uint32_t s4 = block_scale_code(a4, sc);
#pragma unroll
                for (int p = 0; p < 2; ++p) {            // pairs
                    const int b2 = b4 + 2 * p;
                    const uint32_t s2 = block_scale_code(fmaxf(fabsf(xs[b2]), fabsf(xs[b2 + 1])), sc);
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float xv = xs[b2 + e];
                        acc[0] += sq_err(xv, block_scale_code(fabsf(xv), sc), sc.g);
                        acc[1] += sq_err(xv, s2, sc.g);
                        acc[2] += sq_err(xv, s4, sc.g);
                        acc[3] += sq_err(xv, s8, sc.g);
                        acc[4] += sq_err(xv, s16, sc.g);
                        acc[5] += sq_err(xv, s32, sc.g);
                        acc[6] += sq_err(xv, s64, sc.g);
                        acc[7] += (double)xv * (double)xv;
                    }
                }
            }
        }
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
