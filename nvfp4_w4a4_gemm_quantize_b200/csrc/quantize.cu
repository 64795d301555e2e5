// quantize.cu -- the HBM-bound kernels: tensor amax, NVFP4 two-level
// quantization (scales written in the tensor-core scale-factor layout) and
// dequantization.
//
// Operation (web pages, by title and section):
//  "NVFP4-DiT: Efficient 4-Bit Audio-Guided Video Diffusion Transformers for
//   Low-Cost Video Generation", Methodology 1, Definition III.1:
//   Q_FP4(v; s) = s * clip(round(v/s)_FP4, -6, 6), E2M1 elements, and
//   Methodology 3: two FP4 values per byte.
//  "[RFC]: NVFP4 Quantization Support for Diffusion Models", Motivation:
//   one FP8 scale per 16 values plus one FP32 tensor-level scale.
//
// Arithmetic, fixed so that every code is reproducible bit for bit:
//   g  = amax / 2688                     (6 * 448: E2M1 max times E4M3 max)
//   sf = E4M3_rne_satfinite(a_b / (6 g)),  s = e4m3(sf) * g
//   q  = x / s  (IEEE single quotient)   code = E2M1_rne_satfinite(q)
//
// Fast path for the quotient: q' = x * rn(1/s) lies within 3 ulps of the IEEE
// quotient rn(x/s).  E2M1 rounding only depends on where q sits relative to
// the seven midpoints {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5}; all of them (and
// all grid points) have the low 21 fraction bits clear.  A lane whose q' is
// within 4 ulps of such a value redoes that element with the exact quotient,
// so the code always equals RNE(rn(x/s)).  Blocks whose s is outside
// [2^-125, 2^125] (where 1/s loses bits) take the exact quotient throughout.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "quant_math.cuh"
#include "internal.h"

namespace nvfp4 {

// ------------------------------------------------------------------ amax
// Per-half maxima of |x| over 8 bf16 values (sign bits cleared first).
__device__ __forceinline__ uint32_t absmax_bf16x8(uint4 a) {
    return __vmaxu2(__vmaxu2(a.x & 0x7FFF7FFFu, a.y & 0x7FFF7FFFu),
                    __vmaxu2(a.z & 0x7FFF7FFFu, a.w & 0x7FFF7FFFu));
}

// Partial max |x| per CTA over a [rows, k] bf16 tensor with row stride ld.
// For non-negative IEEE values the bit patterns order like unsigned integers,
// so |x| is the pattern with the sign cleared and the max is an integer max
// on bf16 halves.
__global__ void __launch_bounds__(kAmaxThreads)
amax_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t k, int64_t ld,
            float* __restrict__ partials) {
    const int64_t k8 = k >> 3;                        // 16-byte vectors per row
    const int64_t nvec = rows * k8;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    uint32_t m = 0;                                   // two bf16 |x| maxima
    int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (ld == k) {
        const uint4* p = reinterpret_cast<const uint4*>(x);
        for (; v + 3 * stride < nvec; v += 4 * stride) {
            const uint4 a = __ldcs(p + v), b = __ldcs(p + v + stride);
            const uint4 c = __ldcs(p + v + 2 * stride), d = __ldcs(p + v + 3 * stride);
            m = __vmaxu2(m, __vmaxu2(absmax_bf16x8(a), absmax_bf16x8(b)));
            m = __vmaxu2(m, __vmaxu2(absmax_bf16x8(c), absmax_bf16x8(d)));
        }
        for (; v < nvec; v += stride) m = __vmaxu2(m, absmax_bf16x8(__ldcs(p + v)));
    } else {
        for (; v < nvec; v += stride) {
            const int64_t r = v / k8, c = v - r * k8;
            m = __vmaxu2(m, absmax_bf16x8(__ldcs(reinterpret_cast<const uint4*>(x + r * ld) + c)));
        }
    }
    uint32_t h = max(m & 0xFFFFu, m >> 16);
    for (int o = 16; o > 0; o >>= 1) h = max(h, __shfl_xor_sync(0xffffffffu, h, o));
    __shared__ uint32_t red[kAmaxThreads / 32];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = h;
    __syncthreads();
    if (threadIdx.x < 32) {
        uint32_t t = threadIdx.x < kAmaxThreads / 32 ? red[threadIdx.x] : 0u;
        for (int o = 16; o > 0; o >>= 1) t = max(t, __shfl_xor_sync(0xffffffffu, t, o));
        if (threadIdx.x == 0) partials[blockIdx.x] = __uint_as_float(t << 16);
    }
}

// ------------------------------------------------------------------ quantize
// One CTA quantizes a 128-row x 256-column tile (four 512-byte scale atoms).
// Warp w owns rows 8w .. 8w+7; lane l owns columns 8l .. 8l+7 of a row, so a
// 16-value block is a lane pair and a row is one coalesced 512-byte load.  All
// eight loads of a warp are issued before any is used.
template <bool kDynamic>
__global__ void __launch_bounds__(kQuantThreads)
quantize_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t k, int64_t ld,
                uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                float* __restrict__ tensor_scale, const float* __restrict__ partials, int nparts) {
    __shared__ uint32_t sf_stage[4 * 128];      // 4 atoms x 512 bytes
    __shared__ float g_sh;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (warp == 0) {
        float g;
        if (kDynamic) {
            float mx = 0.0f;
            for (int i = lane; i < nparts; i += 32) mx = fmaxf(mx, partials[i]);
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            g = __fdiv_rn(mx, 2688.0f);
            if (blockIdx.x == 0 && blockIdx.y == 0 && lane == 0) *tensor_scale = g;
        } else {
            g = *tensor_scale;
        }
        if (lane == 0) g_sh = g;
    }
    __syncthreads();
    const float g = g_sh;
    const ScaleConsts sc = scale_consts(g);

    const int64_t row0 = (int64_t)blockIdx.y * 128;
    const int64_t c0 = (int64_t)blockIdx.x * 256;
    const int ncols = (k - c0) < 256 ? (int)(k - c0) : 256;   // multiple of 64
    const bool col_ok = lane * 8 < ncols;
    const int64_t kh = k >> 1;

    constexpr int kRows = 128 / (kQuantThreads / 32);   // rows per warp
    uint4 v[kRows];
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
        const int64_t r = row0 + warp * kRows + i;
        if (r < rows && col_ok)
            v[i] = __ldcs(reinterpret_cast<const uint4*>(x + r * ld + c0) + lane);
        else
            v[i] = make_uint4(0u, 0u, 0u, 0u);
    }

#pragma unroll
    for (int i = 0; i < kRows; ++i) {
        const int rt = warp * kRows + i;             // row inside the tile
        const int64_t r = row0 + rt;
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
        // block amax over the lane pair (integer max of |bf16| patterns)
        const uint32_t mm = absmax_bf16x8(v[i]);
        uint32_t hb = max(mm & 0xFFFFu, mm >> 16);
        hb = max(hb, __shfl_xor_sync(0xffffffffu, hb, 1));
        const float ab = __uint_as_float(hb << 16);

        const uint32_t sfc = block_scale_code(ab, sc);
        const float s = __fmul_rn(e4m3_to_f32(sfc), g);
        float f[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            f[2 * j] = __uint_as_float(w[j] << 16);
            f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
        const uint32_t packed = quantize8(f, s);
        if (r < rows && col_ok)
            *reinterpret_cast<uint32_t*>(codes + r * kh + (c0 >> 1) + lane * 4) = packed;

        // scale bytes of blocks 4a..4a+3 live on lanes 8a, 8a+2, 8a+4, 8a+6
        const uint32_t b1 = __shfl_down_sync(0xffffffffu, sfc, 2);
        const uint32_t b2 = __shfl_down_sync(0xffffffffu, sfc, 4);
        const uint32_t b3 = __shfl_down_sync(0xffffffffu, sfc, 6);
        if ((lane & 7) == 0 && col_ok) {
            const int a = lane >> 3;
            sf_stage[a * 128 + (rt & 31) * 4 + (rt >> 5)] = sfc | (b1 << 8) | (b2 << 16) | (b3 << 24);
        }
    }
    __syncthreads();
    // this tile's atoms are consecutive in the scale buffer
    const int natoms = ncols >> 6;
    const int64_t kb4 = k >> 6;                       // atoms per 128-row block
    uint32_t* dst = reinterpret_cast<uint32_t*>(sf + (((int64_t)blockIdx.y * kb4 + blockIdx.x * 4) << 9));
    for (int i = threadIdx.x; i < natoms * 128; i += kQuantThreads) dst[i] = sf_stage[i];
}

// ------------------------------------------------------------------ dequantize
// One thread per 8 elements.  e = e2m1 * e4m3 is exact in FP32; the product
// with g is formed exactly in double and rounded once to the output type
// (bf16 through an FP32 round-to-odd intermediate, which is innocuous with 16
// spare bits).
template <bool kBF16>
__global__ void __launch_bounds__(256)
dequantize_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf,
                  const float* __restrict__ tensor_scale, int64_t rows, int64_t k, void* __restrict__ out) {
    __shared__ float lut[16];
    if (threadIdx.x < 16) {
        const uint32_t c = threadIdx.x, e = (c >> 1) & 3u, m = c & 1u;
        float mag = (e == 0) ? 0.5f * (float)m : ldexpf(1.0f + 0.5f * (float)m, (int)e - 1);
        lut[c] = (c & 8u) ? -mag : mag;
    }
    __syncthreads();
    const double g = (double)*tensor_scale;
    const int64_t k8 = k >> 3, kb = k >> 4;
    const int64_t nvec = rows * k8;
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nvec;
         v += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = v / k8, c8 = v - r * k8;
        const int64_t blk = c8 >> 1;
        const uint32_t word = *reinterpret_cast<const uint32_t*>(codes + r * (k >> 1) + c8 * 4);
        const int64_t off = ((r >> 7) * (kb >> 2) + (blk >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (blk & 3);
        const float s = e4m3_to_f32(sf[off]);
        float o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float e = __fmul_rn(lut[(word >> (4 * j)) & 15u], s);   // exact
            const double p = (double)e * g;                              // exact
            if (kBF16) {
                float t = __double2float_rz(p);
                if ((double)t != p) t = __uint_as_float(__float_as_uint(t) | 1u);
                o[j] = t;
            } else {
                o[j] = __double2float_rn(p);
            }
        }
        if (kBF16) {
            uint4 pk;
            uint32_t* pw = &pk.x;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                __nv_bfloat162 h = __floats2bfloat162_rn(o[2 * j], o[2 * j + 1]);
                pw[j] = *reinterpret_cast<uint32_t*>(&h);
            }
            reinterpret_cast<uint4*>(out)[v] = pk;
        } else {
            float4* po = reinterpret_cast<float4*>(out) + 2 * v;
            po[0] = make_float4(o[0], o[1], o[2], o[3]);
            po[1] = make_float4(o[4], o[5], o[6], o[7]);
        }
    }
}

// ------------------------------------------------------------------ launchers
int amax_grid(int64_t rows, int64_t k) {
    const int64_t nvec = rows * (k >> 3);
    int64_t g = (nvec + kAmaxThreads * 8 - 1) / (kAmaxThreads * 8);
    if (g < 1) g = 1;
    if (g > kAmaxMaxCtas) g = kAmaxMaxCtas;
    return (int)g;
}

cudaError_t launch_quantize(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, uint8_t* codes,
                            uint8_t* sf, float* tensor_scale, bool scale_given, float* partials,
                            cudaStream_t stream) {
    const dim3 grid((unsigned)((k + 255) / 256), (unsigned)((rows + 127) / 128));
    if (scale_given) {
        quantize_kernel<false><<<grid, kQuantThreads, 0, stream>>>(x, rows, k, ld, codes, sf, tensor_scale,
                                                                  nullptr, 0);
        count_launch(1);
        return cudaGetLastError();
    }
    const int ag = amax_grid(rows, k);
    amax_kernel<<<ag, kAmaxThreads, 0, stream>>>(x, rows, k, ld, partials);
    quantize_kernel<true><<<grid, kQuantThreads, 0, stream>>>(x, rows, k, ld, codes, sf, tensor_scale,
                                                             partials, ag);
    count_launch(2);
    return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* sf, const float* tensor_scale, int64_t rows,
                              int64_t k, void* out, bool bf16, cudaStream_t stream) {
    const int64_t nvec = rows * (k >> 3);
    int64_t g = (nvec + 255) / 256;
    if (g > 148 * 16) g = 148 * 16;
    if (g < 1) g = 1;
    if (bf16)
        dequantize_kernel<true><<<(unsigned)g, 256, 0, stream>>>(codes, sf, tensor_scale, rows, k, out);
    else
        dequantize_kernel<false><<<(unsigned)g, 256, 0, stream>>>(codes, sf, tensor_scale, rows, k, out);
    count_launch(1);
    return cudaGetLastError();
}

}  // namespace nvfp4
