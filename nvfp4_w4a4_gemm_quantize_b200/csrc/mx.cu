// mx.cu -- the MX variant of the quantizer: E2M1 elements in blocks of 32
// along k with one power-of-two (unsigned E8M0) scale per block and no tensor
// scale, the format the block32 tensor-core MMA (kind::mxf4) reads; and its
// dequantization.
//
// Source: "[RFC]: NVFP4 Quantization Support for Diffusion Models" names the
// MXFP4 format as the related, different one; the scale rule is the OCP
// Microscaling specification's:
//   e = floor(log2(max|x|)) - 2  (2: E2M1's largest exponent), clamped to
//   [-127, 127] (-127 for an all-zero block); byte = e + 127;
//   code = E2M1_rne_satfinite(x / 2^e), sign of x kept.
// For a bf16 block maximum with exponent field E, floor(log2) = E - 127 (a
// subnormal or zero maximum clamps), so byte = max(E - 2, 0); x / 2^e is a
// multiplication by an exact power of two, so no quotient rounding arises
// (products below FP32's normal range are far below E2M1's 0.25).
#include <cuda_runtime.h>

#include "ptx.cuh"
#include "quant_math.cuh"
#include "internal.h"

namespace nvfp4 {

// One warp covers 8 rows x 128 columns: lane l takes row l / 4 and the
// 32-value block l % 4 (four 16-byte loads; the four lanes of a row read 256
// contiguous bytes), and the row's four scale bytes form one word of the
// scale layout, gathered by shuffles and written by the row's first lane.
constexpr int kMxThreads = 256;
constexpr int kMxRowsPerCta = 8 * (kMxThreads / 32);

__global__ void __launch_bounds__(kMxThreads)
mx_quantize_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t k, int64_t ld, uint8_t* __restrict__ codes,
                   uint8_t* __restrict__ sf) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.y * kMxRowsPerCta + warp * 8 + (lane >> 2);
    const int64_t c0 = (int64_t)blockIdx.x * 128 + (lane & 3) * 32;    // first column of the lane's block
    const bool ok = r < rows;
    uint4 v[4];
    const uint4* src = reinterpret_cast<const uint4*>(x + (ok ? r : 0) * ld + c0);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = ok ? __ldcs(src + i) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t w[16] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w,
                            v[2].x, v[2].y, v[2].z, v[2].w, v[3].x, v[3].y, v[3].z, v[3].w};
    uint32_t m = 0u;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = absmax_bf16x2(m, w[i]);
    const uint32_t hmax = max(m & 0x7FFFu, (m >> 16) & 0x7FFFu);          // |max| bf16 pattern
    const uint32_t ef = hmax >> 7;                                         // its exponent field
    const uint32_t byte = ef > 2u ? ef - 2u : 0u;                          // e + 127
    const float inv = __uint_as_float((254u - byte) << 23);                // 2^-e, e = byte - 127
    const uint64_t inv2 = f32x2(inv, inv);
    uint32_t cw[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint64_t p[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t u = w[4 * q + j];
            p[j] = mul_f32x2(f32x2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u)), inv2);
        }
        cw[q] = cvt_e2m1x8(p[0], p[1], p[2], p[3]);
    }
    if (ok) *reinterpret_cast<uint4*>(codes + r * (k >> 1) + (c0 >> 1)) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    // the row's four scale bytes (blocks 4c .. 4c+3) -> one word
    const int base = lane & ~3;
    const uint32_t b0 = __shfl_sync(0xffffffffu, byte, base), b1 = __shfl_sync(0xffffffffu, byte, base + 1);
    const uint32_t b2 = __shfl_sync(0xffffffffu, byte, base + 2), b3 = __shfl_sync(0xffffffffu, byte, base + 3);
    if ((lane & 3) == 0) {                       // the grid covers exactly the rows padded to 128
        const int64_t kb4 = k >> 7;                                        // words per 128-row block
        const int64_t atom = (r >> 7) * kb4 + blockIdx.x;
        const int rr = (int)(r & 127);
        *reinterpret_cast<uint32_t*>(sf + atom * 512 + (rr & 31) * 16 + (rr >> 5) * 4) =
            b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
    }
}

// v = e2m1(code) * 2^(byte - 127): exact in FP32 and in bf16 (two significant
// bits, exponent within [-128, 127]).  One thread per 8 values.
template <bool kBF16>
__global__ void __launch_bounds__(256)
mx_dequantize_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf, int64_t rows, int64_t k,
                     void* __restrict__ out) {
    const int64_t k8 = k >> 3, kb = k >> 5;
    const int64_t nvec = rows * k8;
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nvec;
         v += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = v / k8, c8 = v - r * k8;
        const int64_t blk = c8 >> 2;
        const uint32_t word = *reinterpret_cast<const uint32_t*>(codes + r * (k >> 1) + c8 * 4);
        const int64_t off = ((r >> 7) * (kb >> 2) + (blk >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (blk & 3);
        const int e = (int)sf[off] - 127;
        float o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t c = (word >> (4 * j)) & 15u, ex = (c >> 1) & 3u, mb = c & 1u;
            const float mag = ex == 0 ? 0.5f * (float)mb : ldexpf(1.0f + 0.5f * (float)mb, (int)ex - 1);
            o[j] = ldexpf((c & 8u) ? -mag : mag, e);                       // exact
        }
        if (kBF16) {
            uint4 pk;
            uint32_t* pw = &pk.x;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                pw[j] = (__float_as_uint(o[2 * j]) >> 16) | (__float_as_uint(o[2 * j + 1]) & 0xFFFF0000u);
            reinterpret_cast<uint4*>(out)[v] = pk;
        } else {
            float4* po = reinterpret_cast<float4*>(out) + 2 * v;
            po[0] = make_float4(o[0], o[1], o[2], o[3]);
            po[1] = make_float4(o[4], o[5], o[6], o[7]);
        }
    }
}

cudaError_t launch_mx_quantize(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, uint8_t* codes, uint8_t* sf,
                               cudaStream_t stream) {
    // the grid covers the rows padded to 128, so the padding rows' scale
    // words are written as zeros by the kernel itself
    const int64_t rpad = ((rows + 127) / 128) * 128;
    const dim3 grid((unsigned)(k / 128), (unsigned)(rpad / kMxRowsPerCta));
    mx_quantize_kernel<<<grid, kMxThreads, 0, stream>>>(x, rows, k, ld, codes, sf);
    count_launch(1);
    return cudaGetLastError();
}

cudaError_t launch_mx_dequantize(const uint8_t* codes, const uint8_t* sf, int64_t rows, int64_t k, void* out,
                                 bool bf16, int num_sms, cudaStream_t stream) {
    const int64_t nvec = rows * (k >> 3);
    int64_t g = (nvec + 255) / 256;
    if (g > (int64_t)num_sms * 16) g = (int64_t)num_sms * 16;
    if (g < 1) g = 1;
    if (bf16)
        mx_dequantize_kernel<true><<<(unsigned)g, 256, 0, stream>>>(codes, sf, rows, k, out);
    else
        mx_dequantize_kernel<false><<<(unsigned)g, 256, 0, stream>>>(codes, sf, rows, k, out);
    count_launch(1);
    return cudaGetLastError();
}

}  // namespace nvfp4
