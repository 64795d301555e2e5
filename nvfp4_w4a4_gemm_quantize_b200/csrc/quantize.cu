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
// The quotient is bracketed by two products with a reciprocal bracket of s,
// on packed FP32 pairs; where the two bounds give the same code it is the
// code of the IEEE quotient, otherwise the values are divided exactly (see
// quant_math.cuh).
#include <atomic>
#include <cstdlib>

#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "quant_math.cuh"
#include "internal.h"
#include "tmap.h"

namespace nvfp4 {

// ------------------------------------------------------------------ amax
// Largest magnitude of two packed bf16 pairs, per half, with NaN propagation
// (a NaN operand gives NaN).  For the tensor amax: finite inputs give the
// same maximum as any other order, and an Inf or NaN anywhere leaves a half
// with the all-ones exponent, which flags the input as non-finite (the
// contract's inputs are finite; the scale is then unspecified).
__device__ __forceinline__ uint32_t absmax_nan_bf16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Per-half largest magnitude of 8 bf16 values (sign bits not meaningful).
__device__ __forceinline__ uint32_t absmax_bf16x8(uint4 a) {
    return absmax_nan_bf16x2(absmax_nan_bf16x2(a.x, a.y), absmax_nan_bf16x2(a.z, a.w));
}

// Partial max |x| per CTA over a [rows, k] bf16 tensor with row stride ld,
// on bf16 pairs (max.NaN.xorsign.abs).  The final per-CTA value compares
// non-negative bf16 patterns as integers (for non-negative IEEE values the
// order of the patterns is the order of the values); a value with the
// all-ones exponent means an Inf or NaN was read.
__global__ void __launch_bounds__(kAmaxThreads)
amax_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t k, int64_t ld,
            float* __restrict__ partials, int* __restrict__ dev_status) {
    // the quantize kernel that follows may start (and load X) now; it waits
    // for this grid's results before it reads the partial maxima
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t k8 = k >> 3;                        // 16-byte vectors per row
    const int64_t nvec = rows * k8;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    uint32_t m = 0;                                   // two bf16 |x| maxima
    int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (ld == k) {
        const uint4* p = reinterpret_cast<const uint4*>(x);
        for (; v + 3 * stride < nvec; v += 4 * stride) {
            const uint4 a = __ldg(p + v), b = __ldg(p + v + stride);
            const uint4 c = __ldg(p + v + 2 * stride), d = __ldg(p + v + 3 * stride);
            m = absmax_nan_bf16x2(m, absmax_nan_bf16x2(absmax_bf16x8(a), absmax_bf16x8(b)));
            m = absmax_nan_bf16x2(m, absmax_nan_bf16x2(absmax_bf16x8(c), absmax_bf16x8(d)));
        }
        for (; v < nvec; v += stride) m = absmax_nan_bf16x2(m, absmax_bf16x8(__ldg(p + v)));
    } else {
        for (; v < nvec; v += stride) {
            const int64_t r = v / k8, c = v - r * k8;
            m = absmax_nan_bf16x2(m, absmax_bf16x8(__ldg(reinterpret_cast<const uint4*>(x + r * ld) + c)));
        }
    }
    m &= 0x7FFF7FFFu;
    // any Inf or NaN: flag it (the first error written stays)
    const bool nonfinite = (m & 0xFFFFu) >= 0x7F80u || (m >> 16) >= 0x7F80u;
    if (__syncthreads_or(nonfinite ? 1 : 0) && threadIdx.x == 0 && dev_status)
        atomicCAS(dev_status, 0, (int)NVFP4_ERR_NONFINITE);
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
// A tile is 128 rows x 256 columns (four 512-byte scale atoms) handled by one
// 512-thread CTA.  Warp w owns rows 8w .. 8w+7, two rows per step: lanes 0-15
// one row, lanes 16-31 the next, lane l owning the 16-value block l % 16 of
// its row (two 16-byte loads; a row is one coalesced 512-byte span).  A lane
// therefore holds a whole block: its maximum, scale and reciprocal are
// computed once per 16 values without any shuffle.
constexpr int kTileRows = 128;
constexpr int kTileCols = 256;
constexpr int kRows = kTileRows / (kQuantThreads / 32);   // rows per warp
constexpr int kSteps = kRows / 2;
// four 512-byte atoms, each padded by 4 bytes so that the eight words two
// rows write (one per atom and row) fall in different banks
constexpr int kAtomPitch = 516;

// Per-lane view of one tile: step i handles row rt0 + 2i of the tile; the
// input pointer is for step 0 and advances by two rows per step (ld is a
// multiple of 8).  e0 is the index of the lane's first value in a contiguous
// [rows, k] layout, from which each output places its results.
struct TileLane {
    const uint4* xp;
    int64_t xstep, rows_left, e0;
    int sbase;
    bool col_ok;
};

__device__ __forceinline__ TileLane tile_lane(const uint16_t* x, int64_t rows, int64_t k, int64_t ld,
                                              int64_t rblk, int64_t cblk, int warp, int lane) {
    TileLane t;
    const int64_t c0 = cblk * kTileCols;
    const int ncols = (k - c0) < kTileCols ? (int)(k - c0) : kTileCols;   // multiple of 64
    const int half = lane >> 4, blk = lane & 15;
    const int rt0 = warp * kRows + half;
    const int64_t r0 = rblk * kTileRows + rt0;
    t.col_ok = blk * 16 < ncols;
    t.rows_left = rows - r0;                      // step i is in range iff 2i < rows_left
    t.xp = reinterpret_cast<const uint4*>(x + r0 * ld + c0) + 2 * blk;
    t.xstep = ld >> 2;                            // two rows, in 16-byte units
    t.e0 = r0 * k + c0 + 16 * blk;
    // block blk of row rt: atom blk / 4, byte blk % 4 of the row's word
    t.sbase = (blk >> 2) * kAtomPitch + (rt0 & 31) * 16 + (rt0 >> 5) * 4 + (blk & 3);
    return t;
}

// All loads of a lane for one tile (rows beyond the tensor and columns beyond
// k read as zeros).
__device__ __forceinline__ void load_tile(const TileLane& t, uint4 (&v)[2 * kSteps]) {
#pragma unroll
    for (int i = 0; i < kSteps; ++i) {
        if (2 * i < t.rows_left && t.col_ok) {
            v[2 * i] = __ldcs(t.xp + i * t.xstep);
            v[2 * i + 1] = __ldcs(t.xp + i * t.xstep + 1);
        } else {
            v[2 * i] = make_uint4(0u, 0u, 0u, 0u);
            v[2 * i + 1] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
}

// Copy a tile's staged scale atoms (consecutive in the scale buffer) out, one
// word per thread.  The caller synchronizes the CTA before and after.
__device__ __forceinline__ void store_tile_scales(const uint8_t* sf_stage, uint8_t* sf, int64_t k, int64_t rblk,
                                                  int64_t cblk) {
    static_assert(4 * 128 <= kQuantThreads, "scale copy-out: one word per thread");
    const int64_t c0 = cblk * kTileCols;
    const int ncols = (k - c0) < kTileCols ? (int)(k - c0) : kTileCols;
    const int natoms = ncols >> 6;
    const int64_t kb4 = k >> 6;                   // atoms per 128-row block
    uint32_t* dst = reinterpret_cast<uint32_t*>(sf + ((rblk * kb4 + cblk * 4) << 9));
    const int i = threadIdx.x;
    if (i < natoms * 128) dst[i] = *reinterpret_cast<const uint32_t*>(sf_stage + (i >> 7) * kAtomPitch + (i & 127) * 4);
}

// ---------------------------------------------------------------- outputs
// What a lane does with a quantized block.  Each output type gives a per-lane
// view (pointers for step 0 and their two-row advance) and emit(), called once
// per step with the block's bf16 words, scale code, decoded scale s and codes.

// nvfp4_quantize: packed codes straight to global memory (8 bytes per block);
// scale bytes staged per tile in the tensor-core layout.
struct CodesOut {
    uint8_t* codes;
    uint8_t* sf;
    static constexpr bool kScales = true;
    static constexpr int kMinBlocks = 0;          // unforced: the compiler fits 64 registers (2 CTAs per SM)
    static constexpr int kGroup = 1;              // lanes (16-value blocks) per scale block
    struct Lane {
        uint2* cp;
        int64_t step;
    };
    __device__ __forceinline__ Lane lane(const TileLane& t, int64_t k) const {
        return {reinterpret_cast<uint2*>(codes) + (t.e0 >> 4), k >> 3};
    }
    __device__ __forceinline__ void emit(const Lane& l, int i, bool ok, const uint32_t (&)[8], uint32_t, float,
                                         uint32_t lo, uint32_t hi, const ScaleConsts&) const {
        if (ok) l.cp[i * l.step] = make_uint2(lo, hi);
    }
    __device__ __forceinline__ void store_scales(const uint8_t* sf_stage, int64_t k, int64_t rblk,
                                                 int64_t cblk) const {
        store_tile_scales(sf_stage, sf, k, rblk, cblk);
    }
};

// Codes and scales with one scale per G consecutive 16-value blocks (blocks
// of 32 or 64 values along k): the G lanes of a scale block share its
// maximum, and each writes the shared scale byte into its own 16-block slot,
// so the block-16 GEMM reads the result unchanged.
template <int G>
struct CodesOutG : CodesOut {
    static constexpr int kGroup = G;
};

// f16x2 of two E2M1 codes (one byte, the low nibble in the low half) times
// the block's decoded scale (f16 in both halves of sd2): exact, since the
// product has at most 6 significant bits and lies within [2^-10, 2688].
__device__ __forceinline__ uint32_t e2m1x2_times_scale(uint32_t byte, uint32_t sd2) {
    uint32_t h2, e2;
    asm("{\n\t.reg .b8 c;\n\t"
        "cvt.u8.u32 c, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, c;\n\t}"
        : "=r"(h2)
        : "r"(byte));
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(e2) : "r"(h2), "r"(sd2));
    return e2;
}

// E4M3 scale byte -> f16 in both halves (exact).
__device__ __forceinline__ uint32_t e4m3_to_f16x2(uint32_t sfc) {
    uint32_t sd2;
    const uint16_t in = (uint16_t)(sfc | (sfc << 8));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(sd2) : "h"(in));
    return sd2;
}

// The two halves of an f16x2 as a packed FP32 pair (low half first).
__device__ __forceinline__ uint64_t f16x2_to_f32x2(uint32_t h2) {
    uint64_t r;
    asm("{\n\t.reg .f16 a, b;\n\t.reg .f32 fa, fb;\n\t"
        "mov.b32 {a, b}, %1;\n\t"
        "cvt.f32.f16 fa, a;\n\t"
        "cvt.f32.f16 fb, b;\n\t"
        "mov.b64 %0, {fa, fb};\n\t}"
        : "=l"(r)
        : "r"(h2));
    return r;
}

// bf16x2 of e * g rounded once (RNE) for a packed pair e of exact FP32
// values, ng2 = (-g, -g): the product truncated to FP32 is made odd when the
// residual e*g - rz(e*g) (exact by the FMA) is not zero, and that
// round-to-odd value, with 16 spare bits, rounds to bf16 as the exact product
// would.  Valid while every nonzero |e * g| >= 2^-120 (the residual is then
// representable); e == 0 gives a zero of e's sign.
__device__ __forceinline__ uint32_t bf16x2_round_once(uint64_t e2, uint64_t g2, uint64_t ng2) {
    uint64_t t, r;
    asm("mul.rz.f32x2 %0, %1, %2;" : "=l"(t) : "l"(e2), "l"(g2));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(e2), "l"(ng2), "l"(t));
    uint32_t tl, th, rl, rh, out;
    asm("mov.b64 {%0, %1}, %2;" : "=r"(tl), "=r"(th) : "l"(t));
    asm("mov.b64 {%0, %1}, %2;" : "=r"(rl), "=r"(rh) : "l"(r));
    tl |= (rl << 1) != 0u ? 1u : 0u;
    th |= (rh << 1) != 0u ? 1u : 0u;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(out) : "f"(__uint_as_float(th)), "f"(__uint_as_float(tl)));
    return out;
}

// The same for blocks with a tiny scale: the product formed exactly in
// double, truncated to FP32 with the sticky bit, then rounded to bf16.
__device__ __forceinline__ uint32_t bf16x2_round_once_slow(uint64_t e2, float g) {
    uint32_t el, eh, out;
    asm("mov.b64 {%0, %1}, %2;" : "=r"(el), "=r"(eh) : "l"(e2));
    float v[2];
    const uint32_t e[2] = {el, eh};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const double p = (double)__uint_as_float(e[h]) * (double)g;    // exact
        float t = __double2float_rz(p);
        if ((double)t != p) t = __uint_as_float(__float_as_uint(t) | 1u);
        v[h] = t;
    }
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(out) : "f"(v[1]), "f"(v[0]));
    return out;
}

// Per-block table of the bf16 results y = RN_bf16(v * e4m3(sf) * g) for the
// eight E2M1 magnitudes v = 0, 0.5, 1, 1.5, 2, 3, 4, 6 (magnitude code m),
// as byte planes for prmt lookups: lo0 / lo1 hold the low bytes of entries
// 0-3 / 4-7, hi0 / hi1 the high bytes.  With b1 = RN_bf16(S) and
// b3 = RN_bf16(1.5 S), S = e4m3(sf) * g exact, every entry is b1 or b3 times
// a power of two (v = 2^j or 1.5 * 2^j), and scaling a normal bf16 by 2^j is
// an exponent add that commutes with rounding -- valid while 0.5 b1 and 4 b3
// stay normal and finite, i.e. for s in [2^-118, 2^124].
struct ValueTable {
    uint32_t lo0, lo1, hi0, hi1;
};

__device__ __forceinline__ ValueTable value_table(float dec, const ScaleConsts& sc) {
    const uint64_t g2 = f32x2(sc.g, sc.g), ng2 = f32x2(-sc.g, -sc.g);
    const uint32_t p = bf16x2_round_once(f32x2(dec, 1.5f * dec), g2, ng2);   // b1 | b3 << 16
    const uint32_t q01 = (p << 16) - 0x00800000u;      // entries 0, 1: 0, b1 / 2
    const uint32_t q45 = p + 0x00800080u;              // entries 4, 5: 2 b1, 2 b3
    const uint32_t q67 = p + 0x01000100u;              // entries 6, 7: 4 b1, 4 b3
    ValueTable t;
    asm("prmt.b32 %0, %1, %2, 0x6420;" : "=r"(t.lo0) : "r"(q01), "r"(p));
    asm("prmt.b32 %0, %1, %2, 0x7531;" : "=r"(t.hi0) : "r"(q01), "r"(p));
    asm("prmt.b32 %0, %1, %2, 0x6420;" : "=r"(t.lo1) : "r"(q45), "r"(q67));
    asm("prmt.b32 %0, %1, %2, 0x7531;" : "=r"(t.hi1) : "r"(q45), "r"(q67));
    return t;
}

// bf16x2 results of four elements (magnitude codes in the low four nibbles of
// cm, sign bits cleared), as two words: elements 0, 1 and elements 2, 3; the
// signs come from the input words (for s > 0 the code keeps the sign of x).
__device__ __forceinline__ void table_lookup4(const ValueTable& t, uint32_t cm, uint32_t w01, uint32_t w23,
                                              uint32_t& y01, uint32_t& y23) {
    uint32_t lo, hi;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(lo) : "r"(t.lo0), "r"(t.lo1), "r"(cm));
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(hi) : "r"(t.hi0), "r"(t.hi1), "r"(cm));
    asm("prmt.b32 %0, %1, %2, 0x5140;" : "=r"(y01) : "r"(lo), "r"(hi));
    asm("prmt.b32 %0, %1, %2, 0x7362;" : "=r"(y23) : "r"(lo), "r"(hi));
    y01 |= w01 & 0x80008000u;
    y23 |= w23 & 0x80008000u;
}

// Clip mask of 16 bf16 values (eight words, element 2j in the low half of
// word j): bit e set where |x_e| > 6 s, s > 0.  For bf16 x, |x| > 6 s exactly
// iff |x| > RD_bf16(6 s), and RD_bf16(RD_f32(6 s)) = RD_bf16(6 s); as
// non-negative patterns compare like their values, each half then tests
// |x| >= tb with tb = RD_bf16(6 s) + 1 by one subtraction from 0x8000 + |x|
// (no borrow crosses the halves).  s == 0 gives tb = 0x8000: nothing clips.
__device__ __forceinline__ uint32_t clip_mask16(const uint32_t (&w)[8], float s) {
    const uint32_t tb = s > 0.0f ? (__float_as_uint(__fmul_rd(6.0f, s)) >> 16) + 1u : 0x8000u;
    const uint32_t t2 = tb | (tb << 16);
    // flags of pair j (bits 15 and 31) move to bits 2j and 16 + 2j
    uint32_t acc = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) acc |= (((w[j] | 0x80008000u) - t2) >> (15 - 2 * j)) & (0x00010001u << (2 * j));
    return (acc & 0x5555u) | ((acc >> 15) & 0xAAAAu);
}

// nvfp4_fake_quantize: y = e2m1(code) * dec(sf) * g rounded once to bf16 (or
// FP32), 16 values per lane and step, and the optional clip mask (2 bytes per
// lane and step).  Scales are not stored.
template <bool kF32>
struct FakeOut {
    void* y;
    uint8_t* mask;                                // nullable
    static constexpr bool kScales = false;
    static constexpr int kMinBlocks = 2;          // 64 registers: 2 CTAs (32 warps) per SM
    static constexpr int kGroup = 1;
    struct Lane {
        uint4* yp;
        uint16_t* mp;
        int64_t ystep, mstep;
    };
    __device__ __forceinline__ Lane lane(const TileLane& t, int64_t k) const {
        Lane l;
        l.yp = reinterpret_cast<uint4*>(y) + (kF32 ? (t.e0 >> 2) : (t.e0 >> 3));
        l.ystep = kF32 ? (k >> 1) : (k >> 2);      // two rows, in 16-byte units
        l.mp = reinterpret_cast<uint16_t*>(mask) + (t.e0 >> 4);
        l.mstep = k >> 3;
        return l;
    }
    __device__ __forceinline__ void emit(const Lane& l, int i, bool ok, const uint32_t (&w)[8], uint32_t sfc,
                                         float s, uint32_t lo, uint32_t hi, const ScaleConsts& sc) const {
        const uint32_t codes[2] = {lo, hi};
        if (kF32) {
            const uint32_t sd2 = e4m3_to_f16x2(sfc);
            const uint64_t g2 = f32x2(sc.g, sc.g);
            uint32_t o[16];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint64_t p = mul_f32x2(f16x2_to_f32x2(e2m1x2_times_scale(codes[h] >> (8 * j), sd2)), g2);
                    asm("mov.b64 {%0, %1}, %2;" : "=r"(o[8 * h + 2 * j]), "=r"(o[8 * h + 2 * j + 1]) : "l"(p));
                }
            if (ok) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    l.yp[i * l.ystep + q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
            }
        } else {
            uint32_t o[8];
            if (s >= 0x1p-118f && s <= 0x1p124f) {
                const ValueTable tb = value_table(e4m3_to_f32(sfc), sc);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t cm = codes[h] & 0x77777777u;
                    table_lookup4(tb, cm, w[4 * h], w[4 * h + 1], o[4 * h], o[4 * h + 1]);
                    table_lookup4(tb, cm >> 16, w[4 * h + 2], w[4 * h + 3], o[4 * h + 2], o[4 * h + 3]);
                }
            } else {
                // tiny, huge or zero block scales: every value rounded exactly
                const uint32_t sd2 = e4m3_to_f16x2(sfc);
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        o[4 * h + j] =
                            bf16x2_round_once_slow(f16x2_to_f32x2(e2m1x2_times_scale(codes[h] >> (8 * j), sd2)), sc.g);
            }
            if (ok) {
                l.yp[i * l.ystep] = make_uint4(o[0], o[1], o[2], o[3]);
                l.yp[i * l.ystep + 1] = make_uint4(o[4], o[5], o[6], o[7]);
            }
        }
        if (mask != nullptr && ok) l.mp[i * l.mstep] = (uint16_t)clip_mask16(w, s);
    }
    __device__ __forceinline__ void store_scales(const uint8_t*, int64_t, int64_t, int64_t) const {}
};

// Quantize a lane's loaded blocks and hand each to the output.  When the
// output stores scales they go to the CTA's staging atoms (kStage) or, word by
// word, straight to the scale buffer: the four lanes holding blocks 4a .. 4a+3
// of a row share one 32-bit word of the layout, gathered by shuffles and
// stored by the first of them (rows past the tensor quantize zeros, so the
// padding rows of the layout get zero scales).
template <class Out, bool kStage = true>
__device__ __forceinline__ void quantize_lane(const TileLane& t, const uint4 (&v)[2 * kSteps], const ScaleConsts& sc,
                                              uint8_t* sf_stage, const Out& out, int64_t k, int64_t rblk = 0,
                                              int64_t cblk = 0) {
    const typename Out::Lane ol = out.lane(t, k);
#pragma unroll
    for (int i = 0; i < kSteps; ++i) {
        const uint32_t w[8] = {v[2 * i].x, v[2 * i].y, v[2 * i].z, v[2 * i].w,
                               v[2 * i + 1].x, v[2 * i + 1].y, v[2 * i + 1].z, v[2 * i + 1].w};
        float ab = __uint_as_float(block_absmax16(w) << 16);            // block amax
        if (Out::kGroup >= 2) ab = fmaxf(ab, __shfl_xor_sync(0xffffffffu, ab, 1));   // lanes of one row:
        if (Out::kGroup >= 4) ab = fmaxf(ab, __shfl_xor_sync(0xffffffffu, ab, 2));   // consecutive blocks
        const uint32_t sfc = block_scale_code(ab, sc);
        const float s = __fmul_rn(e4m3_to_f32(sfc), sc.g);
        const uint32_t lo = quantize8_bf16(w[0], w[1], w[2], w[3], s);
        const uint32_t hi = quantize8_bf16(w[4], w[5], w[6], w[7], s);
        out.emit(ol, i, 2 * i < t.rows_left && t.col_ok, w, sfc, s, lo, hi, sc);
        if constexpr (Out::kScales) {
            if (kStage) {
                if (t.col_ok) sf_stage[t.sbase + 32 * i] = (uint8_t)sfc;
            } else {
                uint32_t word = sfc;
                word |= __shfl_down_sync(0xffffffffu, sfc, 1) << 8;
                word |= __shfl_down_sync(0xffffffffu, sfc, 2) << 16;
                word |= __shfl_down_sync(0xffffffffu, sfc, 3) << 24;
                const int lane = threadIdx.x & 31, blk = lane & 15;
                const int rt = ((threadIdx.x >> 5) & 15) * kRows + (lane >> 4) + 2 * i;     // row inside the tile
                if ((blk & 3) == 0 && t.col_ok) {
                    const int64_t atom = rblk * (k >> 6) + cblk * 4 + (blk >> 2);
                    *reinterpret_cast<uint32_t*>(out.sf + (atom << 9) + (rt & 31) * 16 + (rt >> 5) * 4) = word;
                }
            }
        }
    }
}

// Two-kernel form: one CTA per tile, after the amax pass (or with a given
// tensor scale).
template <bool kDynamic, class Out>
__global__ void __launch_bounds__(kQuantThreads, Out::kMinBlocks)
quantize_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t k, int64_t ld, const Out out,
                float* __restrict__ tensor_scale, const float* __restrict__ partials, int nparts) {
    __shared__ __align__(16) uint8_t sf_stage[4 * kAtomPitch];
    __shared__ ScaleConsts sc_sh;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // row blocks in reverse launch order: the amax pass read the tensor front
    // to back, so its tail is the part still in L2 when the first CTAs start
    const int64_t rblk = (int64_t)(gridDim.y - 1 - blockIdx.y);
    const int64_t cblk = blockIdx.x;
    const TileLane t = tile_lane(x, rows, k, ld, rblk, cblk, warp, lane);
    uint4 v[2 * kSteps];
    load_tile(t, v);

    // the tensor scale and its block-scale constants, once per CTA, after the
    // amax grid (when launched as its programmatic dependent) has completed
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (warp == 0) {
        float g;
        if (kDynamic) {
            float mx = 0.0f;
            for (int i = lane; i < nparts; i += 32) mx = fmaxf(mx, partials[i]);
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            g = __fdiv_rn(mx, 2688.0f);
            if (blockIdx.x == 0 && blockIdx.y == 0 && lane == 0) *tensor_scale = g;   // one writer
        } else {
            g = *tensor_scale;
        }
        if (lane == 0) sc_sh = scale_consts(g);
    }
    __syncthreads();
    quantize_lane(t, v, sc_sh, sf_stage, out, k);
    if (Out::kScales) {
        __syncthreads();
        out.store_scales(sf_stage, k, rblk, cblk);
    }
}

// One-kernel form with a data-derived tensor scale: a persistent grid whose
// CTAs all stay resident (cooperative launch) takes the tiles t = blockIdx.x,
// blockIdx.x + gridDim.x, ...  Phase 1 reduces |x| over the CTA's tiles and
// publishes (generation, partial max) in the CTA's slot; every CTA then waits
// (bounded) until all slots carry this call's generation -- the generation is
// a per-call number from the host, so the slots need no initialisation -- and
// takes the maximum itself.  Phase 2 quantizes the same tiles in reverse
// order, so the first ones re-read what phase 1 read last, still in L2.
template <class Out>
__global__ void __launch_bounds__(kQuantThreads, Out::kMinBlocks)
quantize_fused_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t k, int64_t ld, const Out out,
                      float* __restrict__ tensor_scale,
                      unsigned long long* __restrict__ slots, uint32_t gen, int ntiles_c, int ntiles,
                      int* __restrict__ dev_status) {
    __shared__ __align__(16) uint8_t sf_stage[4 * kAtomPitch];
    __shared__ ScaleConsts sc_sh;
    __shared__ uint32_t red[kQuantThreads / 32];
    __shared__ int ok_sh;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- phase 1: |x| maximum (and the largest exponent field) of this CTA's tiles
    uint32_t m = 0u;
    for (int tt = blockIdx.x; tt < ntiles; tt += gridDim.x) {
        const TileLane t = tile_lane(x, rows, k, ld, tt / ntiles_c, tt % ntiles_c, warp, lane);
        uint4 v[2 * kSteps];
#pragma unroll
        for (int i = 0; i < kSteps; ++i) {
            if (2 * i < t.rows_left && t.col_ok) {
                v[2 * i] = __ldg(t.xp + i * t.xstep);
                v[2 * i + 1] = __ldg(t.xp + i * t.xstep + 1);
            } else {
                v[2 * i] = make_uint4(0u, 0u, 0u, 0u);
                v[2 * i + 1] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
#pragma unroll
        for (int i = 0; i < 2 * kSteps; ++i) m = absmax_nan_bf16x2(m, absmax_bf16x8(v[i]));
    }
    m &= 0x7FFF7FFFu;
    uint32_t h = max(m & 0xFFFFu, m >> 16);
    for (int o = 16; o > 0; o >>= 1) h = max(h, __shfl_xor_sync(0xffffffffu, h, o));
    if (lane == 0) red[warp] = h;
    __syncthreads();
    if (warp == 0) {
        uint32_t tm = lane < kQuantThreads / 32 ? red[lane] : 0u;
        for (int o = 16; o > 0; o >>= 1) tm = max(tm, __shfl_xor_sync(0xffffffffu, tm, o));
        if (lane == 0) {
            if (tm >= 0x7F80u && dev_status) atomicCAS(dev_status, 0, (int)NVFP4_ERR_NONFINITE);
            const unsigned long long word = ((unsigned long long)gen << 32) | (unsigned long long)(tm << 16);
            asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(slots + blockIdx.x), "l"(word) : "memory");
        }
        // ---- every CTA's slot carries this generation: the tensor maximum
        float mx = 0.0f;
        bool ok = true;
        const uint64_t t0 = globaltimer_ns();
        for (int i = lane; i < (int)gridDim.x; i += 32) {
            unsigned long long w;
            uint32_t n = 0;
            while (true) {
                asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(slots + i) : "memory");
                if ((uint32_t)(w >> 32) == gen) break;
                if ((++n & 63u) == 0u && globaltimer_ns() - t0 > kWaitLimitNs) { ok = false; break; }
            }
            if (!ok) break;
            mx = fmaxf(mx, __uint_as_float((uint32_t)w));
        }
        ok = __all_sync(0xffffffffu, ok ? 1 : 0) != 0;
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) {
            if (!ok && dev_status) atomicExch(dev_status, (int)NVFP4_ERR_TIMEOUT);
            const float g = __fdiv_rn(mx, 2688.0f);
            if (blockIdx.x == 0 && ok) *tensor_scale = g;
            sc_sh = scale_consts(g);
            ok_sh = ok ? 1 : 0;
        }
    }
    __syncthreads();
    if (!ok_sh) return;                           // gave up waiting: outputs unspecified
    const ScaleConsts sc = sc_sh;

    // ---- phase 2: quantize the same tiles, last first
    const int nmine = ntiles > (int)blockIdx.x ? (ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    for (int j = nmine - 1; j >= 0; --j) {
        const int tt = (int)blockIdx.x + j * (int)gridDim.x;
        const int64_t rblk = tt / ntiles_c, cblk = tt % ntiles_c;
        const TileLane t = tile_lane(x, rows, k, ld, rblk, cblk, warp, lane);
        uint4 v[2 * kSteps];
        load_tile(t, v);
        quantize_lane(t, v, sc, sf_stage, out, k);
        if (Out::kScales) {
            __syncthreads();
            out.store_scales(sf_stage, k, rblk, cblk);
            __syncthreads();
        }
    }
}

// One-kernel form, streamed: the same two phases, with the tiles brought into
// shared memory by TMA.  One CTA per SM (cooperative launch, so every CTA is
// resident for the handoff): a producer warp keeps a ring of kStreamBufs tile
// buffers filled -- the CTA's tiles in order for phase 1, then in reverse for
// phase 2 -- while sixteen consumer warps work on the tile in front.  Loads
// therefore overlap the arithmetic instead of alternating with it, and the
// first phase-2 tiles are already on their way while the CTAs wait for each
// other's maxima.  A consumer warp releases a buffer as soon as it holds its
// part of the tile in registers.
constexpr int kStreamBufs = 3;
constexpr int kStreamTileBytes = kTileRows * kTileCols * 2;      // 64 KB of bf16
constexpr int kStreamConsumers = kQuantThreads;                  // 16 warps
constexpr int kStreamThreads = kStreamConsumers + 32;            // + the producer warp
constexpr int kStreamSmem = kStreamBufs * kStreamTileBytes + 1024;

__device__ __forceinline__ void consumers_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kStreamConsumers) : "memory");
}

template <class Out>
__global__ void __launch_bounds__(kStreamThreads, 1)
quantize_stream_kernel(const __grid_constant__ CUtensorMap tmap_x, int64_t rows, int64_t k, const Out out,
                       float* __restrict__ tensor_scale, unsigned long long* __restrict__ slots, uint32_t gen,
                       int ntiles_c, int ntiles, int* __restrict__ dev_status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full_bar[kStreamBufs], empty_bar[kStreamBufs];
    __shared__ ScaleConsts sc_sh;
    __shared__ uint32_t red[kStreamConsumers / 32];
    __shared__ int abort_sh, ok_sh;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        abort_sh = 0;
        for (int b = 0; b < kStreamBufs; ++b) {
            mbar_init(&full_bar[b], 1);
            mbar_init(&empty_bar[b], kStreamConsumers / 32);
        }
        fence_barrier_init();
    }
    __syncthreads();
    WaitCtx wc{&abort_sh, dev_status};
    const int nmine = ntiles > (int)blockIdx.x ? (ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

    if (warp == kStreamConsumers / 32) {
        // ---- producer: phase-1 tiles in order, then the same tiles in reverse
        if (lane == 0) {
            tma_prefetch_desc(&tmap_x);
            const uint64_t pol1 = policy_evict_normal(), pol2 = policy_evict_first();
            int b = 0;
            uint32_t ph = 0;
            for (int q = 0; q < 2 * nmine; ++q) {
                const int j = q < nmine ? q : 2 * nmine - 1 - q;
                const int tt = (int)blockIdx.x + j * (int)gridDim.x;
                if (!mbar_wait(&empty_bar[b], ph ^ 1u, wc)) break;
                mbar_arrive_expect_tx(&full_bar[b], kStreamTileBytes);
                tma_load_2d(tiles + b * kStreamTileBytes, &tmap_x, &full_bar[b], (tt % ntiles_c) * kTileCols,
                            (tt / ntiles_c) * kTileRows, q < nmine ? pol1 : pol2);
                if (++b == kStreamBufs) { b = 0; ph ^= 1u; }
            }
        }
        return;
    }

    // ---- consumers, phase 1: |x| maximum of the CTA's tiles
    int b = 0;
    uint32_t ph = 0;
    uint32_t m = 0u;
    bool alive = true;
    for (int q = 0; q < nmine; ++q) {
        alive = alive && mbar_wait(&full_bar[b], ph, wc);
        if (alive) {
            const uint4* t = reinterpret_cast<const uint4*>(tiles + b * kStreamTileBytes);
#pragma unroll
            for (int i = 0; i < kStreamTileBytes / 16 / kStreamConsumers; ++i)
                m = absmax_nan_bf16x2(m, absmax_bf16x8(t[threadIdx.x + i * kStreamConsumers]));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[b]);
        if (++b == kStreamBufs) { b = 0; ph ^= 1u; }
    }
    m &= 0x7FFF7FFFu;
    uint32_t h = max(m & 0xFFFFu, m >> 16);
    for (int o = 16; o > 0; o >>= 1) h = max(h, __shfl_xor_sync(0xffffffffu, h, o));
    if (lane == 0) red[warp] = h;
    consumers_sync();
    if (warp == 0) {
        uint32_t tm = lane < kStreamConsumers / 32 ? red[lane] : 0u;
        for (int o = 16; o > 0; o >>= 1) tm = max(tm, __shfl_xor_sync(0xffffffffu, tm, o));
        if (lane == 0) {
            if (tm >= 0x7F80u && dev_status) atomicCAS(dev_status, 0, (int)NVFP4_ERR_NONFINITE);
            const unsigned long long word = ((unsigned long long)gen << 32) | (unsigned long long)(tm << 16);
            asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(slots + blockIdx.x), "l"(word) : "memory");
        }
        // ---- every CTA's slot carries this generation: the tensor maximum
        float mx = 0.0f;
        bool ok = true;
        const uint64_t t0 = globaltimer_ns();
        for (int i = lane; i < (int)gridDim.x; i += 32) {
            unsigned long long w;
            uint32_t n = 0;
            while (true) {
                asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(slots + i) : "memory");
                if ((uint32_t)(w >> 32) == gen) break;
                if ((++n & 63u) == 0u && globaltimer_ns() - t0 > kWaitLimitNs) { ok = false; break; }
            }
            if (!ok) break;
            mx = fmaxf(mx, __uint_as_float((uint32_t)w));
        }
        ok = __all_sync(0xffffffffu, ok ? 1 : 0) != 0;
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) {
            if (!ok && dev_status) atomicExch(dev_status, (int)NVFP4_ERR_TIMEOUT);
            const float g = __fdiv_rn(mx, 2688.0f);
            if (blockIdx.x == 0 && ok) *tensor_scale = g;
            sc_sh = scale_consts(g);
            ok_sh = ok ? 1 : 0;
        }
    }
    consumers_sync();
    // gave up waiting: the tiles are still consumed (so that no load is left
    // in flight when the CTA exits), but nothing is written
    alive = alive && ok_sh != 0;
    const ScaleConsts sc = sc_sh;

    // ---- consumers, phase 2: quantize the same tiles, last first
    for (int q = nmine - 1; q >= 0; --q) {
        const int tt = (int)blockIdx.x + q * (int)gridDim.x;
        const int64_t rblk = tt / ntiles_c, cblk = tt % ntiles_c;
        alive = alive && mbar_wait(&full_bar[b], ph, wc);
        uint4 v[2 * kSteps];
        const int half = lane >> 4, blk = lane & 15;
        if (alive) {
            const uint8_t* base = tiles + b * kStreamTileBytes + (warp * kRows + half) * (kTileCols * 2) + blk * 32;
#pragma unroll
            for (int i = 0; i < kSteps; ++i) {
                const uint4* r = reinterpret_cast<const uint4*>(base + 2 * i * (kTileCols * 2));
                v[2 * i] = r[0];
                v[2 * i + 1] = r[1];
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[b]);
        if (++b == kStreamBufs) { b = 0; ph ^= 1u; }
        if (alive) {
            const TileLane t = tile_lane(nullptr, rows, k, k, rblk, cblk, warp, lane);
            quantize_lane<Out, false>(t, v, sc, nullptr, out, k, rblk, cblk);
        }
    }
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

// ------------------------------------------------------------------ STE backward
// grad_x = grad_y where the clip mask is clear, +0 where it is set.  One
// thread per 16 elements (one 16-bit mask word), two groups in flight per
// iteration; contiguous [rows, k] buffers seen as a flat array.  grad_x may
// be grad_y (each element is read, then written, by the same thread), so the
// pointers are not declared restrict.
template <bool kF32>
__global__ void __launch_bounds__(256)
ste_backward_kernel(const uint4* gy, const uint16_t* mask, int64_t ngroups, uint4* gx) {
    constexpr int kVec = kF32 ? 4 : 2;                // 16-byte vectors per group
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < ngroups; g += 2 * stride) {
        const bool two = g + stride < ngroups;
        uint4 a[kVec], b[kVec];
        uint32_t ma = __ldcs(mask + g), mb = 0u;
#pragma unroll
        for (int q = 0; q < kVec; ++q) a[q] = __ldcs(gy + g * kVec + q);
        if (two) {
            mb = __ldcs(mask + g + stride);
#pragma unroll
            for (int q = 0; q < kVec; ++q) b[q] = __ldcs(gy + (g + stride) * kVec + q);
        }
        auto apply = [](uint4 (&v)[kVec], uint32_t m) {
#pragma unroll
            for (int q = 0; q < kVec; ++q) {
                uint32_t* w = &v[q].x;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (kF32) {
                        const int e = 4 * q + j;
                        if ((m >> e) & 1u) w[j] = 0u;
                    } else {
                        const int e = 8 * q + 2 * j;      // elements e (low half), e + 1 (high half)
                        const uint32_t clear = (((m >> e) & 1u) * 0x0000FFFFu) | (((m >> (e + 1)) & 1u) * 0xFFFF0000u);
                        w[j] &= ~clear;
                    }
                }
            }
        };
        apply(a, ma);
#pragma unroll
        for (int q = 0; q < kVec; ++q) __stcs(gx + g * kVec + q, a[q]);
        if (two) {
            apply(b, mb);
#pragma unroll
            for (int q = 0; q < kVec; ++q) __stcs(gx + (g + stride) * kVec + q, b[q]);
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

// Two-kernel form (or one kernel with a given scale) for any output.
template <class Out>
static cudaError_t launch_two_kernel(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, const Out& out,
                                     float* tensor_scale, bool scale_given, float* partials, int* dev_status,
                                     cudaStream_t stream) {
    const dim3 grid((unsigned)((k + 255) / 256), (unsigned)((rows + 127) / 128));
    if (scale_given) {
        quantize_kernel<false, Out><<<grid, kQuantThreads, 0, stream>>>(x, rows, k, ld, out, tensor_scale,
                                                                       nullptr, 0);
        count_launch(1);
        return cudaGetLastError();
    }
    const int ag = amax_grid(rows, k);
    amax_kernel<<<ag, kAmaxThreads, 0, stream>>>(x, rows, k, ld, partials, dev_status);
    // programmatic dependent launch: the quantize CTAs start loading X while
    // the amax grid finishes, and wait for it before reading its partials
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kQuantThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, quantize_kernel<true, Out>, x, rows, k, ld, out, tensor_scale,
                                       (const float*)partials, ag);
    count_launch(2);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// Per-call numbers tagging the one-kernel form's workspace slots: one counter
// for every output type, so that no two calls in the process share a number
// (a workspace used by one output type and then another must not hold a
// slot that carries the new call's number).
static std::atomic<uint32_t> g_generation{0};

uint32_t next_generation() {
    uint32_t gen = g_generation.fetch_add(1u) + 1u;
    if (gen == 0u) gen = g_generation.fetch_add(1u) + 1u;     // 0 never marks a slot
    return gen;
}

// One-kernel form with a data-derived scale (see quantize_fused_kernel).
// Returns cudaErrorNotSupported when the grid cannot be co-resident (the
// caller then takes the two-kernel form, which computes the same result).
template <class Out>
static cudaError_t launch_one_kernel_regs(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, const Out& out,
                                          float* tensor_scale, unsigned long long* slots, int max_slots,
                                          int* dev_status, int num_sms, cudaStream_t stream) {
    const int ntiles_c = (int)((k + kTileCols - 1) / kTileCols);
    const int64_t ntiles64 = ((rows + kTileRows - 1) / kTileRows) * ntiles_c;
    if (ntiles64 > (int64_t)1 << 30) return cudaErrorNotSupported;
    const int ntiles = (int)ntiles64;
    int per_sm = 0;
    cudaError_t e =
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_fused_kernel<Out>, kQuantThreads, 0);
    if (e != cudaSuccess) return e;
    int grid = per_sm * num_sms;
    if (grid > max_slots) grid = max_slots;
    if (grid > ntiles) grid = ntiles;
    if (grid < 1) return cudaErrorNotSupported;
    const uint32_t gen = next_generation();
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;           // every CTA resident at once
    attr[0].val.cooperative = 1;
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kQuantThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, quantize_fused_kernel<Out>, x, rows, k, ld, out, tensor_scale, slots, gen,
                           ntiles_c, ntiles, dev_status);
    if (e == cudaErrorCooperativeLaunchTooLarge) {
        (void)cudaGetLastError();
        return cudaErrorNotSupported;
    }
    if (e != cudaSuccess) return e;
    count_launch(1);
    return cudaGetLastError();
}

// One-kernel form with a data-derived scale: for fake quantization the tiles
// are streamed through shared memory by TMA (quantize_stream_kernel); codes
// and scales are faster from registers (quantize_fused_kernel, two CTAs per
// SM: the streamed form's shared-memory reads and scale-word shuffles cost it
// a few per cent there).  NVFP4_QUANT_ONE_KERNEL=regs or =stream forces one
// form, for measurements.  Returns
// cudaErrorNotSupported when the grid cannot be co-resident or the tensor
// cannot be described to TMA (the caller then takes the two-kernel form,
// which computes the same result).
template <class Out>
static cudaError_t launch_one_kernel(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, const Out& out,
                                     float* tensor_scale, unsigned long long* slots, int max_slots, int* dev_status,
                                     int num_sms, cudaStream_t stream) {
    const char* env = getenv("NVFP4_QUANT_ONE_KERNEL");
    const bool stream_form = env ? env[0] == 's' : !Out::kScales;
    if (!stream_form)
        return launch_one_kernel_regs(x, rows, k, ld, out, tensor_scale, slots, max_slots, dev_status, num_sms,
                                      stream);
    const int ntiles_c = (int)((k + kTileCols - 1) / kTileCols);
    const int64_t ntiles64 = ((rows + kTileRows - 1) / kTileRows) * ntiles_c;
    if (ntiles64 > (int64_t)1 << 30) return cudaErrorNotSupported;
    const int ntiles = (int)ntiles64;
    CUtensorMap tm;
    if (make_tmap_2d(&tm, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)k, (uint64_t)rows, (uint64_t)ld * 2,
                     kTileCols, kTileRows, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
        return cudaErrorNotSupported;
    auto kern = quantize_stream_kernel<Out>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kStreamSmem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kStreamThreads, kStreamSmem);
    if (e != cudaSuccess) return e;
    int grid = per_sm * num_sms;
    if (grid > max_slots) grid = max_slots;
    if (grid > ntiles) grid = ntiles;
    if (grid < 1) return cudaErrorNotSupported;
    const uint32_t gen = next_generation();
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;           // every CTA resident at once
    attr[0].val.cooperative = 1;
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kStreamThreads);
    cfg.dynamicSmemBytes = kStreamSmem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, tm, rows, k, out, tensor_scale, slots, gen, ntiles_c, ntiles, dev_status);
    if (e == cudaErrorCooperativeLaunchTooLarge) {
        (void)cudaGetLastError();
        return cudaErrorNotSupported;
    }
    if (e != cudaSuccess) return e;
    count_launch(1);
    return cudaGetLastError();
}

cudaError_t launch_quantize(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, uint8_t* codes,
                            uint8_t* sf, float* tensor_scale, bool scale_given, float* partials,
                            int* dev_status, cudaStream_t stream) {
    return launch_two_kernel(x, rows, k, ld, CodesOut{codes, sf}, tensor_scale, scale_given, partials, dev_status,
                             stream);
}

cudaError_t launch_quantize_fused(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, uint8_t* codes,
                                  uint8_t* sf, float* tensor_scale, unsigned long long* slots, int max_slots,
                                  int* dev_status, int num_sms, cudaStream_t stream) {
    return launch_one_kernel(x, rows, k, ld, CodesOut{codes, sf}, tensor_scale, slots, max_slots, dev_status,
                             num_sms, stream);
}

// Quantization with 32 or 64 values per scale (scales repeated in the block-16
// layout): one kernel with a data-derived scale when the grid can be
// co-resident, else two; one kernel with a given scale.
cudaError_t launch_quantize_block(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, int block, uint8_t* codes,
                                  uint8_t* sf, float* tensor_scale, bool scale_given, void* workspace,
                                  int* dev_status, int num_sms, cudaStream_t stream) {
    auto run = [&](auto out) -> cudaError_t {
        if (!scale_given) {
            const cudaError_t e = launch_one_kernel(x, rows, k, ld, out, tensor_scale,
                                                    static_cast<unsigned long long*>(workspace), kFusedSlots,
                                                    dev_status, num_sms, stream);
            if (e != cudaErrorNotSupported) return e;
        }
        return launch_two_kernel(x, rows, k, ld, out, tensor_scale, scale_given, static_cast<float*>(workspace),
                                 dev_status, stream);
    };
    if (block == 32) return run(CodesOutG<2>{{codes, sf}});
    if (block == 64) return run(CodesOutG<4>{{codes, sf}});
    return run(CodesOut{codes, sf});
}

// Fake quantization: one kernel with a data-derived scale when the grid can
// be co-resident, else the two-kernel form; one kernel with a given scale.
cudaError_t launch_fake_quantize(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, void* y, bool y_f32,
                                 uint8_t* mask, float* tensor_scale, bool scale_given, void* workspace,
                                 int* dev_status, int num_sms, cudaStream_t stream) {
    auto run = [&](auto out) -> cudaError_t {
        if (!scale_given) {
            const cudaError_t e = launch_one_kernel(x, rows, k, ld, out, tensor_scale,
                                                    static_cast<unsigned long long*>(workspace), kFusedSlots,
                                                    dev_status, num_sms, stream);
            if (e != cudaErrorNotSupported) return e;
        }
        return launch_two_kernel(x, rows, k, ld, out, tensor_scale, scale_given, static_cast<float*>(workspace),
                                 dev_status, stream);
    };
    return y_f32 ? run(FakeOut<true>{y, mask}) : run(FakeOut<false>{y, mask});
}

// ------------------------------------------------------------------ failure-detection check
// One warp waits, through the bounded mbarrier wait of the GEMM and quantize
// kernels, on a barrier nothing arrives at; the wait gives up after limit_ns
// and reports NVFP4_ERR_TIMEOUT.
__global__ void __launch_bounds__(32) debug_wait_kernel(int* dev_status, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_sh;
    if (threadIdx.x == 0) {
        abort_sh = 0;
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncwarp();
    WaitCtx wc{&abort_sh, dev_status};
    if (threadIdx.x == 0) mbar_wait_limit(&bar, 0, wc, limit_ns);
    __syncwarp();
}

cudaError_t launch_debug_wait_timeout(int* dev_status, uint64_t limit_ns, cudaStream_t stream) {
    debug_wait_kernel<<<1, 32, 0, stream>>>(dev_status, limit_ns);
    count_launch(1);
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

cudaError_t launch_ste_backward(const void* grad_y, const uint8_t* mask, int64_t rows, int64_t k, bool f32,
                                void* grad_x, int num_sms, cudaStream_t stream) {
    const int64_t ngroups = rows * (k >> 4);
    int64_t g = (ngroups + 2 * 256 - 1) / (2 * 256);
    if (g > (int64_t)num_sms * 16) g = (int64_t)num_sms * 16;
    if (g < 1) g = 1;
    const uint4* src = static_cast<const uint4*>(grad_y);
    const uint16_t* m = reinterpret_cast<const uint16_t*>(mask);
    uint4* dst = static_cast<uint4*>(grad_x);
    if (f32)
        ste_backward_kernel<true><<<(unsigned)g, 256, 0, stream>>>(src, m, ngroups, dst);
    else
        ste_backward_kernel<false><<<(unsigned)g, 256, 0, stream>>>(src, m, ngroups, dst);
    count_launch(1);
    return cudaGetLastError();
}

}  // namespace nvfp4
