// layernorm.cu -- LayerNorm (with a per-group affine) producing the next
// linear layer's NVFP4 input in one kernel: the bf16 LayerNorm output is
// never written, re-read by an amax pass and re-read by the quantizer.
//
// The pages run every linear layer of the DiT blocks in FP4 ("NVFP4-DiT ..."
// README, Abstract and Methodology 3; "[RFC]: NVFP4 Quantization Support for
// Diffusion Models", two-level scaling) but do not define LayerNorm.  The
// reading taken is the DiT pre-norm over the hidden dimension followed by the
// adaLN modulation x (1 + scale) + shift of each sample -- a per-channel
// affine (gamma, beta) shared by a group of rows:
//   S1 = sum_j x_j,  S2 = sum_j x_j^2                     (double)
//   mu = S1 / k,  var = max(S2 / k - mu^2, 0),  rstd = 1 / sqrt(var + eps)
//   y_j = ((x_j - (float)mu) * (float)rstd) * gamma_j + beta_j   (FP32 ops)
// then the NVFP4 quantization of y exactly as nvfp4_quantize does it
// (quant_math.cuh).  Squares of bf16 values are exact in double and so are
// the row sums wherever the values span fewer than about 45 binary orders of
// magnitude; the lanes' partial sums then add up to the same S1, S2 in any
// order.
//
// One warp per row (lane l takes the 16-value blocks l, l + 32, ...); a
// persistent grid.  Each warp streams its rows through two shared-memory row
// buffers: one bulk copy per row (TMA, completion on an mbarrier), the next
// row's copy in flight while the current row is normalised from shared
// memory (statistics pass, then values).  With a data-derived tensor scale
// the grid is co-resident (cooperative launch): phase 1 finds the largest |y|
// of each CTA's rows and hands it over grid-wide through generation-tagged
// slots, exactly as the one-kernel quantizer does; phase 2 streams the rows
// again, last first, and quantizes them.
#include <cstdint>

#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/nvfp4.h"
#include "internal.h"
#include "ptx.cuh"
#include "quant_math.cuh"

namespace nvfp4 {

constexpr int kLnMaxWarps = 16;
constexpr int kLnThreads = kLnMaxWarps * 32;
constexpr int kLnSmemBudget = 220 * 1024;        // row buffers and affine per CTA
constexpr int kLnStatRows = 32;                  // per warp: rows whose phase-1 statistics phase 2 reuses
constexpr int64_t kLnMaxK = 8192;

struct LnArgs {
    const uint16_t* x;
    int64_t rows, k, ld;
    const float* gamma;            // [groups, k] or null
    const float* beta;
    int64_t rows_per_group;        // 0: one group
    double eps;
    uint8_t* codes;
    uint8_t* sf;
    float* tensor_scale;
    unsigned long long* slots;
    uint32_t gen;
    int* dev_status;
};

// Row statistics from the row in shared memory (every lane returns the same
// values).  Each block's values and squares go into their own pair of double
// sums; the sums do not depend on the order wherever they are exact in
// double.
__device__ __forceinline__ void ln_stats(const LnArgs& a, const uint4* row, int lane, float& mu32, float& rstd32) {
    const int kb = (int)(a.k >> 4);
    double s1 = 0.0, s2 = 0.0;
    for (int c = lane; c < kb; c += 32) {
        const uint4 v0 = row[2 * c], v1 = row[2 * c + 1];
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        // four independent chains per sum
        double p1[4] = {0.0, 0.0, 0.0, 0.0}, p2[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const double lo = (double)__uint_as_float(w[j] << 16), hi = (double)__uint_as_float(w[j] & 0xFFFF0000u);
            p1[j & 3] = __dadd_rn(p1[j & 3], __dadd_rn(lo, hi));
            p2[j & 3] = __fma_rn(lo, lo, __fma_rn(hi, hi, p2[j & 3]));
        }
        s1 = __dadd_rn(s1, __dadd_rn(__dadd_rn(p1[0], p1[1]), __dadd_rn(p1[2], p1[3])));
        s2 = __dadd_rn(s2, __dadd_rn(__dadd_rn(p2[0], p2[1]), __dadd_rn(p2[2], p2[3])));
    }
    for (int o = 16; o > 0; o >>= 1) {
        s1 = __dadd_rn(s1, __shfl_xor_sync(0xffffffffu, s1, o));
        s2 = __dadd_rn(s2, __shfl_xor_sync(0xffffffffu, s2, o));
    }
    const double kd = (double)a.k;
    const double mu = __ddiv_rn(s1, kd);
    double var = __dsub_rn(__ddiv_rn(s2, kd), __dmul_rn(mu, mu));
    if (var < 0.0) var = 0.0;
    const double rstd = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(var, a.eps)));
    mu32 = __double2float_rn(mu);
    rstd32 = __double2float_rn(rstd);
}

// The per-channel affine of one row: gamma and beta of its group, from the
// CTA's shared-memory copy when the row belongs to the cached group, else
// from global memory (null: 1 and 0).
// In shared memory the 16-byte chunk q (of 4) of block c sits at chunk
// c * 4 + (q ^ ((c >> 1) & 3)): the eight lanes of a phase reading chunk q of
// blocks c .. c + 7 then hit 32 distinct banks (the plain layout would put
// lanes 64 bytes apart, a four-way conflict).
struct LnAffine {
    const float* gamma;
    const float* beta;
    bool swizzled;
};

__device__ __forceinline__ int ln_affine_slot(int64_t j) {
    const int c = (int)(j >> 4), q = (int)((j >> 2) & 3);
    return ((c * 4 + (q ^ ((c >> 1) & 3))) << 2) | (int)(j & 3);
}

// The CTA caches the groups of its first and last real rows (slot 0 and 1;
// a range shorter than a group touches no other); rows of any other group
// read global memory.  Slot s of the cache holds gamma at aff + s * per and
// beta at aff + s * per + (gamma ? k : 0), per = (gamma + beta) * k floats.
__device__ __forceinline__ LnAffine ln_affine(const LnArgs& a, int64_t r, const int64_t (&cached)[2],
                                              const float* aff) {
    const int64_t grp = a.rows_per_group > 0 ? r / a.rows_per_group : 0;
    const int64_t per = ((a.gamma ? 1 : 0) + (a.beta ? 1 : 0)) * a.k;
    const int slot = grp == cached[0] ? 0 : grp == cached[1] ? 1 : -1;
    if (slot >= 0) {
        const float* g = aff + slot * per;
        return {a.gamma ? g : nullptr, a.beta ? g + (a.gamma ? a.k : 0) : nullptr, true};
    }
    return {a.gamma ? a.gamma + grp * a.k : nullptr, a.beta ? a.beta + grp * a.k : nullptr, false};
}

// The 16 normalised FP32 values of block c of a row (row in shared memory).
__device__ __forceinline__ void ln_block(const uint4* row, const LnAffine& af, int c, float mu32, float rstd32,
                                         float (&y)[16]) {
    const uint4 v0 = row[2 * c], v1 = row[2 * c + 1];
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        y[2 * j] = __fmul_rn(__fsub_rn(__uint_as_float(w[j] << 16), mu32), rstd32);
        y[2 * j + 1] = __fmul_rn(__fsub_rn(__uint_as_float(w[j] & 0xFFFF0000u), mu32), rstd32);
    }
    const int sw = af.swizzled ? ((c >> 1) & 3) : 0;
    if (af.gamma) {
        const float4* g = reinterpret_cast<const float4*>(af.gamma + 16 * c);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 t = g[q ^ sw];
            y[4 * q] = __fmul_rn(y[4 * q], t.x);
            y[4 * q + 1] = __fmul_rn(y[4 * q + 1], t.y);
            y[4 * q + 2] = __fmul_rn(y[4 * q + 2], t.z);
            y[4 * q + 3] = __fmul_rn(y[4 * q + 3], t.w);
        }
    }
    if (af.beta) {
        const float4* b = reinterpret_cast<const float4*>(af.beta + 16 * c);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 t = b[q ^ sw];
            y[4 * q] = __fadd_rn(y[4 * q], t.x);
            y[4 * q + 1] = __fadd_rn(y[4 * q + 1], t.y);
            y[4 * q + 2] = __fadd_rn(y[4 * q + 2], t.z);
            y[4 * q + 3] = __fadd_rn(y[4 * q + 3], t.w);
        }
    }
}

// Largest |y| of a row in shared memory; `bad` is set when the row statistics
// are not finite (an Inf or NaN in the row).
__device__ __forceinline__ float ln_row_amax(const LnArgs& a, const uint4* row, const LnAffine& af, int lane,
                                             bool& bad, float& mu32, float& rstd32) {
    ln_stats(a, row, lane, mu32, rstd32);
    bad |= !(fabsf(mu32) <= 3.402823466e38f) || !(rstd32 <= 3.402823466e38f);
    const int kb = (int)(a.k >> 4);
    float m = 0.0f;
    for (int c = lane; c < kb; c += 32) {
        float y[16];
        ln_block(row, af, c, mu32, rstd32, y);
#pragma unroll
        for (int j = 0; j < 16; ++j) m = fmaxf(m, fabsf(y[j]));
    }
    return m;
}

// Normalise and quantize row r (row null: a padding row of the scale buffer,
// rows <= r < rows rounded up to 128, which gets zero scales).  The four
// lanes 4i .. 4i+3 hold blocks that share one word of the scale layout; lane
// 4i gathers and stores it.  `stats`, when given, holds the row's (mean,
// 1/std) from phase 1 -- the same values ln_stats would compute again.
__device__ __forceinline__ void ln_quantize_row(const LnArgs& a, const uint4* row, const LnAffine& af, int64_t r,
                                                int lane, const ScaleConsts& sc, const float2* stats = nullptr) {
    const int kb = (int)(a.k >> 4);
    const int64_t kb4 = a.k >> 6;
    float mu32 = 0.0f, rstd32 = 0.0f;
    if (row) {
        if (stats) {
            mu32 = stats->x;
            rstd32 = stats->y;
        } else {
            ln_stats(a, row, lane, mu32, rstd32);
        }
    }
    uint8_t* sfrow = a.sf + ((r >> 7) * kb4) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4;
    for (int c0 = 0; c0 < kb; c0 += 32) {
        const int c = c0 + lane;              // kb % 4 == 0: the four lanes of a word agree on c < kb
        uint32_t sfc = 0u;
        if (row && c < kb) {
            float y[16];
            ln_block(row, af, c, mu32, rstd32, y);
            float ab = 0.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) ab = fmaxf(ab, fabsf(y[j]));
            sfc = block_scale_code(ab, sc);
            const float s = __fmul_rn(e4m3_to_f32(sfc), sc.g);
            float lo[8], hi[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) { lo[j] = y[j]; hi[j] = y[8 + j]; }
            const uint32_t wl = quantize8(lo, s), wh = quantize8(hi, s);
            *reinterpret_cast<uint2*>(a.codes + r * (a.k >> 1) + 8 * c) = make_uint2(wl, wh);
        }
        uint32_t word = sfc;
        word |= __shfl_down_sync(0xffffffffu, sfc, 1) << 8;
        word |= __shfl_down_sync(0xffffffffu, sfc, 2) << 16;
        word |= __shfl_down_sync(0xffffffffu, sfc, 3) << 24;
        if ((lane & 3) == 0 && c < kb) *reinterpret_cast<uint32_t*>(sfrow + (c >> 2) * 512) = word;
    }
}

// A warp's two row buffers and their barriers: row i of the warp's sequence
// goes into buffer i % 2; the copy of row i + 1 is issued before row i is
// processed (its buffer held row i - 1, already finished by the whole warp).
struct LnStream {
    uint8_t* buf;
    uint64_t* bar;
    uint32_t phase;                // bit b: the parity buffer b's barrier completes next
    uint32_t bytes;
    uint32_t pending;              // bit b: a copy into buffer b not yet waited for
    __device__ __forceinline__ void issue(const LnArgs& a, int64_t r, int b, int lane) {
        if (lane == 0) {
            mbar_arrive_expect_tx(&bar[b], bytes);
            bulk_load(buf + b * bytes, a.x + r * a.ld, bytes, &bar[b], policy_evict_normal());
        }
        pending |= 1u << b;
    }
    __device__ __forceinline__ const uint4* wait(int b, const WaitCtx& wc, bool& ok) {
        if (mbar_wait(&bar[b], (phase >> b) & 1u, wc)) pending &= ~(1u << b);
        else ok = false;
        phase ^= 1u << b;
        return reinterpret_cast<const uint4*>(buf + b * bytes);
    }
    // before leaving after a failed wait: let copies still in flight land
    // (bounded), so that none writes shared memory after the CTA has exited
    __device__ __forceinline__ void drain(int* dev_status) {
        int no_abort = 0;
        WaitCtx w2{&no_abort, dev_status};
        for (int b = 0; b < 2; ++b)
            if (pending & (1u << b)) {
                (void)mbar_wait(&bar[b], (phase >> b) & 1u, w2);
                pending &= ~(1u << b);
            }
    }
};

// kDynamic: data-derived tensor scale (co-resident grid, grid-wide handoff);
// otherwise the tensor scale is read from a.tensor_scale.
template <bool kDynamic>
__global__ void __launch_bounds__(kLnThreads)
layernorm_quantize_kernel(const LnArgs a, int warps, int64_t per_cta) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    __shared__ __align__(8) uint64_t bars[2 * kLnMaxWarps];
    __shared__ ScaleConsts sc_sh;
    __shared__ float red[kLnMaxWarps];
    __shared__ float2 row_stats[kLnMaxWarps][kLnStatRows];   // phase 1's (mean, 1/std) of a warp's first rows
    __shared__ int ok_sh, abort_sh;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rowbytes = (uint32_t)(a.k * 2);
    // the CTA's rows: a contiguous range, so that they mostly share one group
    // of the affine, whose gamma and beta are kept in shared memory behind the
    // row buffers
    const int64_t rows_pad = (a.rows + 127) & ~(int64_t)127;
    const int64_t r0 = (int64_t)blockIdx.x * per_cta;
    const int64_t r1 = r0 + per_cta < rows_pad ? r0 + per_cta : rows_pad;
    const int64_t rreal = r1 < a.rows ? r1 : a.rows;                   // real rows end here
    float* aff = reinterpret_cast<float*>(smem + (size_t)warps * 2 * rowbytes);
    const int64_t per = ((a.gamma ? 1 : 0) + (a.beta ? 1 : 0)) * a.k;
    const auto group_of = [&](int64_t r) { return a.rows_per_group > 0 ? r / a.rows_per_group : (int64_t)0; };
    int64_t cached[2] = {-1, -1};
    if (r0 < a.rows) {
        cached[0] = group_of(r0);
        cached[1] = group_of(rreal - 1) != cached[0] ? group_of(rreal - 1) : -1;
    }
    if (threadIdx.x == 0) {
        abort_sh = 0;
        for (int i = 0; i < 2 * kLnMaxWarps; ++i) mbar_init(&bars[i], 1);
        fence_barrier_init();
    }
    for (int slot = 0; slot < 2 && per > 0; ++slot) {
        if (cached[slot] < 0) continue;
        float* g = aff + slot * per;
        float* b = g + (a.gamma ? a.k : 0);
        for (int64_t j = threadIdx.x; j < a.k; j += kLnThreads) {
            if (a.gamma) g[ln_affine_slot(j)] = a.gamma[cached[slot] * a.k + j];
            if (a.beta) b[ln_affine_slot(j)] = a.beta[cached[slot] * a.k + j];
        }
    }
    __syncthreads();
    WaitCtx wc{&abort_sh, a.dev_status};
    const bool active = warp < warps;             // warps beyond the row buffers idle
    LnStream st{smem + (size_t)warp * 2 * rowbytes, &bars[2 * warp], 0u, rowbytes, 0u};
    // this warp's real rows: r0 + warp + i * warps, i < n_real
    const int64_t first = r0 + warp;
    const int64_t n_real = active && first < rreal ? (rreal - 1 - first) / warps + 1 : 0;
    bool ok = true;
    if (kDynamic) {
        // ---- phase 1: largest |y| over this warp's rows, in order
        float m = 0.0f;
        bool nonfinite = false;
        if (n_real > 0) st.issue(a, first, 0, lane);
        for (int64_t i = 0; i < n_real; ++i) {
            const int b = (int)(i & 1);
            if (i + 1 < n_real) st.issue(a, first + (i + 1) * warps, b ^ 1, lane);
            const uint4* row = st.wait(b, wc, ok);
            const int64_t r = first + i * warps;
            if (ok) {
                float mu32, rstd32;
                m = fmaxf(m, ln_row_amax(a, row, ln_affine(a, r, cached, aff), lane, nonfinite, mu32, rstd32));
                if (i < kLnStatRows && lane == 0) row_stats[warp][i] = make_float2(mu32, rstd32);
            }
            __syncwarp();
        }
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (__any_sync(0xffffffffu, nonfinite) && lane == 0 && a.dev_status)
            atomicCAS(a.dev_status, 0, (int)NVFP4_ERR_NONFINITE);
        if (lane == 0) red[warp] = active ? m : 0.0f;
        __syncthreads();
        if (warp == 0) {
            float tm = lane < kLnMaxWarps ? red[lane] : 0.0f;
            for (int o = 16; o > 0; o >>= 1) tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, o));
            if (lane == 0) {
                const unsigned long long word = ((unsigned long long)a.gen << 32) | __float_as_uint(tm);
                asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(a.slots + blockIdx.x), "l"(word) : "memory");
            }
            // ---- every CTA's slot carries this generation: the tensor maximum
            float mx = 0.0f;
            bool done = true;
            const uint64_t t0 = globaltimer_ns();
            for (int i = lane; i < (int)gridDim.x; i += 32) {
                unsigned long long w;
                uint32_t n = 0;
                while (true) {
                    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(a.slots + i) : "memory");
                    if ((uint32_t)(w >> 32) == a.gen) break;
                    if ((++n & 63u) == 0u && globaltimer_ns() - t0 > kWaitLimitNs) { done = false; break; }
                }
                if (!done) break;
                mx = fmaxf(mx, __uint_as_float((uint32_t)w));
            }
            done = __all_sync(0xffffffffu, done ? 1 : 0) != 0;
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (lane == 0) {
                if (!done && a.dev_status) atomicExch(a.dev_status, (int)NVFP4_ERR_TIMEOUT);
                const float g = __fdiv_rn(mx, 2688.0f);
                if (blockIdx.x == 0 && done) *a.tensor_scale = g;
                sc_sh = scale_consts(g);
                ok_sh = done ? 1 : 0;
            }
        }
        __syncthreads();
        ok = ok && ok_sh != 0;
    } else {
        if (threadIdx.x == 0) sc_sh = scale_consts(*a.tensor_scale);
        __syncthreads();
    }
    if (!ok || !active) {                         // gave up waiting: outputs unspecified
        if (active && lane == 0) st.drain(a.dev_status);
        return;
    }
    const ScaleConsts sc = sc_sh;
    // ---- phase 2 (or the only phase): the warp's rows last first (so the
    // first ones find what phase 1 read last still in L2), then its padding
    // rows of the scale layout
    if (n_real > 0) st.issue(a, first + (n_real - 1) * warps, 0, lane);
    for (int64_t i = 0; i < n_real; ++i) {
        const int b = (int)(i & 1);
        if (i + 1 < n_real) st.issue(a, first + (n_real - 2 - i) * warps, b ^ 1, lane);
        const uint4* row = st.wait(b, wc, ok);
        const int64_t ir = n_real - 1 - i;
        const int64_t r = first + ir * warps;
        if (ok)
            ln_quantize_row(a, row, ln_affine(a, r, cached, aff), r, lane, sc,
                            kDynamic && ir < kLnStatRows ? &row_stats[warp][ir] : nullptr);
        __syncwarp();
    }
    for (int64_t r = first + n_real * warps; r < r1; r += warps)
        if (r >= a.rows) ln_quantize_row(a, nullptr, {nullptr, nullptr, false}, r, lane, sc);
    if (!ok && lane == 0) st.drain(a.dev_status);
}

cudaError_t launch_layernorm_quantize(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, const float* gamma,
                                      const float* beta, int64_t rows_per_group, double eps, uint8_t* codes,
                                      uint8_t* sf, float* tensor_scale, bool scale_given, unsigned long long* slots,
                                      uint32_t gen, int* dev_status, int num_sms, cudaStream_t stream) {
    LnArgs a{x, rows, k, ld, gamma, beta, rows_per_group, eps, codes, sf, tensor_scale, slots, gen, dev_status};
    if (k > kLnMaxK) return cudaErrorInvalidValue;
    // shared memory: two row buffers per warp, as many warps as fit the
    // budget, then the affine of two groups
    const int affine = (gamma ? 1 : 0) + (beta ? 1 : 0);
    const int affine_bytes = 2 * affine * (int)(4 * k);
    int warps = (int)((kLnSmemBudget - affine_bytes) / (2 * 2 * k));
    if (warps > kLnMaxWarps) warps = kLnMaxWarps;
    if (warps < 1) warps = 1;
    const int smem = warps * 2 * (int)(2 * k) + affine_bytes + 128;
    const int64_t rows_pad = (rows + 127) & ~(int64_t)127;
    auto kern = scale_given ? layernorm_quantize_kernel<false> : layernorm_quantize_kernel<true>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kLnThreads, smem);
    if (e != cudaSuccess) return e;
    int64_t grid = (int64_t)per_sm * num_sms;
    if (!scale_given && grid > kFusedSlots) grid = kFusedSlots;
    const int64_t want = (rows_pad + warps - 1) / warps;
    if (grid > want) grid = want;
    if (grid < 1) return cudaErrorInvalidValue;
    const int64_t per_cta = (rows_pad + grid - 1) / grid;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;           // every CTA resident at once (the handoff)
    attr[0].val.cooperative = 1;
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kLnThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = scale_given ? 0 : 1;
    e = cudaLaunchKernelEx(&cfg, kern, a, warps, per_cta);
    if (e != cudaSuccess) return e;
    count_launch(1);
    return cudaGetLastError();
}

int64_t layernorm_max_k() { return kLnMaxK; }

}  // namespace nvfp4
