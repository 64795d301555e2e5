// gemm_w4a16.cu -- weights-only NVFP4 GEMM: bf16 activations times NVFP4
// weights, the weight dequantization fused into the tcgen05 mainloop.
//
// Operation ("[RFC]: NVFP4 Quantization Support for Diffusion Models", Open
// Questions 1: weight-only W4A16; "Add NVFP4 weights-only quantization support
// to fit Kandinsky-5 Pro into 24 GB VRAM", Changes):
//   Y[m,n] = g_w * sum_k x[m,k] * (e2m1(w[n,k]) * e4m3(sfw[n, k/16]))
// The weight element e2m1 * e4m3 has at most 6 significant bits and lies in
// [2^-10, 2688], so it is exact in f16 and in bf16: the bf16 MMA sees the
// exact dequantized weight, FP32 accumulates in TMEM, g_w is applied in the
// epilogue.
//
// Kernel shape (one CTA per SM, persistent, 640 threads): a 256 x 256 output
// tile per CTA, as two 128-row halves that share each dequantized weight
// stage (the dequantization, not the MMA, bounds a 128-row tile: sharing it
// halves the dequantization per FLOP).
//   warp 0      TMA producer: X tile (256 x 64 bf16, 128-byte swizzle), the
//               weight codes (256 rows x 32 bytes) and two scale atoms.
//   warp 1      MMA issuer: per stage 8 x tcgen05.mma kind::f16 (M=128,
//               N=256, K=16), four per row half, into TMEM columns [0,256)
//               (rows 0-127) and [256,512) (rows 128-255).
//   warps 4-11  dequantizers: thread t owns weight row t of the tile; it
//               reads its 32 code bytes and its 4 scale bytes and writes 64
//               bf16 values as one 128-byte row of the swizzled K-major B
//               tile (fence.proxy.async, then an arrive per warp).  Per two
//               weights: E2M1 pair -> f16 pair, a 3-bit shift that turns it
//               into bf16 times 2^-112, one bf16 multiply by the scale.
//   warps 12-19 epilogue: warp w reads TMEM lane quarter w % 4 of row half
//               (w - 12) / 4 in 32-column chunks, applies alpha = g_w and
//               stores bf16 / FP32 rows straight from registers (16-byte
//               stores; shared memory is all pipeline stages).
// Producer and MMA issuer run on whole warps with one elected lane issuing,
// so descriptors, coordinates and addresses stay warp-uniform.
// TMEM: both accumulators fill its 512 columns, so the MMA issuer waits at a
// tile boundary until the epilogue has read them (a few thousand cycles per
// tile of K/64 stages of ~1100 cycles each).
#include <cstdlib>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "gemm.h"
#include "ptx.cuh"
#include "tmap.h"

namespace nvfp4 {
namespace w4a16 {

constexpr int BM = 256;                           // two 128-row MMA halves
constexpr int BN = 256;
constexpr int BK = 64;                            // bf16 elements per stage (128-byte rows)
constexpr int A_HALF = 128 * BK * 2;              // 16 KB per row half
constexpr int A_BYTES = BM * BK * 2;              // 32 KB
constexpr int B_BYTES = BN * BK * 2;              // 32 KB, dequantized bf16
constexpr int C_BYTES = BN * BK / 2;              // 8 KB of codes
constexpr int SF_ATOM = 512;
constexpr int S_BYTES = 2 * SF_ATOM;              // two 128-row scale atoms
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + C_BYTES + S_BYTES;   // 74752 = 73 KB
constexpr int kThreads = 640;
constexpr int kDeqWarps = 8;
constexpr int kEpiWarps = 8;
constexpr int kEpiWarp0 = 12;
constexpr int kGroupM = 8;
constexpr int kSmemLimit = 232448;
constexpr int STAGES = (kSmemLimit - 1024) / STAGE_BYTES;   // 3
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;
static_assert(STAGES >= 3, "pipeline depth");

enum OutKind { OUT_BF16 = 0, OUT_F32 = 1 };

struct Params {
    const float* w_scale;
    void* y;
    int M, N, K;
    int num_mb, num_nb, num_tiles;
    int* dev_status;
};

// Tile t of an M-block-grouped order: groups of GM M blocks, N blocks outer
// within a group, so the tiles in flight share few X row blocks.
template <int GM = kGroupM>
__device__ __forceinline__ void tile_coords(int t, int num_mb, int num_nb, int& mb, int& nb) {
    const int per_group = GM * num_nb;
    const int group = t / per_group;
    const int first = group * GM;
    const int gm = min(GM, num_mb - first);
    const int idx = t - group * per_group;
    mb = first + idx % gm;
    nb = idx / gm;
}

// Two E2M1 codes (one byte, element 2j in the low nibble) times a block
// scale -> a bf16x2 word (low element in the low half).  Every step is exact:
// the E2M1 pair is converted to f16; an E2M1 value in f16 has a zero low
// mantissa (1 significant bit after the leading one), so moving the f16
// exponent and mantissa down 3 bits yields the bf16 pattern of the same
// value times 2^-112 (zero stays zero, the sign stays in place); one bf16
// multiply by the scale times 2^112 then gives the weight (at most 6
// significant bits, within [2^-10, 2688]).
__device__ __forceinline__ uint32_t dequant_pair(uint32_t byte, uint32_t scale_b2) {
    uint32_t h2, out;
    asm("{\n\t.reg .b8 c;\n\t"
        "cvt.u8.u32 c, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, c;\n\t}"
        : "=r"(h2)
        : "r"(byte));
    const uint32_t b2 = ((h2 >> 3) & 0x0FFF0FFFu) | (h2 & 0x80008000u);
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(out) : "r"(b2), "r"(scale_b2));
    return out;
}

// E4M3 byte -> bf16 of (scale * 2^112) in both halves (exact: 4 significant
// bits, exponent within bf16's range).
__device__ __forceinline__ uint32_t e4m3_to_b2_scaled(uint32_t code) {
    uint32_t h2;
    const uint16_t in = (uint16_t)(code & 0xFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    __half_raw hr;
    hr.x = (unsigned short)(h2 & 0xFFFFu);
    const float f = __half2float(__half(hr)) * 0x1p112f;
    const uint32_t b = __float_as_uint(f) >> 16;          // exact: the low 16 bits are zero
    return b | (b << 16);
}

// 32 accumulator columns of one output row (n .. n + 31, n < N), times alpha,
// stored as bf16 (16-byte stores) or FP32; columns at or past N are skipped.
template <int OUT>
__device__ __forceinline__ void store_row_chunk(const Params& p, int64_t row, int n, float alpha,
                                                const uint32_t (&r)[32]) {
    if (OUT == OUT_BF16) {
        uint16_t* dst = static_cast<uint16_t*>(p.y) + row * p.N + n;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (n + 8 * j >= p.N) break;
            uint32_t pk[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(alpha, __uint_as_float(r[8 * j + 2 * i])),
                                                          __fmul_rn(alpha, __uint_as_float(r[8 * j + 2 * i + 1])));
                pk[i] = *reinterpret_cast<uint32_t*>(&b2);
            }
            *reinterpret_cast<uint4*>(dst + 8 * j) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
    } else {
        float* dst = static_cast<float*>(p.y) + row * p.N + n;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (n + 4 * j >= p.N) break;
            *reinterpret_cast<float4*>(dst + 4 * j) =
                make_float4(__fmul_rn(alpha, __uint_as_float(r[4 * j])), __fmul_rn(alpha, __uint_as_float(r[4 * j + 1])),
                            __fmul_rn(alpha, __uint_as_float(r[4 * j + 2])), __fmul_rn(alpha, __uint_as_float(r[4 * j + 3])));
        }
    }
}

template <int OUT>
__global__ void __launch_bounds__(kThreads, 1)
gemm_w4a16_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_codes,
                  const __grid_constant__ CUtensorMap tmap_sf, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[STAGES], deq_bar[STAGES], empty_bar[STAGES];
    __shared__ __align__(8) uint64_t accf_bar, acce_bar, drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    WaitCtx wc{&abort_sh, p.dev_status};

    if (threadIdx.x == 0) {
        abort_sh = 0;
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&deq_bar[s], kDeqWarps);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&accf_bar, 1);
        mbar_init(&acce_bar, kEpiWarps);
        mbar_init(&drain_bar, 1);
        fence_barrier_init();
        tma_prefetch_desc(&tmap_x);
        tma_prefetch_desc(&tmap_codes);
        tma_prefetch_desc(&tmap_sf);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;

    const int num_kt = p.K / BK;
    const int k_atoms = p.K / 64;                 // scale atoms per 128-row block

    // Producer and MMA issuer run on whole warps with one elected lane issuing,
    // so descriptors, coordinates and addresses stay warp-uniform (issued from
    // a single lane they cost about as much to issue as the MMAs take to run).
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        const uint64_t pol_x = policy_evict_normal();
        const uint64_t pol_w = policy_evict_last();
        int stage = 0;
        uint32_t phase = 0, issued = 0, issued_any = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
            int mb, nb;
            tile_coords(t, p.num_mb, p.num_nb, mb, nb);
            for (int kt = 0; kt < num_kt; ++kt) {
                if (!__all_sync(0xffffffffu, mbar_wait(&empty_bar[stage], phase ^ 1u, wc) ? 1 : 0)) {
                    ok = false;
                    break;
                }
                uint8_t* sb = smem + stage * STAGE_BYTES;
                if (elect_one()) {
                    mbar_arrive_expect_tx(&full_bar[stage], A_BYTES + C_BYTES + S_BYTES);
                    tma_load_2d(sb + A_BYTES + B_BYTES, &tmap_codes, &full_bar[stage], kt * (BK / 2), nb * BN, pol_w);
                    tma_load_2d(sb + A_BYTES + B_BYTES + C_BYTES, &tmap_sf, &full_bar[stage], 0,
                                (nb * 2) * k_atoms + kt, pol_w);
                    tma_load_2d(sb + A_BYTES + B_BYTES + C_BYTES + SF_ATOM, &tmap_sf, &full_bar[stage], 0,
                                (nb * 2 + 1) * k_atoms + kt, pol_w);
                    tma_load_2d(sb, &tmap_x, &full_bar[stage], kt * BK, mb * BM, pol_x);
                }
                __syncwarp();
                issued = (issued & ~(1u << stage)) | (phase << stage);
                issued_any |= 1u << stage;
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
        }
        if (lane == 0) {
            int no_abort = 0;
            WaitCtx w2{&no_abort, p.dev_status};
            for (int s = 0; s < STAGES; ++s)
                if (issued_any & (1u << s)) mbar_wait(&full_bar[s], (issued >> s) & 1u, w2);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = idesc_bf16(128, BN);
        const uint32_t smem0 = smem_u32(smem);
        int stage = 0;
        uint32_t phase = 0, acc_phase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
            if (!__all_sync(0xffffffffu, mbar_wait(&acce_bar, acc_phase ^ 1u, wc) ? 1 : 0)) {
                ok = false;
                break;
            }
            tc_fence_after();
            for (int kt = 0; kt < num_kt; ++kt) {
                if (!__all_sync(0xffffffffu, mbar_wait(&deq_bar[stage], phase, wc) ? 1 : 0)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sb = smem0 + stage * STAGE_BYTES;
                if (elect_one()) {
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t bdesc = sdesc_kmajor_sw128(sb + A_BYTES + ks * 32);
                        tc_mma_bf16(tmem_base, sdesc_kmajor_sw128(sb + ks * 32), bdesc, idesc, (kt | ks) != 0 ? 1u : 0u);
                        tc_mma_bf16(tmem_base + BN, sdesc_kmajor_sw128(sb + A_HALF + ks * 32), bdesc, idesc,
                                    (kt | ks) != 0 ? 1u : 0u);
                    }
                    tc_commit(&empty_bar[stage]);
                }
                __syncwarp();
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
            if (elect_one()) tc_commit(&accf_bar);
            __syncwarp();
            acc_phase ^= 1u;
        }
        if (elect_one()) tc_commit(&drain_bar);
        __syncwarp();
        int no_abort = 0;
        WaitCtx w2{&no_abort, p.dev_status};
        mbar_wait(&drain_bar, 0, w2);
    } else if (warp >= 4 && warp < 4 + kDeqWarps) {
        // ------------------------------------------------------------ dequantizers
        const int row = (warp - 4) * 32 + lane;       // weight row inside the tile
        const int sf_off = (row >> 7) * SF_ATOM + (row & 31) * 16 + ((row & 127) >> 5) * 4;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
            for (int kt = 0; kt < num_kt; ++kt) {
                if (!__all_sync(0xffffffffu, mbar_wait(&full_bar[stage], phase, wc) ? 1 : 0)) { ok = false; break; }
                uint8_t* sb = smem + stage * STAGE_BYTES;
                const uint4* cp = reinterpret_cast<const uint4*>(sb + A_BYTES + B_BYTES + row * 32);
                const uint4 c0 = cp[0], c1 = cp[1];
                const uint32_t sfw = *reinterpret_cast<const uint32_t*>(sb + A_BYTES + B_BYTES + C_BYTES + sf_off);
                const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                uint8_t* brow = sb + A_BYTES + row * 128;
#pragma unroll
                for (int j = 0; j < 8; ++j) {             // 16-byte chunk j: elements 8j .. 8j+7
                    const uint32_t sh2 = e4m3_to_b2_scaled(sfw >> (8 * (j >> 1)));   // block j/2
                    const uint32_t w = cw[j];
                    uint4 o;
                    o.x = dequant_pair(w & 0xFFu, sh2);
                    o.y = dequant_pair((w >> 8) & 0xFFu, sh2);
                    o.z = dequant_pair((w >> 16) & 0xFFu, sh2);
                    o.w = dequant_pair(w >> 24, sh2);
                    *reinterpret_cast<uint4*>(brow + ((j ^ (row & 7)) * 16)) = o;   // 128-byte swizzle
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&deq_bar[stage]);
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
        }
    } else if (warp >= kEpiWarp0) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const int h = (warp - kEpiWarp0) >> 2;        // row half (accumulator)
        const float alpha = *p.w_scale;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
            int mb, nb;
            tile_coords(t, p.num_mb, p.num_nb, mb, nb);
            if (!__all_sync(0xffffffffu, mbar_wait(&accf_bar, acc_phase, wc) ? 1 : 0)) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + h * BN;
            const int64_t row = (int64_t)mb * BM + h * 128 + q * 32 + lane;
            const int n0 = nb * BN;
            const bool row_ok = row < p.M;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tbase + c * 32, r);
                tmem_ld_wait();
                if (c == BN / 32 - 1) {
                    // the whole accumulator is in registers or stored: release TMEM
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acce_bar);
                }
                const int n = n0 + c * 32;
                if (!row_ok || n >= p.N) continue;
                store_row_chunk<OUT>(p, row, n, alpha, r);
            }
            acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

template <int OUT>
cudaError_t launch_out(const GemmW4A16Args& a, int num_sms, cudaStream_t stream) {
    CUtensorMap tx, tc, ts;
    const uint64_t atoms = (uint64_t)((a.N + 127) / 128) * (uint64_t)(a.K / 64);
    if (make_tmap_2d(&tx, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.K * 2,
                     BK, BM, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
        make_tmap_2d(&tc, a.w_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)(a.K / 2), (uint64_t)a.N,
                     (uint64_t)(a.K / 2), BK / 2, BN, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS ||
        make_tmap_2d(&ts, a.w_sf, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, 128, atoms, SF_ATOM, 128, 1,
                     CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;

    Params p;
    p.w_scale = a.w_scale;
    p.y = a.y;
    p.M = (int)a.M;
    p.N = (int)a.N;
    p.K = (int)a.K;
    p.num_mb = (int)((a.M + BM - 1) / BM);
    p.num_nb = (int)((a.N + BN - 1) / BN);
    p.num_tiles = p.num_mb * p.num_nb;
    p.dev_status = a.dev_status;
    auto kern = gemm_w4a16_kernel<OUT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int grid = p.num_tiles < num_sms ? p.num_tiles : num_sms;
    kern<<<grid, kThreads, SMEM_BYTES, stream>>>(tx, tc, ts, p);
    count_launch(1);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// CTA pairs (cta_group::2).  The single-CTA kernel above moves ~176 KB
// through shared memory per 1024-cycle stage (the MMAs read the 32 KB B tile
// once per row half, plus the X and code loads and the dequantizer's reads
// and writes), more than the ~128 bytes per cycle an SM's shared memory
// delivers.  A pair shares one 512 x 256 output tile: each CTA holds 256 rows
// of X (two 128-row halves) and dequantizes 128 of the 256 weight rows, and
// each M=256, N=256 pair MMA reads 128 B rows from each CTA -- per SM and
// stage ~120 KB (X 32, codes 4, dequantizer 4 + 16, MMA operands 64).
//   warp 0      producer, both CTAs: this CTA's X rows (256 x 64 bf16), its
//               weight codes (128 rows x 32 bytes) and scale atom, on its own
//               "full" barrier.
//   warp 1      leader CTA: MMA issuer.  Per stage and row half four
//               tcgen05.mma cta_group::2 kind::f16 (M=256, N=256, K=16) into
//               TMEM columns [256 h, 256 h + 256) of both CTAs; one commit per
//               stage multicast to both CTAs' "empty" barriers, one per tile
//               to both "accf" barriers.
//   warps 4-11  dequantizers, both CTAs: two threads per weight row (32
//               values each) into the 128-byte-swizzled K-major B half; then a
//               proxy fence and one arrive per warp on the LEADER's "deq"
//               barrier (each SM's tensor core reads its own CTA's half, so a
//               CTA-scope release suffices), which thus also tells the MMA
//               issuer that both CTAs' X tiles landed.
//   warps 12-19 epilogue, both CTAs: as in the single-CTA kernel, on this
//               CTA's 256 rows; the accumulators are handed back with one
//               arrive per warp on the leader's "acce" barrier.
// No load uses cluster multicast: every CTA fetches its own tiles.
namespace pair {

constexpr int PM = 512;                           // X rows per pair tile (256 per CTA)
constexpr int PN = 256;                           // weight rows per pair tile (128 per CTA)
constexpr int A2_BYTES = 256 * BK * 2;            // 32 KB: this CTA's X rows
constexpr int B2_BYTES = 128 * BK * 2;            // 16 KB: this CTA's dequantized weight rows
constexpr int C2_BYTES = 128 * BK / 2;            // 4 KB of codes
constexpr int STAGE2_BYTES = 54272;               // the above + one 512-byte scale atom, 1 KB aligned
static_assert(A2_BYTES + B2_BYTES + C2_BYTES + SF_ATOM <= STAGE2_BYTES && STAGE2_BYTES % 1024 == 0, "stage layout");
constexpr int STAGES2 = (kSmemLimit - 1024) / STAGE2_BYTES;      // 4
constexpr int SMEM2_BYTES = STAGES2 * STAGE2_BYTES + 1024;
static_assert(STAGES2 >= 3, "pipeline depth");
constexpr int kGroupM2 = 2;                       // 512-row X blocks per tile group

template <int OUT>
__global__ void __launch_bounds__(kThreads, 1)
gemm_w4a16_pair_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_codes,
                       const __grid_constant__ CUtensorMap tmap_sf, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    // full:  each CTA's own; its X rows, codes and scale atom of a stage landed;
    // deq:   the leader's; both CTAs' weight halves of a stage are dequantized;
    // empty: both CTAs' (multicast commit); the MMAs of a stage have completed;
    // accf:  both CTAs' (multicast commit); the accumulators hold a finished tile;
    // acce:  the leader's; both CTAs' epilogues have read the accumulators.
    __shared__ __align__(8) uint64_t full_bar[STAGES2], deq_bar[STAGES2], empty_bar[STAGES2];
    __shared__ __align__(8) uint64_t accf_bar, acce_bar, drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = (int)cluster_id_x(), npairs = (int)nclusters_x();
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    WaitCtx wc{&abort_sh, p.dev_status};

    if (threadIdx.x == 0) {
        abort_sh = 0;
        for (int s = 0; s < STAGES2; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&deq_bar[s], 2 * kDeqWarps);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&accf_bar, 1);
        mbar_init(&acce_bar, 2 * kEpiWarps);
        mbar_init(&drain_bar, 1);
        fence_barrier_init();
        tma_prefetch_desc(&tmap_x);
        tma_prefetch_desc(&tmap_codes);
        tma_prefetch_desc(&tmap_sf);
    }
    cluster_sync_all();                           // barriers initialised in both CTAs
    if (warp == 1) {
        tmem_alloc2(&tmem_base_sh, 512);
        tmem_relinquish2();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;

    const int num_kt = p.K / BK;
    const int k_atoms = p.K / 64;                 // scale atoms per 128-row block

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        const uint64_t pol_x = policy_evict_normal();
        const uint64_t pol_w = policy_evict_last();
        int stage = 0;
        uint32_t phase = 0, issued = 0, issued_any = 0;
        bool ok = true;
        for (int t = pair; t < p.num_tiles && ok; t += npairs) {
            int mb, nb;
            tile_coords<kGroupM2>(t, p.num_mb, p.num_nb, mb, nb);
            const int xrow = mb * PM + (int)rank * 256;
            const int wrow = nb * PN + (int)rank * 128;
            const int sfrow = (nb * 2 + (int)rank) * k_atoms;
            for (int kt = 0; kt < num_kt; ++kt) {
                if (!__all_sync(0xffffffffu, mbar_wait(&empty_bar[stage], phase ^ 1u, wc) ? 1 : 0)) {
                    ok = false;
                    break;
                }
                uint8_t* sb = smem + stage * STAGE2_BYTES;
                if (elect_one()) {
                    mbar_arrive_expect_tx(&full_bar[stage], A2_BYTES + C2_BYTES + SF_ATOM);
                    tma_load_2d(sb + A2_BYTES + B2_BYTES, &tmap_codes, &full_bar[stage], kt * (BK / 2), wrow, pol_w);
                    tma_load_2d(sb + A2_BYTES + B2_BYTES + C2_BYTES, &tmap_sf, &full_bar[stage], 0, sfrow + kt, pol_w);
                    tma_load_2d(sb, &tmap_x, &full_bar[stage], kt * BK, xrow, pol_x);
                }
                __syncwarp();
                issued = (issued & ~(1u << stage)) | (phase << stage);
                issued_any |= 1u << stage;
                if (++stage == STAGES2) { stage = 0; phase ^= 1u; }
            }
        }
        // this CTA's loads in flight land before it may exit
        if (lane == 0) {
            int no_abort = 0;
            WaitCtx w2{&no_abort, p.dev_status};
            for (int s = 0; s < STAGES2; ++s)
                if (issued_any & (1u << s)) mbar_wait(&full_bar[s], (issued >> s) & 1u, w2);
        }
    } else if (warp == 1) {
        if (rank == 0) {
            // -------------------------------------------------------- MMA issuer (leader)
            constexpr uint32_t idesc = idesc_bf16(256, PN);
            const uint32_t smem0 = smem_u32(smem);
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int t = pair; t < p.num_tiles && ok; t += npairs) {
                // both CTAs' epilogues have read the accumulators' previous tile
                if (!__all_sync(0xffffffffu, mbar_wait_cluster(&acce_bar, acc_phase ^ 1u, wc) ? 1 : 0)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kt = 0; kt < num_kt; ++kt) {
                    if (!__all_sync(0xffffffffu, mbar_wait_cluster(&deq_bar[stage], phase, wc) ? 1 : 0)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sb = smem0 + stage * STAGE2_BYTES;
                    if (elect_one()) {
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
                            const uint64_t bdesc = sdesc_kmajor_sw128(sb + A2_BYTES + ks * 32);
                            tc_mma2_bf16(tmem_base, sdesc_kmajor_sw128(sb + ks * 32), bdesc, idesc,
                                         (kt | ks) != 0 ? 1u : 0u);
                            tc_mma2_bf16(tmem_base + PN, sdesc_kmajor_sw128(sb + A_HALF + ks * 32), bdesc, idesc,
                                         (kt | ks) != 0 ? 1u : 0u);
                        }
                        tc_commit2_mc(&empty_bar[stage], 0x3);
                    }
                    __syncwarp();
                    if (++stage == STAGES2) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                if (elect_one()) tc_commit2_mc(&accf_bar, 0x3);
                __syncwarp();
                acc_phase ^= 1u;
            }
            if (elect_one()) tc_commit2_mc(&drain_bar, 0x1);
            __syncwarp();
            int no_abort = 0;
            WaitCtx w2{&no_abort, p.dev_status};
            mbar_wait(&drain_bar, 0, w2);
        }
    } else if (warp >= 4 && warp < 4 + kDeqWarps) {
        // ------------------------------------------------------------ dequantizers (both CTAs)
        const int tid = (warp - 4) * 32 + lane;
        const int row = tid >> 1, part = tid & 1;     // weight row of this CTA's half; values 32 part .. + 31
        const int sf_off = (row & 31) * 16 + (row >> 5) * 4 + 2 * part;   // blocks 2 part, 2 part + 1
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int t = pair; t < p.num_tiles && ok; t += npairs) {
            for (int kt = 0; kt < num_kt; ++kt) {
                if (!__all_sync(0xffffffffu, mbar_wait(&full_bar[stage], phase, wc) ? 1 : 0)) { ok = false; break; }
                uint8_t* sb = smem + stage * STAGE2_BYTES;
                const uint4 c = *reinterpret_cast<const uint4*>(sb + A2_BYTES + B2_BYTES + row * 32 + part * 16);
                const uint32_t s2 = *reinterpret_cast<const uint16_t*>(sb + A2_BYTES + B2_BYTES + C2_BYTES + sf_off);
                const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
                uint8_t* brow = sb + A2_BYTES + row * 128;
#pragma unroll
                for (int j = 0; j < 4; ++j) {             // 16-byte chunk 4 part + j: 8 values of block 2 part + j / 2
                    const uint32_t sh2 = e4m3_to_b2_scaled(s2 >> (8 * (j >> 1)));
                    const uint32_t w = cw[j];
                    uint4 o;
                    o.x = dequant_pair(w & 0xFFu, sh2);
                    o.y = dequant_pair((w >> 8) & 0xFFu, sh2);
                    o.z = dequant_pair((w >> 16) & 0xFFu, sh2);
                    o.w = dequant_pair(w >> 24, sh2);
                    *reinterpret_cast<uint4*>(brow + (((4 * part + j) ^ (row & 7)) * 16)) = o;   // 128-byte swizzle
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if (rank == 0)
                        mbar_arrive(&deq_bar[stage]);
                    else
                        mbar_arrive_remote(mapa_shared(smem_u32(&deq_bar[stage]), 0));
                }
                if (++stage == STAGES2) { stage = 0; phase ^= 1u; }
            }
        }
    } else if (warp >= kEpiWarp0) {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;
        const int h = (warp - kEpiWarp0) >> 2;        // row half (accumulator)
        const float alpha = *p.w_scale;
        uint32_t acc_phase = 0;
        for (int t = pair; t < p.num_tiles; t += npairs) {
            int mb, nb;
            tile_coords<kGroupM2>(t, p.num_mb, p.num_nb, mb, nb);
            if (!__all_sync(0xffffffffu, mbar_wait(&accf_bar, acc_phase, wc) ? 1 : 0)) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + h * PN;
            const int64_t row = (int64_t)mb * PM + (int)rank * 256 + h * 128 + q * 32 + lane;
            const int n0 = nb * PN;
            const bool row_ok = row < p.M;
#pragma unroll 1
            for (int c = 0; c < PN / 32; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tbase + c * 32, r);
                tmem_ld_wait();
                if (c == PN / 32 - 1) {
                    // the whole accumulator is in registers or stored: release TMEM
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        if (rank == 0)
                            mbar_arrive(&acce_bar);
                        else
                            mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(&acce_bar), 0));
                    }
                }
                const int n = n0 + c * 32;
                if (!row_ok || n >= p.N) continue;
                store_row_chunk<OUT>(p, row, n, alpha, r);
            }
            acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                           // the leader's MMAs are done with both CTAs' memory
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc2(tmem_base, 512);
    }
}

template <int OUT>
cudaError_t launch_out(const GemmW4A16Args& a, int num_sms, cudaStream_t stream) {
    CUtensorMap tx, tc, ts;
    const uint64_t atoms = (uint64_t)((a.N + 127) / 128) * (uint64_t)(a.K / 64);
    if (make_tmap_2d(&tx, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.K * 2,
                     BK, 256, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
        make_tmap_2d(&tc, a.w_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)(a.K / 2), (uint64_t)a.N,
                     (uint64_t)(a.K / 2), BK / 2, 128, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS ||
        make_tmap_2d(&ts, a.w_sf, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, 128, atoms, SF_ATOM, 128, 1,
                     CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;

    Params p;
    p.w_scale = a.w_scale;
    p.y = a.y;
    p.M = (int)a.M;
    p.N = (int)a.N;
    p.K = (int)a.K;
    p.num_mb = (int)((a.M + PM - 1) / PM);
    p.num_nb = (int)((a.N + PN - 1) / PN);
    p.num_tiles = p.num_mb * p.num_nb;
    p.dev_status = a.dev_status;
    auto kern = gemm_w4a16_pair_kernel<OUT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM2_BYTES);
    if (e != cudaSuccess) return e;

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = SMEM2_BYTES;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // as many pairs as can be resident at once (persistent over tiles)
    int max_clusters = 0;
    cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
    if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg) != cudaSuccess || max_clusters < 1)
        max_clusters = num_sms / 2;
    const int pairs = p.num_tiles < max_clusters ? p.num_tiles : max_clusters;
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    e = cudaLaunchKernelEx(&cfg, kern, tx, tc, ts, p);
    count_launch(1);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// Pair tiles that fill at least half the SMs' pairs go to the pair kernel
// (NVFP4_W4A16_KERNEL=single|pair forces one, for tests and measurements).
bool use(int64_t M, int64_t N, int num_sms) {
    const char* env = getenv("NVFP4_W4A16_KERNEL");
    if (env && env[0] == 's') return false;
    if (env && env[0] == 'p') return true;
    const int64_t tiles = ((M + PM - 1) / PM) * ((N + PN - 1) / PN);
    return tiles >= num_sms / 2;
}

}  // namespace pair

}  // namespace w4a16

cudaError_t launch_gemm_w4a16(const GemmW4A16Args& a, int num_sms, cudaStream_t stream) {
    if (a.M == 0) return cudaSuccess;
    if (w4a16::pair::use(a.M, a.N, num_sms)) {
        if (a.y_dtype == 1) return w4a16::pair::launch_out<w4a16::OUT_F32>(a, num_sms, stream);
        return w4a16::pair::launch_out<w4a16::OUT_BF16>(a, num_sms, stream);
    }
    if (a.y_dtype == 1) return w4a16::launch_out<w4a16::OUT_F32>(a, num_sms, stream);
    return w4a16::launch_out<w4a16::OUT_BF16>(a, num_sms, stream);
}

}  // namespace nvfp4
