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
// Kernel shape (one CTA per SM, persistent, 512 threads):
//   warp 0      TMA producer: X tile (128 x 64 bf16, 128-byte swizzle), the
//               weight codes (256 rows x 32 bytes) and two scale atoms.
//   warp 1      MMA issuer: 4 x tcgen05.mma kind::f16 (M=128, N=256, K=16)
//               per stage into one of two TMEM accumulators.
//   warps 4-11  dequantizers: thread t owns weight row t of the tile; it
//               reads its 32 code bytes and its 4 scale bytes and writes 64
//               bf16 values as one 128-byte row of the swizzled K-major B
//               tile (fence.proxy.async, then an arrive per warp).
//   warps 12-15 epilogue: tcgen05.ld, alpha = g_w, bf16 / FP32, TMA stores.
// TMEM: accumulators at columns [0,256) and [256,512); no scale factors live
// in TMEM (the tensor core sees plain bf16).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"
#include "tmap.h"

namespace nvfp4 {
namespace w4a16 {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;                            // bf16 elements per stage (128-byte rows)
constexpr int A_BYTES = BM * BK * 2;              // 16 KB
constexpr int B_BYTES = BN * BK * 2;              // 32 KB, dequantized bf16
constexpr int C_BYTES = BN * BK / 2;              // 8 KB of codes
constexpr int SF_ATOM = 512;
constexpr int S_BYTES = 2 * SF_ATOM;              // two 128-row scale atoms
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + C_BYTES + S_BYTES;   // 58368 = 57 KB
constexpr int kThreads = 512;
constexpr int kDeqWarps = 8;
constexpr int kEpiWarps = 4;
constexpr int kGroupM = 16;
constexpr int kSmemLimit = 232448;

enum OutKind { OUT_BF16 = 0, OUT_F32 = 1 };

template <int OUT>
struct Cfg {
    static constexpr int EPI_BUF = OUT == OUT_F32 ? 4096 : 2048;
    static constexpr int EPI_BYTES = kEpiWarps * 2 * EPI_BUF;
    static constexpr int FIT = (kSmemLimit - 1024 - EPI_BYTES) / STAGE_BYTES;
    static constexpr int STAGES = FIT < 4 ? FIT : 4;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024;
    static_assert(STAGES >= 3, "pipeline depth");
};

struct Params {
    const float* w_scale;
    int M, N, K;
    int num_mb, num_nb, num_tiles;
    int* dev_status;
};

__device__ __forceinline__ void tile_coords(int t, int num_mb, int num_nb, int& mb, int& nb) {
    const int per_group = kGroupM * num_nb;
    const int group = t / per_group;
    const int first = group * kGroupM;
    const int gm = min(kGroupM, num_mb - first);
    const int idx = t - group * per_group;
    mb = first + idx % gm;
    nb = idx / gm;
}

// Two E2M1 codes (one byte, element 2j in the low nibble) times an f16 scale
// pair -> a bf16x2 word (low element in the low half).  Every step is exact.
__device__ __forceinline__ uint32_t dequant_pair(uint32_t byte, uint32_t scale_h2) {
    uint32_t h2, out;
    asm("{\n\t.reg .b8 c;\n\t.reg .b16 lo, hi;\n\t.reg .b32 p;\n\t.reg .f32 f0, f1;\n\t"
        "cvt.u8.u32 c, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 p, c;\n\t"
        "mul.rn.f16x2 p, p, %2;\n\t"
        "mov.b32 {lo, hi}, p;\n\t"
        "cvt.f32.f16 f0, lo;\n\t"
        "cvt.f32.f16 f1, hi;\n\t"
        "cvt.rn.bf16x2.f32 %0, f1, f0;\n\t}"
        : "=r"(out)
        : "r"(byte), "r"(scale_h2));
    (void)h2;
    return out;
}

// E4M3 byte -> f16 scale replicated in both halves.
__device__ __forceinline__ uint32_t e4m3_to_h2(uint32_t code) {
    uint32_t h2;
    const uint16_t in = (uint16_t)((code & 0xFFu) | ((code & 0xFFu) << 8));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return h2;
}

template <int OUT>
__global__ void __launch_bounds__(kThreads, 1)
gemm_w4a16_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_codes,
                  const __grid_constant__ CUtensorMap tmap_sf, const __grid_constant__ CUtensorMap tmap_y,
                  const Params p) {
    using C = Cfg<OUT>;
    constexpr int STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[STAGES], deq_bar[STAGES], empty_bar[STAGES];
    __shared__ __align__(8) uint64_t accf_bar[2], acce_bar[2], drain_bar;
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
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accf_bar[b], 1);
            mbar_init(&acce_bar[b], kEpiWarps);
        }
        mbar_init(&drain_bar, 1);
        fence_barrier_init();
        tma_prefetch_desc(&tmap_x);
        tma_prefetch_desc(&tmap_codes);
        tma_prefetch_desc(&tmap_sf);
        tma_prefetch_desc(&tmap_y);
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

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol_x = policy_evict_normal();
            const uint64_t pol_w = policy_evict_last();
            int stage = 0;
            uint32_t phase = 0, issued = 0, issued_any = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
                int mb, nb;
                tile_coords(t, p.num_mb, p.num_nb, mb, nb);
                for (int kt = 0; kt < num_kt; ++kt) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1u, wc)) { ok = false; break; }
                    uint8_t* sb = smem + stage * STAGE_BYTES;
                    mbar_arrive_expect_tx(&full_bar[stage], A_BYTES + C_BYTES + S_BYTES);
                    tma_load_2d(sb, &tmap_x, &full_bar[stage], kt * BK, mb * BM, pol_x);
                    tma_load_2d(sb + A_BYTES + B_BYTES, &tmap_codes, &full_bar[stage], kt * (BK / 2), nb * BN, pol_w);
                    tma_load_2d(sb + A_BYTES + B_BYTES + C_BYTES, &tmap_sf, &full_bar[stage], 0,
                                (nb * 2) * k_atoms + kt, pol_w);
                    tma_load_2d(sb + A_BYTES + B_BYTES + C_BYTES + SF_ATOM, &tmap_sf, &full_bar[stage], 0,
                                (nb * 2 + 1) * k_atoms + kt, pol_w);
                    issued = (issued & ~(1u << stage)) | (phase << stage);
                    issued_any |= 1u << stage;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            int no_abort = 0;
            WaitCtx w2{&no_abort, p.dev_status};
            for (int s = 0; s < STAGES; ++s)
                if (issued_any & (1u << s)) mbar_wait(&full_bar[s], (issued >> s) & 1u, w2);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(BM, BN);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
                if (!mbar_wait(&acce_bar[acc], acc_phase ^ 1u, wc)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN;
                for (int kt = 0; kt < num_kt; ++kt) {
                    if (!mbar_wait(&deq_bar[stage], phase, wc)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sb = smem_u32(smem + stage * STAGE_BYTES);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        tc_mma_bf16(d_tmem, sdesc_kmajor_sw128(sb + ks * 32), sdesc_kmajor_sw128(sb + A_BYTES + ks * 32),
                                    idesc, (kt | ks) != 0 ? 1u : 0u);
                    tc_commit(&empty_bar[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit(&accf_bar[acc]);
                if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
            }
            tc_commit(&drain_bar);
            int no_abort = 0;
            WaitCtx w2{&no_abort, p.dev_status};
            mbar_wait(&drain_bar, 0, w2);
        }
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
                    const uint32_t sh2 = e4m3_to_h2(sfw >> (8 * (j >> 1)));   // block j/2
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
    } else if (warp >= 12) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const float alpha = *p.w_scale;
        uint8_t* ebuf = smem + STAGES * STAGE_BYTES + (warp - 12) * 2 * C::EPI_BUF;
        int acc = 0, nstore = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
            int mb, nb;
            tile_coords(t, p.num_mb, p.num_nb, mb, nb);
            if (!__all_sync(0xffffffffu, mbar_wait(&accf_bar[acc], acc_phase, wc) ? 1 : 0)) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
            const int m0 = mb * BM + q * 32, n0 = nb * BN;
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tbase + c * 32, r);
                tmem_ld_wait();
                if (n0 + c * 32 >= p.N) continue;
                uint8_t* buf = ebuf + (nstore & 1) * C::EPI_BUF;
                if (lane == 0) bulk_wait_group_read<1>();
                __syncwarp();
                if (OUT == OUT_BF16) {
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(alpha, __uint_as_float(r[2 * j])),
                                                                 __fmul_rn(alpha, __uint_as_float(r[2 * j + 1])));
                        pk[j] = *reinterpret_cast<uint32_t*>(&h);
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int pos = j ^ ((lane >> 1) & 3);
                        *reinterpret_cast<uint4*>(buf + lane * 64 + pos * 16) =
                            make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int pos = j ^ (lane & 7);
                        *reinterpret_cast<float4*>(buf + lane * 128 + pos * 16) =
                            make_float4(__fmul_rn(alpha, __uint_as_float(r[4 * j])), __fmul_rn(alpha, __uint_as_float(r[4 * j + 1])),
                                        __fmul_rn(alpha, __uint_as_float(r[4 * j + 2])), __fmul_rn(alpha, __uint_as_float(r[4 * j + 3])));
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmap_y, buf, n0 + c * 32, m0);
                    bulk_commit_group();
                }
                ++nstore;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce_bar[acc]);
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
        if (lane == 0) bulk_wait_group<0>();
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
    using C = Cfg<OUT>;
    CUtensorMap tx, tc, ts, ty;
    const uint64_t atoms = (uint64_t)((a.N + 127) / 128) * (uint64_t)(a.K / 64);
    if (make_tmap_2d(&tx, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.K * 2,
                     BK, BM, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
        make_tmap_2d(&tc, a.w_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)(a.K / 2), (uint64_t)a.N,
                     (uint64_t)(a.K / 2), BK / 2, BN, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS ||
        make_tmap_2d(&ts, a.w_sf, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, 128, atoms, SF_ATOM, 128, 1,
                     CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    CUresult r;
    if (OUT == OUT_BF16)
        r = make_tmap_2d(&ty, a.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.N, (uint64_t)a.M,
                         (uint64_t)a.N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
    else
        r = make_tmap_2d(&ty, a.y, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)a.N, (uint64_t)a.M,
                         (uint64_t)a.N * 4, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;

    Params p;
    p.w_scale = a.w_scale;
    p.M = (int)a.M;
    p.N = (int)a.N;
    p.K = (int)a.K;
    p.num_mb = (int)((a.M + BM - 1) / BM);
    p.num_nb = (int)((a.N + BN - 1) / BN);
    p.num_tiles = p.num_mb * p.num_nb;
    p.dev_status = a.dev_status;
    auto kern = gemm_w4a16_kernel<OUT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int grid = p.num_tiles < num_sms ? p.num_tiles : num_sms;
    kern<<<grid, kThreads, C::SMEM_BYTES, stream>>>(tx, tc, ts, ty, p);
    count_launch(1);
    return cudaGetLastError();
}

}  // namespace w4a16

cudaError_t launch_gemm_w4a16(const GemmW4A16Args& a, int num_sms, cudaStream_t stream) {
    if (a.M == 0) return cudaSuccess;
    if (a.y_dtype == 1) return w4a16::launch_out<w4a16::OUT_F32>(a, num_sms, stream);
    return w4a16::launch_out<w4a16::OUT_BF16>(a, num_sms, stream);
}

}  // namespace nvfp4
