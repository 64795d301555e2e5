// gemm_w4a4.cu -- block-scaled FP4 x FP4 GEMM on the 5th-generation tensor
// cores (tcgen05, kind::mxf4nvf4 with UE4M3 scales per 16 elements), FP32
// accumulation in TMEM, and an alpha epilogue that writes bf16, FP32, or the
// next layer's NVFP4 codes and scales.
//
// Operation ("NVFP4-DiT ..." README, Methodology 3: FP4-packed operands, two
// values per byte, FP32 accumulation; "[RFC]: NVFP4 Quantization Support for
// Diffusion Models", Open Questions 1: W4A4):
//   Y[m,n] = (g_a g_b) * sum_k (e2m1(a) e4m3(sfa)) (e2m1(b) e4m3(sfb))
//
// One launch may carry up to kMaxGroup independent problems (a grouped GEMM:
// e.g. a block's QKV projection and its cross-attention K and V projections,
// each with its own operands, shape and output); their tiles form one tile
// space that the persistent CTAs walk, each tile finding its problem from the
// problems' first-tile indices.  A plain call is a group of one.
//
// Kernel shape (one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: code tiles (tensor maps, 128-byte swizzle) and
//               scale atoms (bulk copies) into a STAGES-deep shared ring.
//   warp 1      TMEM owner and MMA issuer: per K=64 step, tcgen05.cp moves
//               the step's scale atoms into TMEM, then one tcgen05.mma.
//   (both run the loop on the whole warp; one elected lane issues)
//   warps 2..5  epilogue: tcgen05.ld of the accumulator, alpha, conversion,
//               TMA stores (bf16 / FP32) or direct stores (NVFP4).
// Tile: 128 (M) x BN (N) x 256 (K per stage).  TMEM: 512 columns, the
// accumulator(s) in [0, 256) (two buffers when BN = 128 so the epilogue of
// one tile overlaps the mainloop of the next), the scale ring in [256, 512).
#include <cstring>

#include <cstdlib>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "internal.h"
#include "gemm.h"
#include "ptx.cuh"
#include "quant_math.cuh"
#include "epilogue.cuh"
#include "tmap.h"

namespace nvfp4 {

namespace w4a4 {

constexpr int BM = 128;
constexpr int BK_BYTES = 128;                    // 256 FP4 values per row per stage
constexpr int A_BYTES = BM * BK_BYTES;           // 16 KB
constexpr int SF_ATOM = 512;                     // 128 rows x 4 blocks
constexpr int kThreads = 192;
constexpr int kEpiWarps = 4;
constexpr int kGroupM = 16;                      // rasterisation group (M blocks)

enum OutKind { OUT_BF16 = 0, OUT_F32 = 1, OUT_NVFP4 = 2 };

// MXS: the MX operand format (blocks of 32 with E8M0 scales, kind::mxf4,
// two scale atoms per 256-K stage, one per two K = 64 steps); otherwise
// NVFP4 (blocks of 16 with E4M3 scales, four atoms per stage).
template <int BN, int STAGES, bool MXS = false>
struct Cfg {
    static constexpr int SF_ATOMS = MXS ? 2 : 4;              // scale atoms per 128 rows per stage
    static constexpr int SFA_BYTES = SF_ATOMS * SF_ATOM;
    static constexpr int B_BYTES = BN * BK_BYTES;
    static constexpr int SFB_BYTES = (BN / 128) * SFA_BYTES;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr int ACC_BUFS = (BN == 128) ? 2 : 1;
    static constexpr int SF_COLS_STEP = 4 + BN / 32;          // per atom group: SFA 4 columns + SFB BN/32
    static constexpr int SF_COLS_STAGE = SF_ATOMS * SF_COLS_STEP;
    static constexpr int EPI_BUF_BYTES = 32 * 128;            // 32 rows x 128 B (f32 worst case)
    static constexpr int EPI_BYTES = kEpiWarps * 2 * EPI_BUF_BYTES;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024;
    static_assert(ACC_BUFS * BN <= 256, "accumulators must fit TMEM columns [0,256)");
    static_assert(STAGES * SF_COLS_STAGE <= 256, "scale ring must fit TMEM columns [256,512)");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

constexpr int kMaxGroup = 8;

struct Problem {
    const uint8_t* a_sf;
    const uint8_t* b_sf;
    const float* a_scale;
    const float* b_scale;
    uint8_t* y_codes;
    uint8_t* y_sf;
    const float* y_scale;
    float* y_amax;
    int M, N, K;
    int num_mb, num_nb, tile0;                   // tiles [tile0, tile0 + num_mb * num_nb)
};

struct Params {
    Problem pr[kMaxGroup];
    int count, num_tiles;
    int* dev_status;
};

// Tensor maps of every problem: A codes, B codes, Y (bf16 / FP32 output).
struct Maps {
    CUtensorMap a[kMaxGroup], b[kMaxGroup], y[kMaxGroup];
};
static_assert(sizeof(Maps) + sizeof(Params) <= 4096, "kernel parameters");

// Problem of global tile t (problems are in tile order).
__device__ __forceinline__ int find_problem(const Params& p, int t) {
    int g = 0;
#pragma unroll 1
    for (int i = 1; i < p.count; ++i)
        if (t >= p.pr[i].tile0) g = i;
    return g;
}

__device__ __forceinline__ void tile_coords(int t, int num_mb, int num_nb, int& mb, int& nb) {
    const int per_group = kGroupM * num_nb;
    const int group = t / per_group;
    const int first_mb = group * kGroupM;
    const int gm = min(kGroupM, num_mb - first_mb);
    const int idx = t - group * per_group;
    mb = first_mb + idx % gm;
    nb = idx / gm;
}

// Warp-wide maximum of a non-negative running |y| maximum, merged into the
// caller's device float (atomic max on the bit pattern: order-preserving for
// non-negative floats).  Whole warp; a null destination is skipped.
__device__ __forceinline__ void flush_amax(float v, float* dst, int lane) {
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (dst != nullptr && lane == 0 && v > 0.0f) atomicMax(reinterpret_cast<int*>(dst), __float_as_int(v));
}

template <int BN, int STAGES, int OUT, int ACT, bool MXS>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ Maps maps, const __grid_constant__ Params p) {
    using C = Cfg<BN, STAGES, MXS>;
    constexpr int kAtomK = MXS ? 128 : 64;        // K covered by one 128-row scale atom
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[STAGES], empty_bar[STAGES];
    __shared__ __align__(8) uint64_t accf_bar[C::ACC_BUFS], acce_bar[C::ACC_BUFS];
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    WaitCtx wc{&abort_sh, p.dev_status};

    if (threadIdx.x == 0) {
        abort_sh = 0;
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < C::ACC_BUFS; ++b) {
            mbar_init(&accf_bar[b], 1);
            mbar_init(&acce_bar[b], kEpiWarps);
        }
        mbar_init(&drain_bar, 1);
        fence_barrier_init();
        for (int g = 0; g < p.count; ++g) {
            tma_prefetch_desc(&maps.a[g]);
            tma_prefetch_desc(&maps.b[g]);
            if (OUT != OUT_NVFP4) tma_prefetch_desc(&maps.y[g]);
        }
    }
    // Scale bytes of absent 128-row blocks are never loaded; zero every scale
    // region once so such rows read finite scales (their codes are zero).
    for (int s = 0; s < STAGES; ++s) {
        uint32_t* z = reinterpret_cast<uint32_t*>(smem + s * C::STAGE_BYTES + A_BYTES + C::B_BYTES);
        for (int i = threadIdx.x; i < (C::SFA_BYTES + C::SFB_BYTES) / 4; i += kThreads) z[i] = 0u;
    }
    fence_proxy_async_smem();
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;


    // Producer and MMA issuer run on whole warps with one elected lane issuing,
    // so descriptors, coordinates and addresses stay warp-uniform (from a
    // single lane each tcgen05 or TMA instruction costs tens of cycles to issue).
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        const uint64_t pol_a = policy_evict_normal();
        const uint64_t pol_b = policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        uint32_t issued = 0;                     // bit s: parity of the last load into stage s
        uint32_t issued_any = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
            const int g = find_problem(p, t);
            const Problem& pr = p.pr[g];
            int mb, nb;
            tile_coords(t - pr.tile0, pr.num_mb, pr.num_nb, mb, nb);
            const int nblk0 = nb * (BN / 128);
            const int nblk_total = (pr.N + 127) / 128;
            const int num_kt = (pr.K + 255) / 256;
            const int k_atoms = pr.K / kAtomK;    // scale atoms per 128-row block
            for (int kt = 0; kt < num_kt; ++kt) {
                if (!__all_sync(0xffffffffu, mbar_wait(&empty_bar[stage], phase ^ 1u, wc) ? 1 : 0)) {
                    ok = false;
                    break;
                }
                uint8_t* sbase = smem + stage * C::STAGE_BYTES;
                const int natoms = min(C::SF_ATOMS, k_atoms - kt * C::SF_ATOMS);
                int nsfb = 0;
                for (int j = 0; j < BN / 128; ++j) nsfb += (nblk0 + j < nblk_total) ? 1 : 0;
                if (elect_one()) {
                    const uint32_t bytes = A_BYTES + C::B_BYTES + natoms * SF_ATOM * (1 + nsfb);
                    mbar_arrive_expect_tx(&full_bar[stage], bytes);
                    tma_load_2d(sbase, &maps.a[g], &full_bar[stage], kt * BK_BYTES, mb * BM, pol_a);
                    tma_load_2d(sbase + A_BYTES, &maps.b[g], &full_bar[stage], kt * BK_BYTES, nb * BN, pol_b);
                    bulk_load(sbase + A_BYTES + C::B_BYTES,
                              pr.a_sf + ((int64_t)mb * k_atoms + kt * C::SF_ATOMS) * SF_ATOM, natoms * SF_ATOM,
                              &full_bar[stage], pol_a);
                    for (int j = 0; j < nsfb; ++j)
                        bulk_load(sbase + A_BYTES + C::B_BYTES + C::SFA_BYTES + j * C::SFA_BYTES,
                                  pr.b_sf + ((int64_t)(nblk0 + j) * k_atoms + kt * C::SF_ATOMS) * SF_ATOM,
                                  natoms * SF_ATOM, &full_bar[stage], pol_b);
                }
                __syncwarp();
                issued = (issued & ~(1u << stage)) | (phase << stage);
                issued_any |= 1u << stage;
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
        }
        // every load this warp issued has landed before the CTA may exit
        if (lane == 0) {
            for (int s = 0; s < STAGES; ++s)
                if (issued_any & (1u << s)) {
                    WaitCtx w2{&abort_sh, p.dev_status};
                    int dummy_abort = 0;
                    w2.abort_flag = &dummy_abort;        // wait for own copies even when aborting
                    mbar_wait(&full_bar[s], (issued >> s) & 1u, w2);
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = MXS ? idesc_mxf4(BM, BN) : idesc_nvf4(BM, BN);
        const uint32_t smem0 = smem_u32(smem);
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        const uint32_t sf_base = tmem_base + 256;
        for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
            if (!__all_sync(0xffffffffu, mbar_wait(&acce_bar[acc], acc_phase ^ 1u, wc) ? 1 : 0)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const Problem& pr = p.pr[find_problem(p, t)];
            const int num_kt = (pr.K + 255) / 256;
            const int k_steps = pr.K / 64;       // K = 64 MMA steps
            const uint32_t d_tmem = tmem_base + acc * BN;
            for (int kt = 0; kt < num_kt; ++kt) {
                if (!__all_sync(0xffffffffu, mbar_wait(&full_bar[stage], phase, wc) ? 1 : 0)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sbase = smem0 + stage * C::STAGE_BYTES;
                const uint32_t sfa_s = sbase + A_BYTES + C::B_BYTES;
                const uint32_t sfb_s = sfa_s + C::SFA_BYTES;
                const uint32_t sf_col = sf_base + stage * C::SF_COLS_STAGE;
                const int nks = min(4, k_steps - kt * 4);
                if (elect_one()) {
                    for (int ks = 0; ks < nks; ++ks) {
                        // NVFP4: one atom per K = 64 step; MX: one per two steps,
                        // the step's two scale bytes selected by a byte id (0 or 2)
                        const int at = MXS ? (ks >> 1) : ks;
                        const uint32_t col = sf_col + at * C::SF_COLS_STEP;
                        if (!MXS || (ks & 1) == 0) {
                            tc_cp_32x128b_warpx4(col, sdesc_sf(sfa_s + at * SF_ATOM));
#pragma unroll
                            for (int j = 0; j < BN / 128; ++j)
                                tc_cp_32x128b_warpx4(col + 4 + 4 * j,
                                                     sdesc_sf(sfb_s + j * C::SFA_BYTES + at * SF_ATOM));
                        }
                        if (MXS) {
                            const uint32_t byte = (uint32_t)(ks & 1) * 2u;
                            tc_mma_mxf4(d_tmem, sdesc_kmajor_sw128(sbase + ks * 32),
                                        sdesc_kmajor_sw128(sbase + A_BYTES + ks * 32),
                                        idesc | (byte << 29) | (byte << 4), col | (byte << 30),
                                        (col + 4) | (byte << 30), (kt | ks) != 0 ? 1u : 0u);
                        } else {
                            tc_mma_nvf4(d_tmem, sdesc_kmajor_sw128(sbase + ks * 32),
                                        sdesc_kmajor_sw128(sbase + A_BYTES + ks * 32), idesc, col, col + 4,
                                        (kt | ks) != 0 ? 1u : 0u);
                        }
                    }
                    tc_commit(&empty_bar[stage]);
                }
                __syncwarp();
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
            if (elect_one()) tc_commit(&accf_bar[acc]);
            __syncwarp();
            if (++acc == C::ACC_BUFS) { acc = 0; acc_phase ^= 1u; }
        }
        // all MMAs issued by this warp complete before TMEM is released
        if (elect_one()) tc_commit(&drain_bar);
        __syncwarp();
        WaitCtx w2{&abort_sh, p.dev_status};
        int dummy_abort = 0;
        w2.abort_flag = &dummy_abort;
        mbar_wait(&drain_bar, 0, w2);
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                       // TMEM lane quarter
        const int row_t = q * 32 + lane;              // row inside the tile
        uint8_t* ebuf = smem + STAGES * C::STAGE_BYTES + (warp - 2) * 2 * C::EPI_BUF_BYTES;
        int acc = 0;
        uint32_t acc_phase = 0;
        int nstore = 0;
        int g_prev = -1;
        float alpha = 0.0f, g_y = 0.0f, amax_run = 0.0f;
        ScaleConsts sc_y = scale_consts(0.0f);
        for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
            const int g = find_problem(p, t);
            const Problem& pr = p.pr[g];
            if (g != g_prev) {
                // a new problem: flush the previous one's running amax, load this one's scales
                if (OUT == OUT_NVFP4 && g_prev >= 0) flush_amax(amax_run, p.pr[g_prev].y_amax, lane);
                amax_run = 0.0f;
                // MX operands have no tensor scale: a null scale reads as 1
                alpha = __fmul_rn(pr.a_scale ? *pr.a_scale : 1.0f, pr.b_scale ? *pr.b_scale : 1.0f);
                if (OUT == OUT_NVFP4) {
                    g_y = *pr.y_scale;
                    sc_y = scale_consts(g_y);
                }
                g_prev = g;
            }
            int mb, nb;
            tile_coords(t - pr.tile0, pr.num_mb, pr.num_nb, mb, nb);
            // warp-uniform decision: the TMEM loads below are .sync.aligned
            if (!__all_sync(0xffffffffu, mbar_wait(&accf_bar[acc], acc_phase, wc) ? 1 : 0)) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
            const int m0 = mb * BM, n0 = nb * BN;
            if (OUT == OUT_NVFP4) {
                const int64_t grow = (int64_t)m0 + row_t;
                const int kb4 = pr.N / 64;
                for (int c = 0; c < BN / 64; ++c) {
                    const int ncol = n0 + c * 64;
                    uint32_t r0[32], r1[32];
                    tmem_ld_32x32b_x32(tbase + c * 64, r0);
                    tmem_ld_32x32b_x32(tbase + c * 64 + 32, r1);
                    tmem_ld_wait();
                    if (ncol >= pr.N) continue;
                    uint32_t sfw = 0u;
                    uint32_t cw[8];
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        float v[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const uint32_t bits = (b < 2) ? r0[b * 16 + j] : r1[(b - 2) * 16 + j];
                            v[j] = epi_value<ACT>(alpha, bits);
                        }
                        float ab = 0.0f;
#pragma unroll
                        for (int j = 0; j < 16; ++j) ab = fmaxf(ab, fabsf(v[j]));
                        if (grow < pr.M) amax_run = fmaxf(amax_run, ab);
                        const uint32_t sfc = block_scale_code(ab, sc_y);
                        const float s = __fmul_rn(e4m3_to_f32(sfc), g_y);
                        float lo[8], hi[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) { lo[j] = v[j]; hi[j] = v[8 + j]; }
                        cw[2 * b] = quantize8(lo, s);
                        cw[2 * b + 1] = quantize8(hi, s);
                        sfw |= sfc << (8 * b);
                    }
                    if (grow < pr.M) {
                        uint4* dst = reinterpret_cast<uint4*>(pr.y_codes + grow * (pr.N / 2) + ncol / 2);
                        dst[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
                        dst[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
                    }
                    const int64_t atom = (int64_t)mb * kb4 + ncol / 64;
                    *reinterpret_cast<uint32_t*>(pr.y_sf + atom * SF_ATOM + (row_t & 31) * 16 + (row_t >> 5) * 4) = sfw;
                }
            } else {
                for (int c = 0; c < BN / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, r);
                    tmem_ld_wait();
                    if (n0 + c * 32 >= pr.N) continue;
                    uint8_t* buf = ebuf + (nstore & 1) * C::EPI_BUF_BYTES;
                    // the store that last used this buffer has finished reading it
                    if (lane == 0) bulk_wait_group_read<1>();
                    __syncwarp();
                    if (OUT == OUT_BF16) {
                        uint32_t pk[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            __nv_bfloat162 h = __floats2bfloat162_rn(epi_value<ACT>(alpha, r[2 * j]),
                                                                     epi_value<ACT>(alpha, r[2 * j + 1]));
                            pk[j] = *reinterpret_cast<uint32_t*>(&h);
                        }
                        // 64-byte rows, 64-byte swizzle: chunk j of row i at j ^ ((i >> 1) & 3)
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int pos = j ^ ((lane >> 1) & 3);
                            *reinterpret_cast<uint4*>(buf + lane * 64 + pos * 16) =
                                make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                        }
                    } else {
                        // 128-byte rows, 128-byte swizzle: chunk j of row i at j ^ (i & 7)
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int pos = j ^ (lane & 7);
                            float4 o = make_float4(epi_value<ACT>(alpha, r[4 * j]), epi_value<ACT>(alpha, r[4 * j + 1]),
                                                   epi_value<ACT>(alpha, r[4 * j + 2]), epi_value<ACT>(alpha, r[4 * j + 3]));
                            *reinterpret_cast<float4*>(buf + lane * 128 + pos * 16) = o;
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&maps.y[g], buf, n0 + c * 32, m0 + q * 32);
                        bulk_commit_group();
                    }
                    ++nstore;
                }
            }
            // accumulator drained: hand it back to the MMA warp
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce_bar[acc]);
            if (++acc == C::ACC_BUFS) { acc = 0; acc_phase ^= 1u; }
        }
        if (lane == 0) bulk_wait_group<0>();
        if (OUT == OUT_NVFP4 && g_prev >= 0) flush_amax(amax_run, p.pr[g_prev].y_amax, lane);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

template <int BN, int STAGES, int OUT, int ACT, bool MXS>
cudaError_t launch_cfg(const GemmW4A4Args* probs, int count, int num_sms, cudaStream_t stream) {
    using C = Cfg<BN, STAGES, MXS>;
    if (count < 1 || count > kMaxGroup) return cudaErrorInvalidValue;
    Maps maps;
    Params p;
    memset(&maps, 0, sizeof(maps));
    memset(&p, 0, sizeof(p));
    int tiles = 0;
    for (int g = 0; g < count; ++g) {
        const GemmW4A4Args& a = probs[g];
        CUresult r;
        r = make_tmap_2d(&maps.a[g], a.a_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)(a.K / 2),
                         (uint64_t)(a.M > 0 ? a.M : 1), (uint64_t)(a.K / 2), BK_BYTES, BM, CU_TENSOR_MAP_SWIZZLE_128B);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
        r = make_tmap_2d(&maps.b[g], a.b_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)(a.K / 2), (uint64_t)a.N,
                         (uint64_t)(a.K / 2), BK_BYTES, BN, CU_TENSOR_MAP_SWIZZLE_128B);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
        if (OUT == OUT_BF16) {
            r = make_tmap_2d(&maps.y[g], a.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.N,
                             (uint64_t)(a.M > 0 ? a.M : 1), (uint64_t)a.N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
        } else if (OUT == OUT_F32) {
            r = make_tmap_2d(&maps.y[g], a.y, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)a.N,
                             (uint64_t)(a.M > 0 ? a.M : 1), (uint64_t)a.N * 4, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B);
        }
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
        Problem& pr = p.pr[g];
        pr.a_sf = a.a_sf;
        pr.b_sf = a.b_sf;
        pr.a_scale = a.a_scale;
        pr.b_scale = a.b_scale;
        pr.y_codes = a.y_codes;
        pr.y_sf = a.y_sf;
        pr.y_scale = a.y_scale;
        pr.y_amax = a.y_amax;
        pr.M = (int)a.M;
        pr.N = (int)a.N;
        pr.K = (int)a.K;
        pr.num_mb = (int)((a.M + BM - 1) / BM);
        pr.num_nb = (int)((a.N + BN - 1) / BN);
        pr.tile0 = tiles;
        tiles += pr.num_mb * pr.num_nb;          // M == 0: no tiles
    }
    p.count = count;
    p.num_tiles = tiles;
    p.dev_status = probs[0].dev_status;
    if (tiles == 0) return cudaSuccess;

    auto kern = gemm_kernel<BN, STAGES, OUT, ACT, MXS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int grid = tiles < num_sms ? tiles : num_sms;
    kern<<<grid, kThreads, C::SMEM_BYTES, stream>>>(maps, p);
    count_launch(1);
    return cudaGetLastError();
}

template <int OUT>
static cudaError_t launch_group(const GemmW4A4Args* probs, int count, int num_sms, cudaStream_t stream) {
    const bool gelu = probs[0].act == ACT_GELU_TANH;
    if (probs[0].mx)
        return gelu ? launch_cfg<128, 5, OUT, ACT_GELU_TANH, true>(probs, count, num_sms, stream)
                    : launch_cfg<128, 5, OUT, ACT_NONE, true>(probs, count, num_sms, stream);
    return gelu ? launch_cfg<128, 5, OUT, ACT_GELU_TANH, false>(probs, count, num_sms, stream)
                : launch_cfg<128, 5, OUT, ACT_NONE, false>(probs, count, num_sms, stream);
}

}  // namespace w4a4

cudaError_t launch_gemm_w4a4(const GemmW4A4Args& a, int num_sms, cudaStream_t stream) {
    using namespace w4a4;
    if (a.M == 0) return cudaSuccess;
    // N a multiple of 192 or 256: CTA-pair kernel (256 x 192 or 256 x 256
    // tiles) when there are enough pair tiles to fill the GPU; otherwise
    // single-CTA 128 x 128 tiles with a double-buffered accumulator, whose
    // finer tiles waste less of a small problem.  NVFP4_GEMM_KERNEL=pair or
    // =single overrides the choice (where the shape allows) for measurements.
    const char* env = getenv("NVFP4_GEMM_KERNEL");
    const int forced = env ? (env[0] == 'p' ? 1 : env[0] == 's' ? 2 : 0) : 0;
    if (gemm_w4a4_2sm_supports(a.N) && forced != 2) {
        const int64_t bn = a.N % 256 == 0 ? 256 : 192;
        const int64_t pair_tiles = ((a.M + 255) / 256) * (a.N / bn);
        if (forced == 1 || pair_tiles >= num_sms / 2) return launch_gemm_w4a4_2sm(a, num_sms, stream);
    }
    return launch_group_single(&a, 1, num_sms, stream);
}

// Up to kMaxGroup problems in one launch; every problem has the same output
// kind (bf16, FP32 or NVFP4) and activation.  When every N allows one pair
// tile width and the problems' pair tiles fill the GPU, the CTA-pair kernel
// takes the whole group (one tile space); otherwise the single-CTA kernel.
// NVFP4_GEMM_KERNEL=pair or =single overrides the choice (where the shapes
// allow) for measurements.
cudaError_t launch_gemm_w4a4_grouped(const GemmW4A4Args* probs, int count, int num_sms, cudaStream_t stream) {
    using namespace w4a4;
    const char* env = getenv("NVFP4_GEMM_KERNEL");
    const int forced = env ? (env[0] == 'p' ? 1 : env[0] == 's' ? 2 : 0) : 0;
    const int bn = count > 1 && forced != 2 && !probs[0].mx ? gemm_w4a4_2sm_tile_n(probs, count) : 0;
    if (bn != 0) {
        int64_t tiles = 0;
        for (int i = 0; i < count; ++i) tiles += ((probs[i].M + 255) / 256) * (probs[i].N / bn);
        if (forced == 1 || tiles >= num_sms / 2) return launch_gemm_w4a4_2sm_grouped(probs, count, num_sms, stream);
    }
    return launch_group_single(probs, count, num_sms, stream);
}

// The single-CTA kernel on a group (a plain call is a group of one).
cudaError_t launch_group_single(const GemmW4A4Args* probs, int count, int num_sms, cudaStream_t stream) {
    using namespace w4a4;
    const int out = probs[0].y != nullptr ? (probs[0].y_dtype == 1 ? OUT_F32 : OUT_BF16) : OUT_NVFP4;
    if (out == OUT_BF16) return launch_group<OUT_BF16>(probs, count, num_sms, stream);
    if (out == OUT_F32) return launch_group<OUT_F32>(probs, count, num_sms, stream);
    return launch_group<OUT_NVFP4>(probs, count, num_sms, stream);
}

int gemm_w4a4_max_group() { return w4a4::kMaxGroup; }

}  // namespace nvfp4
