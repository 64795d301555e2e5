// attn.cu -- attention over an NVFP4 key / value cache ("NVFP4-DiT ..."
// README, Algorithmic framework, Eq. 10: Attention(Q, K, V) =
// softmax(Q K^T / sqrt(d_k) + log(s_head)) V with a per-head scale s_head;
// Systems optimization: FP4-packed attention).
//
// Q, K, V are NVFP4 tensors quantized along the head dimension d = 128
// (blocks of 16, tensor scales g_q, g_k, g_v): Q [H*Lq, d], K and V [H*Lk, d].
// Two kernels:
//   v_decode      V decoded exactly to bf16 (e2m1 * e4m3: at most 6
//                 significant bits), [H*Lk, d] in the caller's workspace --
//                 once per call, instead of once per query tile;
//   attention     persistent, one CTA per SM; a work item is 128 (or 256)
//                 queries of one head, keys in tiles of 128:
//     S = Q K^T   block-scaled FP4 MMA (kind::mxf4nvf4, K = d), FP32 in TMEM,
//                 two S buffers so the next tile's product overlaps softmax;
//     softmax     one query row per thread (online: reference maximum m, sum
//                 l), exp2 of (S * g_q g_k log2(e) / sqrt(d) + log2(s_head) - m),
//                 P rounded to bf16 into a 128-byte-swizzled K-major tile; the
//                 running output is rescaled in TMEM when m moves;
//     O += P V    bf16 MMA (kind::f16) on TMA-loaded V tiles (B operand
//                 MN-major: d contiguous), FP32 in TMEM;
//     output      O * g_v / l, rounded to bf16.
// Roles: warp 0 loads Q and the K ring, warp 3 the V ring; warp 1 owns TMEM
// and issues S = Q K^T, warp 2 issues O += P V (two issuers, so that neither
// product waits behind the other's operands); warps 4-7 softmax and output;
// every wait is bounded.
#include <cstdlib>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"
#include "quant_math.cuh"
#include "tmap.h"

namespace nvfp4 {

namespace attn {

constexpr int kD = 128;                      // head dimension
constexpr int kBQ = 128;                     // queries per CTA
constexpr int kBK = 128;                     // keys per tile
constexpr int kThreads = 256;
constexpr int kKStages = 4;                  // K code + scale stages
constexpr int kVStages = 3;                  // V stages
constexpr int kCodeBytes = kBK * kD / 2;     // 8 KB: 128 rows x 64 bytes
constexpr int kSfBytes = 1024;               // two 512-byte scale atoms (128 rows x 8 blocks)
constexpr int kKStageBytes = kCodeBytes + kSfBytes;
constexpr int kTileBf16 = kBQ * kBK * 2;     // 32 KB: two 64-column chunks of 128 rows x 128 bytes
constexpr int kChunk = 128 * 128;            // 16 KB

// shared memory (offsets from a 1024-aligned base): two Q buffers (codes with
// the 64-byte swizzle, scales), so that the next work item's Q lands while
// this one runs; the K ring (codes with the 64-byte swizzle, scales); the V
// ring (bf16 rows of keys, d 0-63 then d 64-127, 128-byte swizzle); two P
// tiles (bf16, 128-byte swizzle)
constexpr int kOffQ = 0;                     // + qb * kKStageBytes
constexpr int kOffK = 2 * kKStageBytes;
constexpr int kOffV = kOffK + kKStages * kKStageBytes;
constexpr int kOffP = kOffV + kVStages * kTileBf16;
constexpr int kSmemBytes = kOffP + 2 * kTileBf16 + 1024;
static_assert(kOffK % 1024 == 0 && kKStageBytes % 1024 == 0 && kOffV % 1024 == 0 && kOffP % 1024 == 0,
              "swizzled tiles are 1024-byte aligned");
static_assert(kSmemBytes <= 232448, "shared memory budget");

// TMEM columns
constexpr uint32_t kColS = 0;                // two S buffers: [0,128), [128,256)
constexpr uint32_t kColO = 256;              // O: [256, 384)
constexpr uint32_t kColSfQ = 384;            // Q scales per Q buffer: 2 x (2 K-steps x 4 columns)
constexpr uint32_t kColSfK = 400;            // K scales per S buffer: 2 x (2 x 4)

struct Params {
    const uint8_t* q_sf;
    const uint8_t* k_sf;
    const float* g_q;
    const float* g_k;
    const float* g_v;
    const float* s_head;                     // nullable: 1 for every head
    uint16_t* out;                           // bf16 [H*Lq, d]
    int Lq, Lk, H;
    int* dev_status;
};

// K-major operand rows of 64 bytes with the 64-byte swizzle (8-row groups
// 512 bytes apart).
__device__ __forceinline__ uint64_t sdesc_kmajor_sw64(uint32_t saddr) { return make_sdesc(saddr, 16, 512, 4); }

__device__ __forceinline__ void tmem_st_x32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
          "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
          "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Two E2M1 codes (one byte, low nibble first) times their shared scale,
// exactly, as a bf16 pair: the f16 decode shifted down three bits is the bf16
// pattern of the value times 2^-112 (sign kept), and one bf16 multiply by the
// scale times 2^112 gives the product (at most 6 significant bits).
__device__ __forceinline__ uint32_t dequant_pair_attn(uint32_t byte, uint32_t scale_b2) {
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

// E4M3 byte -> bf16 of (scale * 2^112) in both halves (exact).
__device__ __forceinline__ uint32_t e4m3_to_b2_scaled_attn(uint32_t code) {
    const float f = e4m3_to_f32(code) * 0x1p112f;
    const uint32_t b = __float_as_uint(f) >> 16;
    return b | (b << 16);
}

// The V tile as the B operand of O += P V (K = keys, N = d), MN-major: rows
// of 128 bytes hold 64 values of d for one key, 128-byte swizzle; 8-key
// groups are 1024 bytes apart (stride offset) and the two 64-column chunks
// 16 KB apart (leading offset).
__device__ __forceinline__ uint64_t sdesc_v(uint32_t saddr) { return make_sdesc(saddr, kChunk, 1024, 2); }

// Start-address steps (descriptor units of 16 bytes) of the kk-th 16-key MMA
// of a tile: in V, 16 rows of 128 bytes; in the K-major P tile, 32 bytes
// within a 64-key chunk, chunks 16 KB apart.  Tiles lie below 256 KB, so the
// 14-bit address field does not carry.
__device__ __forceinline__ uint64_t v_step(int kk) { return (uint64_t)(kk * 2048 >> 4); }
__device__ __forceinline__ uint64_t p_step(int kk) { return (uint64_t)(((kk >> 2) * kChunk + (kk & 3) * 32) >> 4); }

// kind::f16 instruction descriptor with B MN-major (bit 16).
__host__ __device__ constexpr uint32_t idesc_bf16_bmn(int M, int N) { return idesc_bf16(M, N) | (1u << 16); }

// Persistent: CTA c takes work items (head, 128-query tile) c, c + grid, ...
// Key tiles carry one running number n over all of a CTA's items, which
// selects ring slots, S / P buffers and barrier phases, so every pipeline
// stays full across item boundaries: the next item's Q, K and S go ahead
// while this item's last products and output finish.
__global__ void __launch_bounds__(kThreads, 1)
attn_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
            const __grid_constant__ CUtensorMap tmap_v, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t q_full[2], q_empty[2], k_full[kKStages], k_empty[kKStages];
    __shared__ __align__(8) uint64_t v_full[kVStages], v_empty[kVStages];
    __shared__ __align__(8) uint64_t s_full[2], s_empty[2], p_full[2], p_empty[2], o_done, o_free, drain_s, drain_o;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    WaitCtx wc{&abort_sh, p.dev_status};
    const int ntiles = p.Lk / kBK;
    const int qtiles = p.Lq / kBQ;
    const int nitems = p.H * qtiles;
    // item -> head and first query row
    auto item_head = [&](int it) { return it / qtiles; };
    auto item_qrow = [&](int it) { return (it / qtiles) * p.Lq + (it % qtiles) * kBQ; };

    if (threadIdx.x == 0) {
        abort_sh = 0;
        for (int b = 0; b < 2; ++b) {
            mbar_init(&q_full[b], 1);
            mbar_init(&q_empty[b], 1);               // the item's last S product's commit
        }
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);               // the S product's commit
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);               // the PV product's commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_empty[b], 4);
            mbar_init(&p_full[b], 4);
            mbar_init(&p_empty[b], 1);
        }
        mbar_init(&o_done, 1);
        mbar_init(&o_free, 4);                       // the softmax warps have read O out
        mbar_init(&drain_s, 1);
        mbar_init(&drain_o, 1);
        fence_barrier_init();
        tma_prefetch_desc(&tmap_q);
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp < 4) {
    if (warp == 0) {
        // ------------------------------------------------------------ Q and K producer
        const uint64_t pol = policy_evict_normal();
        bool ok = true;
        int n = 0, i = 0;
        for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++i) {
            const int qb = i & 1, qrow0 = item_qrow(it), krow0 = item_head(it) * p.Lk;
            if (!__all_sync(0xffffffffu, mbar_wait(&q_empty[qb], ((uint32_t)(i >> 1) & 1u) ^ 1u, wc) ? 1 : 0)) {
                ok = false;
                break;
            }
            if (elect_one()) {
                uint8_t* qs = smem + kOffQ + qb * kKStageBytes;
                mbar_arrive_expect_tx(&q_full[qb], kKStageBytes);
                tma_load_2d(qs, &tmap_q, &q_full[qb], 0, qrow0, pol);
                bulk_load(qs + kCodeBytes, p.q_sf + (int64_t)(qrow0 >> 7) * kSfBytes, kSfBytes, &q_full[qb], pol);
            }
            __syncwarp();
            for (int j = 0; j < ntiles; ++j, ++n) {
                const int s = n % kKStages;
                const uint32_t ph = (uint32_t)(n / kKStages) & 1u;
                if (!__all_sync(0xffffffffu, mbar_wait(&k_empty[s], ph ^ 1u, wc) ? 1 : 0)) { ok = false; break; }
                uint8_t* st = smem + kOffK + s * kKStageBytes;
                const int kr = krow0 + j * kBK;
                if (elect_one()) {
                    mbar_arrive_expect_tx(&k_full[s], kKStageBytes);
                    tma_load_2d(st, &tmap_k, &k_full[s], 0, kr, pol);
                    bulk_load(st + kCodeBytes, p.k_sf + (int64_t)(kr >> 7) * kSfBytes, kSfBytes, &k_full[s], pol);
                }
                __syncwarp();
            }
        }
        // every load this warp issued has landed before the CTA may exit
        if (lane == 0) {
            int dummy = 0;
            WaitCtx w2{&dummy, p.dev_status};
            for (int q = (i > 2 ? i - 2 : 0); q < i; ++q) mbar_wait(&q_full[q & 1], (uint32_t)(q >> 1) & 1u, w2);
            for (int m = (n > kKStages ? n - kKStages : 0); m < n; ++m)
                mbar_wait(&k_full[m % kKStages], (uint32_t)(m / kKStages) & 1u, w2);
        }
    } else if (warp == 3) {
        // ------------------------------------------------------------ V producer
        const uint64_t pol = policy_evict_normal();
        bool ok = true;
        int n = 0;
        for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
            const int h = item_head(it);
            for (int j = 0; j < ntiles; ++j, ++n) {
                const int s = n % kVStages;
                const uint32_t ph = (uint32_t)(n / kVStages) & 1u;
                if (!__all_sync(0xffffffffu, mbar_wait(&v_empty[s], ph ^ 1u, wc) ? 1 : 0)) { ok = false; break; }
                uint8_t* st = smem + kOffV + s * kTileBf16;
                if (elect_one()) {
                    // keys h*Lk + j*128 .. + 127 of V, as two 64-column chunks
                    mbar_arrive_expect_tx(&v_full[s], kTileBf16);
                    tma_load_2d(st, &tmap_v, &v_full[s], 0, h * p.Lk + j * kBK, pol);
                    tma_load_2d(st + kChunk, &tmap_v, &v_full[s], 64, h * p.Lk + j * kBK, pol);
                }
                __syncwarp();
            }
        }
        if (lane == 0) {
            int dummy = 0;
            WaitCtx w2{&dummy, p.dev_status};
            for (int m = (n > kVStages ? n - kVStages : 0); m < n; ++m)
                mbar_wait(&v_full[m % kVStages], (uint32_t)(m / kVStages) & 1u, w2);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ S = Q K^T issuer (and TMEM owner)
        constexpr uint32_t idesc_s = idesc_nvf4(kBQ, kBK);
        const uint32_t sm0 = smem_u32(smem);
        bool ok = true;
        int n = 0, i = 0;
        for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++i) {
            const int qb = i & 1;
            const uint32_t qs = sm0 + kOffQ + qb * kKStageBytes, sfq = tmem + kColSfQ + qb * 8;
            if (!__all_sync(0xffffffffu, mbar_wait(&q_full[qb], (uint32_t)(i >> 1) & 1u, wc) ? 1 : 0)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (elect_one()) {
                tc_cp_32x128b_warpx4(sfq, sdesc_sf(qs + kCodeBytes));
                tc_cp_32x128b_warpx4(sfq + 4, sdesc_sf(qs + kCodeBytes + 512));
            }
            __syncwarp();
            for (int j = 0; j < ntiles; ++j, ++n) {
                const int s = n % kKStages, b = n & 1;
                if (!__all_sync(0xffffffffu, mbar_wait(&k_full[s], (uint32_t)(n / kKStages) & 1u, wc) ? 1 : 0) ||
                    !__all_sync(0xffffffffu, mbar_wait(&s_empty[b], ((uint32_t)(n >> 1) & 1u) ^ 1u, wc) ? 1 : 0)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t st = sm0 + kOffK + s * kKStageBytes;
                const uint32_t sfk = tmem + kColSfK + b * 8;
                if (elect_one()) {
                    tc_cp_32x128b_warpx4(sfk, sdesc_sf(st + kCodeBytes));
                    tc_cp_32x128b_warpx4(sfk + 4, sdesc_sf(st + kCodeBytes + 512));
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks)
                        tc_mma_nvf4(tmem + kColS + b * kBK, sdesc_kmajor_sw64(qs + ks * 32),
                                    sdesc_kmajor_sw64(st + ks * 32), idesc_s, sfq + ks * 4, sfk + ks * 4,
                                    ks != 0 ? 1u : 0u);
                    tc_commit(&s_full[b]);
                    tc_commit(&k_empty[s]);
                    if (j == ntiles - 1) tc_commit(&q_empty[qb]);
                }
                __syncwarp();
            }
        }
        if (elect_one()) tc_commit(&drain_s);
        __syncwarp();
        int dummy = 0;
        WaitCtx w2{&dummy, p.dev_status};
        mbar_wait(&drain_s, 0, w2);
    } else {
        // ------------------------------------------------------------ O += P V issuer
        constexpr uint32_t idesc_o = idesc_bf16_bmn(kBQ, kD);
        const uint32_t sm0 = smem_u32(smem);
        bool ok = true;
        int n = 0, i = 0;
        for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++i) {
            for (int j = 0; j < ntiles; ++j, ++n) {
                const int s = n % kVStages, b = n & 1;
                if (!__all_sync(0xffffffffu, mbar_wait(&p_full[b], (uint32_t)(n >> 1) & 1u, wc) ? 1 : 0) ||
                    !__all_sync(0xffffffffu, mbar_wait(&v_full[s], (uint32_t)(n / kVStages) & 1u, wc) ? 1 : 0) ||
                    // the first product of an item overwrites O: the previous item's O has been read out
                    (j == 0 && i >= 1 &&
                     !__all_sync(0xffffffffu, mbar_wait(&o_free, (uint32_t)(i - 1) & 1u, wc) ? 1 : 0))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t pt = sm0 + kOffP + b * kTileBf16;
                const uint32_t vt = sm0 + kOffV + s * kTileBf16;
                if (elect_one()) {
                    const uint64_t ad = sdesc_kmajor_sw128(pt), bd = sdesc_v(vt);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)             // 16 keys per MMA
                        tc_mma_bf16(tmem + kColO, ad + p_step(kk), bd + v_step(kk), idesc_o, (j | kk) != 0 ? 1u : 0u);
                    tc_commit(&p_empty[b]);
                    tc_commit(&v_empty[s]);
                    tc_commit(&o_done);
                }
                __syncwarp();
            }
        }
        if (elect_one()) tc_commit(&drain_o);
        __syncwarp();
        int dummy = 0;
        WaitCtx w2{&dummy, p.dev_status};
        mbar_wait(&drain_o, 0, w2);
    }
    } else {
        // ------------------------------------------------------------ softmax and output
        const int q = warp & 3;                     // TMEM lane quarter
        const int r = q * 32 + lane;                // query row in the tile
        // z = s c + bias: the logit in base 2 (c > 0, so the tile maximum of z
        // is c times that of s, plus bias)
        const float c = __fmul_rn(__fmul_rn(*p.g_q, *p.g_k), 1.4426950408889634f / 11.313708498984761f);
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        bool ok = true;
        int n = 0;
        for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
            const float bias = p.s_head ? log2f(p.s_head[item_head(it)]) : 0.0f;
            float m = -INFINITY, l = 0.0f;
            for (int j = 0; j < ntiles; ++j, ++n) {
                const int b = n & 1;
                if (!__all_sync(0xffffffffu, mbar_wait(&s_full[b], (uint32_t)(n >> 1) & 1u, wc) ? 1 : 0)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // the tile's 128 logits of this row, in registers (one TMEM wait)
                uint32_t v[kBK];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4)
                    tmem_ld_32x32b_x32(tmem + lane_base + kColS + b * kBK + c4 * 32,
                                       *reinterpret_cast<uint32_t(*)[32]>(&v[c4 * 32]));
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_empty[b]);
                // eight independent running maxima of s: short dependency chains
                float mx8[8];
#pragma unroll
                for (int i8 = 0; i8 < 8; ++i8) mx8[i8] = -INFINITY;
#pragma unroll
                for (int i8 = 0; i8 < kBK; ++i8) mx8[i8 & 7] = fmaxf(mx8[i8 & 7], __uint_as_float(v[i8]));
                const float smax = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                         fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
                const float mt = fmaf(smax, c, bias);
                // lazy rescaling: the reference maximum moves only when the tile's
                // maximum exceeds it by more than 8 (p stays below 2^8); O and l are
                // rescaled then, and share the reference
                const bool move = mt > m + 8.0f;
                const float mref = move ? mt : m;
                const float alpha = move ? ex2(m - mt) : 1.0f;          // 0 on the first tile (m = -inf)
                const float off = bias - mref;                          // exponent: s c + (bias - mref)
                float sum4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                // P tile reuse: the product that read this buffer two tiles ago is done
                if (n >= 2 &&
                    !__all_sync(0xffffffffu, mbar_wait(&p_empty[b], ((uint32_t)(n >> 1) & 1u) ^ 1u, wc) ? 1 : 0)) {
                    ok = false;
                    break;
                }
                // p = exp2(s c + bias - mref), rounded to bf16 into the swizzled K-major P tile
                uint8_t* prow = smem + kOffP + b * kTileBf16 + r * 128;
#pragma unroll
                for (int c8 = 0; c8 < 16; ++c8) {              // 8 keys per 16-byte unit
                    uint32_t w[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const float e0 = ex2(fmaf(__uint_as_float(v[c8 * 8 + 2 * t]), c, off));
                        const float e1 = ex2(fmaf(__uint_as_float(v[c8 * 8 + 2 * t + 1]), c, off));
                        sum4[t] += e0 + e1;
                        __nv_bfloat162 hb = __floats2bfloat162_rn(e0, e1);
                        w[t] = *reinterpret_cast<uint32_t*>(&hb);
                    }
                    const int kc = c8 >> 3, pos = (c8 & 7) ^ (r & 7);
                    *reinterpret_cast<uint4*>(prow + kc * kChunk + pos * 16) = make_uint4(w[0], w[1], w[2], w[3]);
                }
                l = fmaf(l, alpha, (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]));
                m = mref;
                // rescale the running output by alpha once the previous product is done
                if (j >= 1) {
                    if (!__all_sync(0xffffffffu, mbar_wait(&o_done, (uint32_t)(n - 1) & 1u, wc) ? 1 : 0)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4) {
                            uint32_t o[32];
                            tmem_ld_32x32b_x32(tmem + lane_base + kColO + c4 * 32, o);
                            tmem_ld_wait();
#pragma unroll
                            for (int i8 = 0; i8 < 32; ++i8) o[i8] = __float_as_uint(__uint_as_float(o[i8]) * alpha);
                            tmem_st_x32(tmem + lane_base + kColO + c4 * 32, o);
                        }
                        tmem_st_wait();
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[b]);
            }
            if (!ok) break;
            // output: O * g_v / l, once the item's last product is done; O is
            // read into registers and released before the global stores
            if (!__all_sync(0xffffffffu, mbar_wait(&o_done, (uint32_t)(n - 1) & 1u, wc) ? 1 : 0)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t o[kD];
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
                tmem_ld_32x32b_x32(tmem + lane_base + kColO + c4 * 32, *reinterpret_cast<uint32_t(*)[32]>(&o[c4 * 32]));
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&o_free);
            const float sc = __fdiv_rn(*p.g_v, l);
            uint16_t* orow = p.out + (int64_t)(item_qrow(it) + r) * kD;
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                uint32_t w[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    __nv_bfloat162 hb = __floats2bfloat162_rn(__uint_as_float(o[t * 8 + 2 * u]) * sc,
                                                              __uint_as_float(o[t * 8 + 2 * u + 1]) * sc);
                    w[u] = *reinterpret_cast<uint32_t*>(&hb);
                }
                *reinterpret_cast<uint4*>(orow + t * 8) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
// Two query tiles per CTA.  A work item is 256 queries of one head (query
// tiles A and B); the K and V tiles are loaded once for both.  Two softmax
// warpgroups, one per tile, take turns on the tensor core: while one computes
// its exponentials the other's S = Q K^T runs, so the special-function units
// (the exponentials) rather than one warp's latency set the pace.
// TMEM: one S buffer, used in turn by A and B (a group releases it as soon as
// its logits are in registers), O_A, O_B, and the scale slots.  Shared
// memory: three bf16 P tiles taken in turn by the uses A0, B0, A1, B1, ... (a
// group writes use u once the product of use u - 3 has read that tile, so it
// never waits for its own previous product), a 3-stage K ring, a 2-stage V
// ring and two Q buffers per tile.
// Roles (384 threads): warp 0 Q and K producer, warp 3 V producer, warp 1 S
// issuer (and TMEM owner), warp 2 P V issuer; warps 4-7 softmax of tile A,
// warps 8-11 of tile B.  The register budget moves to the softmax warpgroups
// (setmaxnreg: 48 for warpgroup 0, 224 for 1 and 2; 128 x 48 + 256 x 224 <=
// 384 x 168).
constexpr int kThreads2 = 384;
constexpr int kKStages2 = 3;
constexpr int kVStages2 = 2;
constexpr int kPBufs2 = 3;                                   // P tiles, rotated over the two groups' uses
constexpr int kOffQ2 = 0;                                    // + (qb * 2 + g) * kKStageBytes
constexpr int kOffK2 = 4 * kKStageBytes;
constexpr int kOffV2 = kOffK2 + kKStages2 * kKStageBytes;
constexpr int kOffP2 = kOffV2 + kVStages2 * kTileBf16;        // + b * kTileBf16
constexpr int kSmemBytes2 = kOffP2 + kPBufs2 * kTileBf16 + 1024;
static_assert(kOffK2 % 1024 == 0 && kOffV2 % 1024 == 0 && kOffP2 % 1024 == 0, "swizzled tiles are 1024-byte aligned");
static_assert(kSmemBytes2 <= 232448 - 512, "shared memory budget");
constexpr uint32_t kColS2 = 0;                               // S: [0, 128)
constexpr uint32_t kColO2 = 128;                             // O_g: [128 + 128 g, 256 + 128 g)
constexpr uint32_t kColSfQ2 = 384;                           // Q scales: (qb * 2 + g) * 8
constexpr uint32_t kColSfK2 = 416;                           // K scales: (n & 1) * 8
constexpr int kRegsLow2 = 48;
constexpr int kRegsHigh2 = 224;
static_assert(128 * kRegsLow2 + 256 * kRegsHigh2 <= kThreads2 * 168, "register split exceeds the launch budget");

// Products of group g commit o_done[2 g + (n & 1)] (n: the running tile
// number), so a wait for tile n's product has tile n - 2's as the barrier's
// previous phase -- which the P tile wait has already covered.  The read-out
// after an item's last tile then needs no wait on the second-to-last.
__device__ __forceinline__ int o_bar(int g, int n) { return 2 * g + (n & 1); }
__device__ __forceinline__ uint32_t o_par(int n) { return (uint32_t)(n >> 1) & 1u; }

__global__ void __launch_bounds__(kThreads2, 1)
attn2_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
             const __grid_constant__ CUtensorMap tmap_v, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t q_full[2], q_empty[2], k_full[kKStages2], k_empty[kKStages2];
    __shared__ __align__(8) uint64_t v_full[kVStages2], v_empty[kVStages2];
    __shared__ __align__(8) uint64_t s_full[2], s_empty, p_full[kPBufs2], p_empty[kPBufs2];
    __shared__ __align__(8) uint64_t o_done[4], o_free[2];
    __shared__ __align__(8) uint64_t drain_s, drain_o;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    WaitCtx wc{&abort_sh, p.dev_status};
    const int ntiles = p.Lk / kBK;
    const int qpairs = p.Lq / (2 * kBQ);
    const int nitems = p.H * qpairs;
    auto item_head = [&](int it) { return it / qpairs; };
    auto item_qrow = [&](int it, int g) { return (it / qpairs) * p.Lq + ((it % qpairs) * 2 + g) * kBQ; };

    if (threadIdx.x == 0) {
        abort_sh = 0;
        for (int b = 0; b < 2; ++b) {
            mbar_init(&q_full[b], 1);
            mbar_init(&q_empty[b], 1);               // the item's last S product's commit
            mbar_init(&s_full[b], 1);
            mbar_init(&o_done[2 * b], 1);            // group b's products of even / odd tiles
            mbar_init(&o_done[2 * b + 1], 1);
            mbar_init(&o_free[b], 4);                // the group's softmax warps have read O out
        }
        for (int s = 0; s < kKStages2; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);               // both S products' commit
        }
        for (int s = 0; s < kVStages2; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);               // both P V products' commit
        }
        for (int b = 0; b < kPBufs2; ++b) {
            mbar_init(&p_full[b], 4);                // written by one group's softmax warps
            mbar_init(&p_empty[b], 1);               // the P V product that read it
        }
        mbar_init(&s_empty, 4);                      // the S buffer read out by one group
        mbar_init(&drain_s, 1);
        mbar_init(&drain_o, 1);
        fence_barrier_init();
        tma_prefetch_desc(&tmap_q);
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp < 4) {
        regs_dec<kRegsLow2>();
        if (warp == 0) {
            // -------------------------------------------------------- Q (both tiles) and K producer
            const uint64_t pol = policy_evict_normal();
            bool ok = true;
            int n = 0, i = 0;
            for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++i) {
                const int qb = i & 1, krow0 = item_head(it) * p.Lk;
                if (!__all_sync(0xffffffffu, mbar_wait(&q_empty[qb], ((uint32_t)(i >> 1) & 1u) ^ 1u, wc) ? 1 : 0)) {
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    mbar_arrive_expect_tx(&q_full[qb], 2 * kKStageBytes);
                    for (int g = 0; g < 2; ++g) {
                        uint8_t* qs = smem + kOffQ2 + (qb * 2 + g) * kKStageBytes;
                        const int qrow0 = item_qrow(it, g);
                        tma_load_2d(qs, &tmap_q, &q_full[qb], 0, qrow0, pol);
                        bulk_load(qs + kCodeBytes, p.q_sf + (int64_t)(qrow0 >> 7) * kSfBytes, kSfBytes, &q_full[qb],
                                  pol);
                    }
                }
                __syncwarp();
                for (int j = 0; j < ntiles; ++j, ++n) {
                    const int s = n % kKStages2;
                    const uint32_t ph = (uint32_t)(n / kKStages2) & 1u;
                    if (!__all_sync(0xffffffffu, mbar_wait(&k_empty[s], ph ^ 1u, wc) ? 1 : 0)) { ok = false; break; }
                    uint8_t* st = smem + kOffK2 + s * kKStageBytes;
                    const int kr = krow0 + j * kBK;
                    if (elect_one()) {
                        mbar_arrive_expect_tx(&k_full[s], kKStageBytes);
                        tma_load_2d(st, &tmap_k, &k_full[s], 0, kr, pol);
                        bulk_load(st + kCodeBytes, p.k_sf + (int64_t)(kr >> 7) * kSfBytes, kSfBytes, &k_full[s], pol);
                    }
                    __syncwarp();
                }
            }
            // every load this warp issued has landed before the CTA may exit
            if (lane == 0) {
                int dummy = 0;
                WaitCtx w2{&dummy, p.dev_status};
                for (int q = (i > 2 ? i - 2 : 0); q < i; ++q) mbar_wait(&q_full[q & 1], (uint32_t)(q >> 1) & 1u, w2);
                for (int m = (n > kKStages2 ? n - kKStages2 : 0); m < n; ++m)
                    mbar_wait(&k_full[m % kKStages2], (uint32_t)(m / kKStages2) & 1u, w2);
            }
        } else if (warp == 3) {
            // -------------------------------------------------------- V producer
            const uint64_t pol = policy_evict_normal();
            bool ok = true;
            int n = 0;
            for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
                const int h = item_head(it);
                for (int j = 0; j < ntiles; ++j, ++n) {
                    const int s = n % kVStages2;
                    const uint32_t ph = (uint32_t)(n / kVStages2) & 1u;
                    if (!__all_sync(0xffffffffu, mbar_wait(&v_empty[s], ph ^ 1u, wc) ? 1 : 0)) { ok = false; break; }
                    uint8_t* st = smem + kOffV2 + s * kTileBf16;
                    if (elect_one()) {
                        mbar_arrive_expect_tx(&v_full[s], kTileBf16);
                        tma_load_2d(st, &tmap_v, &v_full[s], 0, h * p.Lk + j * kBK, pol);
                        tma_load_2d(st + kChunk, &tmap_v, &v_full[s], 64, h * p.Lk + j * kBK, pol);
                    }
                    __syncwarp();
                }
            }
            if (lane == 0) {
                int dummy = 0;
                WaitCtx w2{&dummy, p.dev_status};
                for (int m = (n > kVStages2 ? n - kVStages2 : 0); m < n; ++m)
                    mbar_wait(&v_full[m % kVStages2], (uint32_t)(m / kVStages2) & 1u, w2);
            }
        } else if (warp == 1) {
            // -------------------------------------------------------- S = Q K^T issuer (and TMEM owner)
            // The S buffer's uses alternate A, B, A, B, ...; use u waits until
            // the group of use u - 1 has read it out.
            constexpr uint32_t idesc_s = idesc_nvf4(kBQ, kBK);
            const uint32_t sm0 = smem_u32(smem);
            bool ok = true;
            int n = 0, i = 0;
            uint32_t u = 0;
            for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++i) {
                const int qb = i & 1;
                if (!__all_sync(0xffffffffu, mbar_wait(&q_full[qb], (uint32_t)(i >> 1) & 1u, wc) ? 1 : 0)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (elect_one()) {
                    for (int g = 0; g < 2; ++g) {
                        const uint32_t qs = sm0 + kOffQ2 + (qb * 2 + g) * kKStageBytes;
                        const uint32_t sfq = tmem + kColSfQ2 + (qb * 2 + g) * 8;
                        tc_cp_32x128b_warpx4(sfq, sdesc_sf(qs + kCodeBytes));
                        tc_cp_32x128b_warpx4(sfq + 4, sdesc_sf(qs + kCodeBytes + 512));
                    }
                }
                __syncwarp();
                for (int j = 0; j < ntiles && ok; ++j, ++n) {
                    const int s = n % kKStages2;
                    if (!__all_sync(0xffffffffu, mbar_wait(&k_full[s], (uint32_t)(n / kKStages2) & 1u, wc) ? 1 : 0)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = sm0 + kOffK2 + s * kKStageBytes;
                    const uint32_t sfk = tmem + kColSfK2 + (n & 1) * 8;
                    if (elect_one()) {
                        tc_cp_32x128b_warpx4(sfk, sdesc_sf(st + kCodeBytes));
                        tc_cp_32x128b_warpx4(sfk + 4, sdesc_sf(st + kCodeBytes + 512));
                    }
                    __syncwarp();
                    for (int g = 0; g < 2; ++g, ++u) {
                        if (!__all_sync(0xffffffffu, mbar_wait(&s_empty, (u & 1u) ^ 1u, wc) ? 1 : 0)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t qs = sm0 + kOffQ2 + (qb * 2 + g) * kKStageBytes;
                        const uint32_t sfq = tmem + kColSfQ2 + (qb * 2 + g) * 8;
                        if (elect_one()) {
#pragma unroll
                            for (int ks = 0; ks < 2; ++ks)
                                tc_mma_nvf4(tmem + kColS2, sdesc_kmajor_sw64(qs + ks * 32),
                                            sdesc_kmajor_sw64(st + ks * 32), idesc_s, sfq + ks * 4, sfk + ks * 4,
                                            ks != 0 ? 1u : 0u);
                            tc_commit(&s_full[g]);
                            if (g == 1) {
                                tc_commit(&k_empty[s]);
                                if (j == ntiles - 1) tc_commit(&q_empty[qb]);
                            }
                        }
                        __syncwarp();
                    }
                }
            }
            if (elect_one()) tc_commit(&drain_s);
            __syncwarp();
            int dummy = 0;
            WaitCtx w2{&dummy, p.dev_status};
            mbar_wait(&drain_s, 0, w2);
        } else {
            // -------------------------------------------------------- O_g += P_g V issuer
            constexpr uint32_t idesc_o = idesc_bf16_bmn(kBQ, kD);
            const uint32_t sm0 = smem_u32(smem);
            bool ok = true;
            int n = 0, i = 0;
            for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++i) {
                for (int j = 0; j < ntiles && ok; ++j, ++n) {
                    const int s = n % kVStages2;
                    if (!__all_sync(0xffffffffu, mbar_wait(&v_full[s], (uint32_t)(n / kVStages2) & 1u, wc) ? 1 : 0)) {
                        ok = false;
                        break;
                    }
                    const uint32_t vt = sm0 + kOffV2 + s * kTileBf16;
                    for (int g = 0; g < 2; ++g) {
                        const uint32_t u = 2u * (uint32_t)n + (uint32_t)g;
                        const int pb = (int)(u % kPBufs2);
                        if (!__all_sync(0xffffffffu, mbar_wait(&p_full[pb], (u / kPBufs2) & 1u, wc) ? 1 : 0) ||
                            // the first product of an item overwrites O_g: the previous item's O_g has been read out
                            (j == 0 && i >= 1 &&
                             !__all_sync(0xffffffffu, mbar_wait(&o_free[g], (uint32_t)(i - 1) & 1u, wc) ? 1 : 0))) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t pt = sm0 + kOffP2 + pb * kTileBf16;
                        if (elect_one()) {
                            const uint64_t ad = sdesc_kmajor_sw128(pt), bd = sdesc_v(vt);
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk)     // 16 keys per MMA
                                tc_mma_bf16(tmem + kColO2 + g * kD, ad + p_step(kk), bd + v_step(kk), idesc_o,
                                            (j | kk) != 0 ? 1u : 0u);
                            tc_commit(&p_empty[pb]);
                            tc_commit(&o_done[o_bar(g, n)]);
                            if (g == 1) tc_commit(&v_empty[s]);
                        }
                        __syncwarp();
                    }
                }
            }
            if (elect_one()) tc_commit(&drain_o);
            __syncwarp();
            int dummy = 0;
            WaitCtx w2{&dummy, p.dev_status};
            mbar_wait(&drain_o, 0, w2);
        }
    } else {
        regs_inc<kRegsHigh2>();
        // ------------------------------------------------------------ softmax and output of tile g
        const int g = (warp - 4) >> 2;              // 0: tile A (warps 4-7), 1: tile B (warps 8-11)
        const int q = warp & 3;                     // TMEM lane quarter
        const int r = q * 32 + lane;                // query row in the tile
        const float c = __fmul_rn(__fmul_rn(*p.g_q, *p.g_k), 1.4426950408889634f / 11.313708498984761f);
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const uint32_t col_o = kColO2 + g * kD;
        bool ok = true;
        int n = 0;
        for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
            const float bias = p.s_head ? log2f(p.s_head[item_head(it)]) : 0.0f;
            float m = -INFINITY, l = 0.0f;
            for (int j = 0; j < ntiles; ++j, ++n) {
                if (!__all_sync(0xffffffffu, mbar_wait(&s_full[g], (uint32_t)n & 1u, wc) ? 1 : 0)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t v[kBK];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4)
                    tmem_ld_32x32b_x32(tmem + lane_base + kColS2 + c4 * 32, *reinterpret_cast<uint32_t(*)[32]>(&v[c4 * 32]));
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_empty);
                float mx8[8];
#pragma unroll
                for (int i8 = 0; i8 < 8; ++i8) mx8[i8] = -INFINITY;
#pragma unroll
                for (int i8 = 0; i8 < kBK; ++i8) mx8[i8 & 7] = fmaxf(mx8[i8 & 7], __uint_as_float(v[i8]));
                const float smax = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                         fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
                const float mt = fmaf(smax, c, bias);
                // lazy rescaling, as in the one-tile kernel
                const bool move = mt > m + 8.0f;
                const float mref = move ? mt : m;
                const float alpha = move ? ex2(m - mt) : 1.0f;
                const float off = bias - mref;
                float sum4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                // P tile of use u = 2 n + g: the product that read it at use u - 3 is done
                const uint32_t u = 2u * (uint32_t)n + (uint32_t)g;
                const int pb = (int)(u % kPBufs2);
                if (!__all_sync(0xffffffffu, mbar_wait(&p_empty[pb], ((u / kPBufs2) & 1u) ^ 1u, wc) ? 1 : 0)) {
                    ok = false;
                    break;
                }
                uint8_t* pbase = smem + kOffP2 + pb * kTileBf16 + r * 128;
#pragma unroll
                for (int c8 = 0; c8 < 16; ++c8) {
                    uint32_t w[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const float e0 = ex2(fmaf(__uint_as_float(v[c8 * 8 + 2 * t]), c, off));
                        const float e1 = ex2(fmaf(__uint_as_float(v[c8 * 8 + 2 * t + 1]), c, off));
                        sum4[t] += e0 + e1;
                        __nv_bfloat162 hb = __floats2bfloat162_rn(e0, e1);
                        w[t] = *reinterpret_cast<uint32_t*>(&hb);
                    }
                    const int kc = c8 >> 3, pos = (c8 & 7) ^ (r & 7);
                    *reinterpret_cast<uint4*>(pbase + kc * kChunk + pos * 16) = make_uint4(w[0], w[1], w[2], w[3]);
                }
                l = fmaf(l, alpha, (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]));
                m = mref;
                // O_g rescaled by alpha once this group's previous product is done
                if (j >= 1 && __any_sync(0xffffffffu, alpha != 1.0f)) {
                    if (!__all_sync(0xffffffffu, mbar_wait(&o_done[o_bar(g, n - 1)], o_par(n - 1), wc) ? 1 : 0)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        uint32_t o[32];
                        tmem_ld_32x32b_x32(tmem + lane_base + col_o + c4 * 32, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int i8 = 0; i8 < 32; ++i8) o[i8] = __float_as_uint(__uint_as_float(o[i8]) * alpha);
                        tmem_st_x32(tmem + lane_base + col_o + c4 * 32, o);
                    }
                    tmem_st_wait();
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[pb]);
            }
            if (!ok) break;
            if (!__all_sync(0xffffffffu, mbar_wait(&o_done[o_bar(g, n - 1)], o_par(n - 1), wc) ? 1 : 0)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t o[kD];
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
                tmem_ld_32x32b_x32(tmem + lane_base + col_o + c4 * 32, *reinterpret_cast<uint32_t(*)[32]>(&o[c4 * 32]));
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&o_free[g]);
            const float sc = __fdiv_rn(*p.g_v, l);
            uint16_t* orow = p.out + (int64_t)(item_qrow(it, g) + r) * kD;
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                uint32_t w[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    __nv_bfloat162 hb = __floats2bfloat162_rn(__uint_as_float(o[t * 8 + 2 * u]) * sc,
                                                              __uint_as_float(o[t * 8 + 2 * u + 1]) * sc);
                    w[u] = *reinterpret_cast<uint32_t*>(&hb);
                }
                *reinterpret_cast<uint4*>(orow + t * 8) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// V [H*Lk, d] NVFP4 -> V [H*Lk, d] bf16, exact (the tensor scale g_v is
// applied with the output).  A thread decodes one 4-byte code word (8 values,
// half a 16-value block) into one 16-byte store, so a warp reads 128 and
// writes 512 contiguous bytes; 4 words per thread, a block-width apart.
constexpr int kVdThreads = 256;
constexpr int kVdWords = 4;                      // code words per thread

__global__ void __launch_bounds__(kVdThreads)
v_decode_kernel(const uint8_t* __restrict__ v_codes, const uint8_t* __restrict__ v_sf, int64_t rows,
                uint16_t* __restrict__ v) {
    const int64_t words = rows * (kD / 8);                 // 16 code words per row
    const int64_t w0 = (int64_t)blockIdx.x * (kVdThreads * kVdWords) + threadIdx.x;
#pragma unroll
    for (int u = 0; u < kVdWords; ++u) {
        const int64_t w = w0 + u * kVdThreads;
        if (w >= words) break;
        const uint32_t cw = *reinterpret_cast<const uint32_t*>(v_codes + w * 4);
        // scale of block (w % 16) / 2 of row w / 16; layout of a [rows, 128]
        // tensor: two 512-byte atoms per 128-row group
        const int64_t row = w >> 4;
        const int blk = (int)(w & 15) >> 1, rr = (int)(row & 127);
        const uint32_t sc = e4m3_to_b2_scaled_attn(
            v_sf[(row >> 7) * 1024 + (blk >> 2) * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (blk & 3)]);
        uint4 o;
        o.x = dequant_pair_attn(cw & 0xFFu, sc);
        o.y = dequant_pair_attn((cw >> 8) & 0xFFu, sc);
        o.z = dequant_pair_attn((cw >> 16) & 0xFFu, sc);
        o.w = dequant_pair_attn(cw >> 24, sc);
        *reinterpret_cast<uint4*>(v + w * 8) = o;
    }
}

}  // namespace attn

size_t attention_workspace_bytes(int64_t H, int64_t Lk, int64_t d) { return (size_t)(H * d * Lk) * 2; }

cudaError_t launch_attention(const uint8_t* q_codes, const uint8_t* q_sf, const float* g_q, const uint8_t* k_codes,
                             const uint8_t* k_sf, const float* g_k, const uint8_t* v_codes, const uint8_t* v_sf,
                             const float* g_v, const float* s_head, int64_t H, int64_t Lq, int64_t Lk, void* out,
                             void* workspace, int* dev_status, cudaStream_t stream) {
    using namespace attn;
    uint16_t* vd = static_cast<uint16_t*>(workspace);
    CUtensorMap tq, tk, tv;
    if (make_tmap_2d(&tq, q_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kD / 2, (uint64_t)(H * Lq), kD / 2, kD / 2, kBQ,
                     CU_TENSOR_MAP_SWIZZLE_64B) != CUDA_SUCCESS ||
        make_tmap_2d(&tk, k_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kD / 2, (uint64_t)(H * Lk), kD / 2, kD / 2, kBK,
                     CU_TENSOR_MAP_SWIZZLE_64B) != CUDA_SUCCESS ||
        make_tmap_2d(&tv, vd, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kD, (uint64_t)(H * Lk), kD * 2, 64, kBK,
                     CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const int64_t vwords = H * Lk * (kD / 8);
    v_decode_kernel<<<(unsigned)((vwords + kVdThreads * kVdWords - 1) / (kVdThreads * kVdWords)), kVdThreads, 0,
                      stream>>>(v_codes, v_sf, H * Lk, vd);
    count_launch(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    Params p;
    p.q_sf = q_sf;
    p.k_sf = k_sf;
    p.g_q = g_q;
    p.g_k = g_k;
    p.g_v = g_v;
    p.s_head = s_head;
    p.out = static_cast<uint16_t*>(out);
    p.Lq = (int)Lq;
    p.Lk = (int)Lk;
    p.H = (int)H;
    p.dev_status = dev_status;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    // two query tiles per CTA when a head's query tiles pair up
    // (NVFP4_ATTN_TILES=1 keeps one, for measurements)
    const char* env = getenv("NVFP4_ATTN_TILES");
    const bool two = (Lq / kBQ) % 2 == 0 && !(env && env[0] == '1');
    const int64_t items = (Lq / (two ? 2 * kBQ : kBQ)) * H;
    const unsigned grid = (unsigned)(items < sms ? items : sms);     // one persistent CTA per SM
    if (two) {
        e = cudaFuncSetAttribute(attn2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes2);
        if (e != cudaSuccess) return e;
        attn2_kernel<<<grid, kThreads2, kSmemBytes2, stream>>>(tq, tk, tv, p);
    } else {
        e = cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        attn_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tq, tk, tv, p);
    }
    count_launch(1);
    return cudaGetLastError();
}

}  // namespace nvfp4
