// attn.cu -- attention over an NVFP4 key / value cache ("NVFP4-DiT ..."
// README, Algorithmic framework, Eq. 10: Attention(Q, K, V) =
// softmax(Q K^T / sqrt(d_k) + log(s_head)) V with a per-head scale s_head;
// Systems optimization: FP4-packed attention).
//
// Q, K, V are NVFP4 tensors quantized along the head dimension d = 128
// (blocks of 16, tensor scales g_q, g_k, g_v): Q [H*Lq, d], K and V [H*Lk, d].
// Two kernels:
//   v_decode      V decoded exactly to f16 (e2m1 * e4m3: at most 6
//                 significant bits, within f16's normal range), [H*Lk, d] in
//                 the caller's workspace -- once per call, instead of once per
//                 query tile (the two-tile kernel decodes V itself instead);
//   attention     persistent, one CTA per SM; a work item is 128 (or 256)
//                 queries of one head, keys in tiles of 128:
//     S = Q K^T   block-scaled FP4 MMA (kind::mxf4nvf4, K = d), FP32 in TMEM,
//                 two S buffers so the next tile's product overlaps softmax;
//     softmax     one query row per thread (online: reference maximum m, sum
//                 l), exp2 of (S * g_q g_k log2(e) / sqrt(d) + log2(s_head) - m),
//                 P rounded to f16 into a 128-byte-swizzled K-major tile; the
//                 running output is rescaled in TMEM when m moves;
//     O += P V    f16 MMA (kind::f16) on TMA-loaded V tiles (B operand
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
#include <cuda_fp16.h>

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
// ring (f16 rows of keys, d 0-63 then d 64-127, 128-byte swizzle); two P
// tiles (f16, 128-byte swizzle)
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
    // V decoded inside the two-tile kernel (null slots: decoded by a pre-pass)
    const uint8_t* v_codes;
    const uint8_t* v_sf;
    uint16_t* vd;                            // f16 V [H*Lk, d] in the workspace
    uint32_t* slots;                         // per head 32 words: the call number once a part is decoded
    uint32_t gen;                            // this call's number
    int rpp;                                 // V rows per part (one part per work item of a head)
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

// Two E2M1 codes (one byte, low nibble first) times their block scale, as an
// f16 pair, exactly: the product has at most 6 significant bits and lies in
// [2^-10, 2688], inside f16's normal range.
__device__ __forceinline__ uint32_t dequant_pair_f16(uint32_t byte, uint32_t scale_h2) {
    uint32_t h2, out;
    asm("{\n\t.reg .b8 c;\n\t"
        "cvt.u8.u32 c, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, c;\n\t}"
        : "=r"(h2)
        : "r"(byte));
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(out) : "r"(h2), "r"(scale_h2));
    return out;
}

// E4M3 byte -> its value in both halves of an f16 pair (exact).
__device__ __forceinline__ uint32_t e4m3_to_h2(uint32_t code) {
    uint32_t h2;
    const uint16_t in = (uint16_t)((code & 0xFFu) * 0x101u);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return h2;
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

// kind::f16 instruction descriptor: A and B f16 (formats 0 in bits [7,10) and
// [10,13)), FP32 accumulate (bit 4), B MN-major (bit 16), N >> 3 in [17,23),
// M >> 4 in [24,29).
__host__ __device__ constexpr uint32_t idesc_f16_bmn(int M, int N) {
    return (1u << 4) | (1u << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Block b of V (row b / 8, values 16 (b % 8) .. + 15): its scale byte sits in
// the scale layout of a [rows, 128] tensor, two 512-byte atoms per 128-row
// group; its 8 code bytes decode to 32 bytes of f16 V [H*Lk, d].
__device__ __forceinline__ const uint8_t* v_scale_ptr(const uint8_t* v_sf, int64_t b) {
    const int64_t row = b >> 3;
    const int blk = (int)(b & 7), rr = (int)(row & 127);
    return v_sf + (row >> 7) * 1024 + (blk >> 2) * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (blk & 3);
}

__device__ __forceinline__ void decode_store_v(uint2 c, uint32_t sf, int64_t b, uint16_t* __restrict__ v) {
    const uint32_t sc = e4m3_to_h2(sf);
    uint4 o0, o1;
    o0.x = dequant_pair_f16(c.x & 0xFFu, sc);
    o0.y = dequant_pair_f16((c.x >> 8) & 0xFFu, sc);
    o0.z = dequant_pair_f16((c.x >> 16) & 0xFFu, sc);
    o0.w = dequant_pair_f16(c.x >> 24, sc);
    o1.x = dequant_pair_f16(c.y & 0xFFu, sc);
    o1.y = dequant_pair_f16((c.y >> 8) & 0xFFu, sc);
    o1.z = dequant_pair_f16((c.y >> 16) & 0xFFu, sc);
    o1.w = dequant_pair_f16(c.y >> 24, sc);
    uint4* dst = reinterpret_cast<uint4*>(v + b * 16);
    dst[0] = o0;
    dst[1] = o1;
}

// Up to four blocks b = c0 + t + stride i (i < 4, b < c1): every load is
// issued before any value is used (V's codes and scales are read-only here),
// so one batch costs about one memory latency.
constexpr int kVBatch = 4;

__device__ __forceinline__ void v_batch_load(const uint8_t* __restrict__ v_codes, const uint8_t* __restrict__ v_sf,
                                             int64_t c0, int64_t c1, int t, int stride, uint2 (&c)[kVBatch],
                                             uint32_t (&sf)[kVBatch]) {
#pragma unroll
    for (int i = 0; i < kVBatch; ++i) {
        const int64_t b = c0 + t + (int64_t)stride * i;
        if (b < c1) {
            c[i] = __ldg(reinterpret_cast<const uint2*>(v_codes) + b);
            sf[i] = __ldg(v_scale_ptr(v_sf, b));
        }
    }
}

__device__ __forceinline__ void v_batch_store(int64_t c0, int64_t c1, int t, int stride, const uint2 (&c)[kVBatch],
                                              const uint32_t (&sf)[kVBatch], uint16_t* __restrict__ v) {
#pragma unroll
    for (int i = 0; i < kVBatch; ++i) {
        const int64_t b = c0 + t + (int64_t)stride * i;
        if (b < c1) decode_store_v(c[i], sf[i], b, v);
    }
}

// ---------------------------------------------------------------------------
// V decoded inside the two-tile kernel.  Work item (head h, query pair q)
// decodes V rows [q rpp, (q + 1) rpp) of its head into the f16 workspace --
// rpp = ceil(Lk / qpairs), so the items of a head share its rows -- and
// marks part q done by storing the call number in the head's slot q.
// An item may load its head's V once every part is marked.  A CTA decodes
// the parts of its own items two rounds ahead: items c and c + grid with all
// its threads at the start, then, while it runs item it, the part of item
// it + 2 grid, a slice of at most 4 blocks per lane per key tile on the V
// producer warp (which otherwise waits for ring slots; the next slice's
// loads are in flight during that wait).  Every wait is on parts published a round earlier
// or at the start, never on the waiter's own progress, and the grid is
// cooperative (every CTA resident); waits are bounded all the same.
// Writers order their stores before the slot update with a proxy fence (the
// readers load V by TMA) and a GPU-scope fence; readers acquire the slot and
// fence the async proxy before their loads.

// 16-value blocks of part q of head h: [first, last).
__device__ __forceinline__ void part_blocks(const Params& p, int h, int q, int64_t& first, int64_t& last) {
    const int r0 = q * p.rpp, r1 = min(p.Lk, (q + 1) * p.rpp);
    first = ((int64_t)h * p.Lk + r0) * (kD / 16);
    last = ((int64_t)h * p.Lk + (r1 > r0 ? r1 : r0)) * (kD / 16);
}

__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Marks a part decoded for call `gen` (a store with release semantics; the
// caller's threads have fenced the part's stores and joined).
__device__ __forceinline__ void publish_part(uint32_t* slot, uint32_t gen) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(slot), "r"(gen) : "memory");
}

// One warp: waits (bounded) until the head's `parts` slots all carry call
// `gen`; lane q reads slot q.
__device__ __forceinline__ bool wait_parts(const uint32_t* slots, int parts, uint32_t gen, int lane, const WaitCtx& w) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        uint32_t v = gen;
        if (lane < parts) asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(slots + lane) : "memory");
        if (__all_sync(0xffffffffu, v == gen)) return true;
        if ((n & 63u) == 0u) {
            const bool give_up = *w.abort_flag || globaltimer_ns() - t0 > kWaitLimitNs;
            if (__any_sync(0xffffffffu, give_up)) {
                if (lane == 0 && !*w.abort_flag) report_timeout(w);
                return false;
            }
        }
        __nanosleep(64);
    }
}

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
        constexpr uint32_t idesc_o = idesc_f16_bmn(kBQ, kD);
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
                // p = exp2(s c + bias - mref), rounded to f16 into the swizzled K-major P tile
                uint8_t* prow = smem + kOffP + b * kTileBf16 + r * 128;
#pragma unroll
                for (int c8 = 0; c8 < 16; ++c8) {              // 8 keys per 16-byte unit
                    uint32_t w[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const float e0 = ex2(fmaf(__uint_as_float(v[c8 * 8 + 2 * t]), c, off));
                        const float e1 = ex2(fmaf(__uint_as_float(v[c8 * 8 + 2 * t + 1]), c, off));
                        sum4[t] += e0 + e1;
                        __half2 hh = __floats2half2_rn(e0, e1);
                        w[t] = *reinterpret_cast<uint32_t*>(&hh);
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
// memory: three f16 P tiles taken in turn by the uses A0, B0, A1, B1, ... (a
// group writes use u once the product of use u - 3 has read that tile, so it
// never waits for its own previous product), a 3-stage K ring, a 2-stage V
// ring and two Q buffers per tile.
// Roles (384 threads): warp 0 Q and K producer, warp 3 V producer, warp 1 S
// issuer (and TMEM owner), warp 2 P V issuer; warps 4-7 softmax of tile A,
// warps 8-11 of tile B.  The register budget moves to the softmax warpgroups
// (setmaxnreg: 64 for warpgroup 0, whose V producer also decodes V, 208 for
// 1 and 2; 128 x 64 + 256 x 208 <= 384 x 168).
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
constexpr int kRegsLow2 = 64;
constexpr int kRegsHigh2 = 208;
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

    if (p.slots != nullptr) {
        // V decoded here: the parts of this CTA's first two items, by every thread
        for (int k = 0; k < 2; ++k) {
            const int it = blockIdx.x + k * gridDim.x;
            if (it >= nitems) break;
            int64_t b0, b1;
            part_blocks(p, item_head(it), it % qpairs, b0, b1);
            for (int64_t b = b0; b < b1; b += kVBatch * kThreads2) {
                uint2 c[kVBatch];
                uint32_t sf[kVBatch];
                v_batch_load(p.v_codes, p.v_sf, b, b1, threadIdx.x, kThreads2, c, sf);
                v_batch_store(b, b1, threadIdx.x, kThreads2, c, sf, p.vd);
            }
        }
        fence_proxy_async_global();
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0)
            for (int k = 0; k < 2; ++k) {
                const int it = blockIdx.x + k * gridDim.x;
                if (it < nitems) publish_part(p.slots + item_head(it) * 32 + it % qpairs, p.gen);
            }
    }

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
            // -------------------------------------------------------- V producer (and decoder)
            const uint64_t pol = policy_evict_normal();
            bool ok = true;
            int n = 0;
            for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
                const int h = item_head(it);
                // the part of item it + 2 grid, a slice after each key tile's loads
                const int ahead = it + 2 * (int)gridDim.x;
                const bool decode_ahead = p.slots != nullptr && ahead < nitems;
                int64_t a0 = 0, a1 = 0, per = 0;
                uint2 cw[kVBatch];                            // the next slice, in flight
                uint32_t sf[kVBatch];
                if (p.slots != nullptr) {
                    // every part of this item's head decoded
                    if (!wait_parts(p.slots + h * 32, qpairs, p.gen, lane, wc)) { ok = false; break; }
                    fence_proxy_async_global();
                    if (decode_ahead) {
                        part_blocks(p, item_head(ahead), ahead % qpairs, a0, a1);
                        per = (a1 - a0 + ntiles - 1) / ntiles;      // <= 32 lanes x 4 (host check)
                        v_batch_load(p.v_codes, p.v_sf, a0, a0 + per < a1 ? a0 + per : a1, lane, 32, cw, sf);
                    }
                }
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
                    if (decode_ahead) {
                        const int64_t c0 = a0 + j * per, c1 = c0 + per < a1 ? c0 + per : a1;
                        v_batch_store(c0, c1, lane, 32, cw, sf, p.vd);
                        if (j + 1 < ntiles) {
                            const int64_t n0 = c0 + per;
                            v_batch_load(p.v_codes, p.v_sf, n0, n0 + per < a1 ? n0 + per : a1, lane, 32, cw, sf);
                        }
                        if (j == ntiles - 1) {                  // published even when the part is empty
                            fence_proxy_async_global();
                            __threadfence();
                            __syncwarp();
                            if (lane == 0) publish_part(p.slots + item_head(ahead) * 32 + ahead % qpairs, p.gen);
                        }
                    }
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
            // the group of use u - 1 has read it out.  Each use is issued as two
            // N = 64 products (keys 0-63, 64-127: the B operand and its scales
            // start 64 rows -- 4 KB of codes, two TMEM columns -- on for the
            // second), measured a little faster than one N = 128 product.
            constexpr uint32_t idesc_s = idesc_nvf4(kBQ, 64);
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
                            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                                for (int ks = 0; ks < 2; ++ks)
                                    tc_mma_nvf4(tmem + kColS2 + 64 * hh, sdesc_kmajor_sw64(qs + ks * 32),
                                                sdesc_kmajor_sw64(st + 4096 * hh + ks * 32), idesc_s, sfq + ks * 4,
                                                sfk + ks * 4 + 2 * hh, ks != 0 ? 1u : 0u);
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
            constexpr uint32_t idesc_o = idesc_f16_bmn(kBQ, kD);
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
                        __half2 hh = __floats2half2_rn(e0, e1);
                        w[t] = *reinterpret_cast<uint32_t*>(&hh);
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

// V [H*Lk, d] NVFP4 -> V [H*Lk, d] f16, exact (the tensor scale g_v is
// applied with the output): kernel used when the attention kernel does not
// decode V itself.  A thread decodes two 16-value blocks, a block-width
// apart (8 code bytes in, 32 bytes out each).
constexpr int kVdThreads = 256;
constexpr int kVdBlocks = 2;                     // blocks per thread

__global__ void __launch_bounds__(kVdThreads)
v_decode_kernel(const uint8_t* __restrict__ v_codes, const uint8_t* __restrict__ v_sf, int64_t rows,
                uint16_t* __restrict__ v) {
    const int64_t blocks = rows * (kD / 16);
    const int64_t b0 = (int64_t)blockIdx.x * (kVdThreads * kVdBlocks) + threadIdx.x;
#pragma unroll
    for (int u = 0; u < kVdBlocks; ++u) {
        const int64_t b = b0 + u * kVdThreads;
        if (b >= blocks) break;
        decode_store_v(__ldg(reinterpret_cast<const uint2*>(v_codes) + b), __ldg(v_scale_ptr(v_sf, b)), b, v);
    }
}

}  // namespace attn

// f16 V [H*Lk, d], then 32 four-byte decode slots per head
size_t attention_workspace_bytes(int64_t H, int64_t Lk, int64_t d) { return (size_t)(H * d * Lk) * 2 + (size_t)H * 128; }

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
        make_tmap_2d(&tv, vd, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, kD, (uint64_t)(H * Lk), kD * 2, 64, kBK,
                     CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
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
    p.v_codes = v_codes;
    p.v_sf = v_sf;
    p.vd = vd;
    p.slots = nullptr;
    p.gen = 0;
    p.rpp = 0;
    int dev = 0, sms = 0;
    cudaError_t e;
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
        // V decoded inside the kernel (a head's items share its rows; at most 32
        // parts per head, and no more than CTAs, so that a head's items fall in
        // at most two consecutive rounds and every part an item waits for is
        // published before its round starts; at most one 8-word batch per lane
        // and key tile), on a cooperative grid; NVFP4_ATTN_DECODE=prepass keeps
        // the separate pass, for measurements
        const char* denv = getenv("NVFP4_ATTN_DECODE");
        const int64_t qpairs = Lq / (2 * kBQ);
        const int64_t rpp = (Lk + qpairs - 1) / qpairs, per = (rpp * (kD / 16) + Lk / kBK - 1) / (Lk / kBK);
        if (qpairs <= 32 && qpairs <= (int64_t)grid && per <= 32 * kVBatch && !(denv && denv[0] == 'p')) {
            p.slots = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + (size_t)(H * kD * Lk) * 2);
            p.gen = next_generation();
            p.rpp = (int)rpp;
            cudaLaunchConfig_t cfg = {};
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeCooperative;      // every CTA resident: the parts' waits
            attr[0].val.cooperative = 1;
            cfg.gridDim = dim3(grid);
            cfg.blockDim = dim3(kThreads2);
            cfg.dynamicSmemBytes = kSmemBytes2;
            cfg.stream = stream;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            e = cudaLaunchKernelEx(&cfg, attn2_kernel, tq, tk, tv, p);
            if (e == cudaSuccess) {
                count_launch(1);
                return cudaGetLastError();
            }
            if (e != cudaErrorCooperativeLaunchTooLarge) return e;
            (void)cudaGetLastError();                           // not co-resident: the separate pass
            p.slots = nullptr;
        }
    }
    const int64_t vblocks = H * Lk * (kD / 16);
    v_decode_kernel<<<(unsigned)((vblocks + kVdThreads * kVdBlocks - 1) / (kVdThreads * kVdBlocks)), kVdThreads, 0,
                      stream>>>(v_codes, v_sf, H * Lk, vd);
    count_launch(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (two) {
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
