// gemm_w4a4_2sm.cu -- the W4A4 GEMM on CTA pairs (tcgen05 cta_group::2):
// one 256 x BN output tile per pair (BN = 192 or 256), each CTA holding 128
// rows of A, one BN/2-row half of B and the scales of every B row of the
// tile; per K step the leader CTA issues a single M=256, N=BN, K=64
// block-scaled MMA whose accumulator rows land in both CTAs' TMEM.
//
// Same operation as gemm_w4a4.cu ("NVFP4-DiT ..." README, Methodology 3;
// "[RFC]: NVFP4 Quantization Support for Diffusion Models", Open Questions 1):
//   Y[m,n] = (g_a g_b) * sum_k (e2m1(a) e4m3(sfa)) (e2m1(b) e4m3(sfb))
//
// Why pairs: per SM, a 128 x 256 x 256 K-stage needs 38 KB of operands
// instead of 54 KB for a single-CTA 128 x 256 tile, and L2 -> SM operand
// traffic per output drops by a third.
//
// Why BN = 192: TMEM has 512 columns.  A 256-wide tile's FP32 accumulator
// takes 256 of them and the scale atoms of a stage 48 more, so a second
// accumulator cannot fit and every tile boundary waits for the epilogue to
// drain TMEM (about 1.5-2 k cycles per tile).  With BN = 192 two
// accumulators (384 columns) and a two-slot scale ring (96 columns) fit: the
// next tile's MMAs run while the epilogue drains the previous one.  A 192-row
// B tile starts half-way into a 128-row scale atom on odd tiles; the atoms
// are copied whole and the MMA's B-scale address is moved two columns on
// (one TMEM column holds the scales of 32 B rows).
//
// Roles (512 threads per CTA):
//   warp 0     producer, both CTAs: TMA loads of this CTA's scale atoms (its
//              128 A rows, both 128-row atom blocks the tile's B rows touch),
//              A rows and B half into a STAGES-deep ring.  Every load of the
//              pair completes on the LEADER's full barrier (cta_group::2),
//              which the leader arms with the bytes of both CTAs: one wait
//              per stage tells the MMA issuer that both CTAs' operands landed.
//   warp 2     leader CTA, 256-wide tiles: scale copier.  Per K=64 step three
//              tcgen05.cp of the scale atoms into the stage's TMEM scale slot;
//              one commit per stage to the leader's "scaled" barrier.  With
//              192-wide tiles (two slots) the MMA warp issues the same copies
//              itself, just before the stage's MMAs.
//   warp 1     leader CTA: MMA issuer.  Per K=64 step one tcgen05.mma
//              cta_group::2; one commit per stage, multicast to both CTAs'
//              "empty" barriers; one per tile to the accumulator's "full".
//   warps 8-15 epilogue, both CTAs: the 128 x BN FP32 accumulator slice is
//              read into registers (two warps per TMEM lane quarter, BN/2
//              columns each) and released to the MMA issuer at once, then
//              converted and stored while the mainloop runs.  With the
//              NVFP4 output (activation and block quantization per element:
//              about 13 instructions per value, more than two warps per
//              sub-partition issue within a tile's mainloop) warps 4-15: three
//              per lane quarter, 96 (BN 256) or 64 (BN 192) columns each.
// Producer, copier and MMA issuer run on whole warps with one elected lane
// issuing: the descriptors, coordinates and addresses then stay warp-uniform.
// Issued from a single lane, the same copies and MMAs took longer to issue
// than to execute; on one warp the twelve copies still cost the MMA loop ~90
// cycles per stage (~626 against ~533), hence the separate copier.
// The cross-CTA release of the accumulator is a relaxed arrive ordered by
// tcgen05.wait::ld and tcgen05.fence::before_thread_sync (a cluster-scope
// release costs about a microsecond per arrive).
// Registers: launched at 128 per thread; warpgroups 0-1 drop to 56 and the
// epilogue warpgroups rise to 200 (256 x 56 + 256 x 200 = 512 x 128); 80 and
// 176 with 192-wide tiles; with the NVFP4 output warpgroup 0 drops to 56 (80)
// and warpgroups 1-3 rise to 152 (144).
// No load uses cluster multicast: every CTA fetches its own tiles.
#include <cstdlib>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "gemm.h"
#include "ptx.cuh"
#include "quant_math.cuh"
#include "epilogue.cuh"
#include "tmap.h"

namespace nvfp4 {
namespace w4a4_2sm {

constexpr int BK_BYTES = 128;                    // 256 FP4 values per row per stage
constexpr int A_BYTES = 128 * BK_BYTES;          // this CTA's 128 rows of A
constexpr int SF_ATOM = 512;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 512;
// register split (setmaxnreg): warpgroups 0-1 (producer, MMA, copier) drop
// to REGS_LOW, the epilogue warpgroups 2-3 rise to REGS_HIGH; a 256-wide
// tile's epilogue holds 128 accumulator columns per thread, a 192-wide one 96
template <int BN>
struct Regs {
    static constexpr int LOW = BN == 192 ? 80 : 56;
    static constexpr int HIGH = BN == 192 ? 176 : 200;
    static_assert(256 * LOW + 256 * HIGH <= kThreads * 128, "register split exceeds the launch budget");
};
constexpr int SF_COLS_ATOM = 4 + 8;              // SFA 4 columns, SFB 8 columns (two 128-row atoms) per scale atom
constexpr int kGroupM = 8;                       // rasterisation group, in 256-row pair tiles
constexpr int kPairGroup = 8;                    // problems of a grouped launch
constexpr int kSmemLimit = 232448;

enum OutKind { OUT_BF16 = 0, OUT_F32 = 1, OUT_NVFP4 = 2 };

// Per-stage layout.  NVFP4 (kind::mxf4nvf4, block16): a 128-row scale atom
// covers K = 64, four per stage.  MX (kind::mxf4, block32): an atom covers
// K = 128, two per stage; each K = 64 MMA step reads two of a row's four
// scale bytes, selected by a byte id.  B scales: the two 128-row atom blocks
// that the tile's BN rows touch.
template <int BN, bool MXS>
struct Lay {
    static_assert(BN == 192 || BN == 256, "pair tile width");
    static constexpr int B_ROWS = BN / 2;                         // this CTA's half of the tile's B rows
    static constexpr int B_BYTES = B_ROWS * BK_BYTES;
    static constexpr int SF_PER = MXS ? 2 : 4;   // scale atoms per 128 rows per stage
    static constexpr int K_ATOM = MXS ? 128 : 64;
    static constexpr int SFA_BYTES = SF_PER * SF_ATOM;            // this CTA's 128 A rows
    static constexpr int SFB_BYTES = 2 * SFA_BYTES;               // two 128-row blocks of B
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;   // NVFP4: 38912 / 34816
    static constexpr int SF_COLS_STAGE = SF_PER * SF_COLS_ATOM;
    static_assert(STAGE_BYTES % 1024 == 0, "stages keep the 128-byte-swizzled tiles 1024-byte aligned");
};

template <int BN, int OUT, bool MXS>
struct Cfg {
    using L = Lay<BN, MXS>;
    static constexpr int STAGE_BYTES = L::STAGE_BYTES;
    static constexpr int EPI_BUF = OUT == OUT_F32 ? 4096 : (OUT == OUT_BF16 ? 2048 : 0);   // 32 rows x 32 cols
    // epilogue warps: 8 (two per TMEM lane quarter) for bf16 / FP32 output;
    // the NVFP4 output (activation and quantization per element, no staging
    // buffers) takes warpgroup 1 as well: 12, three per lane quarter
    static constexpr int EPI_WARPS = OUT == OUT_NVFP4 ? 12 : kEpiWarps;
    static constexpr int EPI_WARP0 = kThreads / 32 - EPI_WARPS;
    static constexpr int EPI_PARTS = EPI_WARPS / 4;               // column parts per lane quarter
    static constexpr int EPI_BYTES = EPI_WARPS * 2 * EPI_BUF;
    static constexpr int FIT = (kSmemLimit - 1024 - EPI_BYTES) / STAGE_BYTES;
    static constexpr int MAX_STAGES = BN == 192 ? 6 : 5;
    static constexpr int STAGES = FIT < MAX_STAGES ? FIT : MAX_STAGES;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024;
    // BN = 192: two accumulators and two scale slots; BN = 256: one
    // accumulator and a scale slot per stage
    static constexpr int ACC_BUFS = BN == 192 ? 2 : 1;
    static constexpr int SF_SLOTS = BN == 192 ? 2 : STAGES;
    // who copies the scale atoms into TMEM: with a slot per stage, a separate
    // copier warp; with two slots, the MMA warp itself, right before the
    // stage's MMAs (tcgen05 copies and MMAs issued by one thread execute in
    // issue order, so a copy into a slot cannot overtake the MMAs that read it
    // two stages earlier, and no barrier round trip sits between stages)
    static constexpr bool COPY_IN_MMA = SF_SLOTS < STAGES;
    static constexpr int EPI_COLS = (BN / EPI_PARTS + 31) / 32 * 32;   // accumulator columns per epilogue warp
    // register split (setmaxnreg): warpgroup 0 (producer, MMA, copier) drops to
    // REGS_LOW, the epilogue warpgroups rise to REGS_HIGH
    static constexpr int REGS_LOW = Regs<BN>::LOW;
    static constexpr int REGS_HIGH =
        EPI_WARPS == kEpiWarps ? Regs<BN>::HIGH : (kThreads * 128 - 128 * REGS_LOW) / (32 * EPI_WARPS) / 8 * 8;
    static_assert((kThreads - 32 * EPI_WARPS) * REGS_LOW + 32 * EPI_WARPS * REGS_HIGH <= kThreads * 128,
                  "register split exceeds the launch budget");
    static_assert(STAGES >= 3, "pipeline depth");
    static_assert(ACC_BUFS * BN + SF_SLOTS * L::SF_COLS_STAGE <= 512, "TMEM columns");
    static_assert(EPI_COLS % 32 == 0, "epilogue chunks of 32 columns");
};

struct PairProblem {
    const float* a_scale;
    const float* b_scale;
    int M, N, K;
    int num_mb2, num_nb, first_tile;
    uint8_t* y_codes;
    uint8_t* y_sf;
    const float* y_scale;
    float* y_amax;
};

// Up to G independent problems sharing one tile space (G = 1: a plain call):
// per problem its tensor maps (A, B, A scales, B scales, Y) and sizes; its
// tiles are numbered from first_tile on.  Every role walks the same tile
// sequence and finds a tile's problem by comparing with the first tiles.
template <int G>
struct alignas(64) PairGroup {
    CUtensorMap map[G][5];
    PairProblem prob[G];
    int count, num_tiles;
    int* dev_status;
};

template <int G>
__device__ __forceinline__ int problem_of(const PairGroup<G>& g, int t) {
    int pi = 0;
#pragma unroll
    for (int i = 1; i < G; ++i)
        if (i < g.count && t >= g.prob[i].first_tile) pi = i;
    return pi;
}

__device__ __forceinline__ void tile_coords(int t, int num_mb2, int num_nb, int& mb2, int& nb) {
    const int per_group = kGroupM * num_nb;
    const int group = t / per_group;
    const int first = group * kGroupM;
    const int gm = min(kGroupM, num_mb2 - first);
    const int idx = t - group * per_group;
    mb2 = first + idx % gm;
    nb = idx / gm;
}

// Store 32 FP32 accumulator columns (alpha applied) of one row per lane
// through a swizzled staging buffer and a TMA store of a 32 x 32 box.
template <int OUT, int ACT>
__device__ __forceinline__ void store_chunk(const uint32_t* r, float alpha, uint8_t* buf, int lane,
                                            const CUtensorMap* map, int x, int y, uint64_t policy) {
    if (OUT == OUT_BF16) {
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            __nv_bfloat162 h = __floats2bfloat162_rn(epi_value<ACT>(alpha, r[2 * j]), epi_value<ACT>(alpha, r[2 * j + 1]));
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
            *reinterpret_cast<float4*>(buf + lane * 128 + pos * 16) =
                make_float4(epi_value<ACT>(alpha, r[4 * j]), epi_value<ACT>(alpha, r[4 * j + 1]),
                            epi_value<ACT>(alpha, r[4 * j + 2]), epi_value<ACT>(alpha, r[4 * j + 3]));
        }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d_hint(map, buf, x, y, policy);
        bulk_commit_group();
    }
}

// Fold a warp's running maximum of |y| into a problem's y_amax (nullable) and
// start a new one.  Non-negative floats order like their bit patterns.
__device__ __forceinline__ void flush_amax(float& amax_run, float* y_amax, int lane) {
    for (int o = 16; o > 0; o >>= 1) amax_run = fmaxf(amax_run, __shfl_xor_sync(0xffffffffu, amax_run, o));
    if (y_amax != nullptr && lane == 0 && amax_run > 0.0f)
        atomicMax(reinterpret_cast<int*>(y_amax), __float_as_int(amax_run));
    amax_run = 0.0f;
}

// Scale atom `at` of a stage of the pair (A: 128 rows of this CTA, B: the
// tile's two 128-row atom blocks, in both CTAs) into the atom's TMEM columns.
template <int BN, bool MXS>
__device__ __forceinline__ void k_copy_scales(uint32_t sfs, uint32_t sf_col, int at) {
    using L = Lay<BN, MXS>;
    const uint32_t col = sf_col + at * SF_COLS_ATOM;
    tc_cp2_32x128b_warpx4(col, sdesc_sf(sfs + at * SF_ATOM));
    tc_cp2_32x128b_warpx4(col + 4, sdesc_sf(sfs + L::SFA_BYTES + at * SF_ATOM));
    tc_cp2_32x128b_warpx4(col + 8, sdesc_sf(sfs + L::SFA_BYTES + L::SF_PER * SF_ATOM + at * SF_ATOM));
}

// One K=64 step of the pair: the block-scaled MMA reading the step's scale
// columns (MX: the atom of steps 2i and 2i + 1, bytes 0-1 or 2-3 of each row's
// scale word).  One TMEM column holds the scales of 32 B rows, so a tile
// whose first B row lies `sfb_off` * 32 rows into its first atom block reads
// B scales from `sfb_off` columns further on.
template <int BN, bool MXS>
__device__ __forceinline__ void k_mma(uint32_t tmem_acc, uint32_t sb, uint32_t sf_col, uint32_t sfb_off, int ks,
                                      uint32_t idesc, bool accumulate) {
    const uint64_t ad = sdesc_kmajor_sw128(sb + ks * 32), bd = sdesc_kmajor_sw128(sb + A_BYTES + ks * 32);
    if (MXS) {
        const uint32_t col = sf_col + (ks >> 1) * SF_COLS_ATOM, byte = (uint32_t)(ks & 1) * 2u;
        tc_mma2_mxf4(tmem_acc, ad, bd, idesc | (byte << 29) | (byte << 4), col | (byte << 30),
                     (col + 4 + sfb_off) | (byte << 30), accumulate ? 1u : 0u);
    } else {
        const uint32_t col = sf_col + ks * SF_COLS_ATOM;
        tc_mma2_nvf4(tmem_acc, ad, bd, idesc, col, col + 4 + sfb_off, accumulate ? 1u : 0u);
    }
}

template <int G, int BN, int OUT, int ACT, bool MXS>
__global__ void __launch_bounds__(kThreads, 1)
gemm2_kernel(const __grid_constant__ PairGroup<G> g) {
    using C = Cfg<BN, OUT, MXS>;
    using L = Lay<BN, MXS>;
    constexpr int STAGES = C::STAGES;
    constexpr int STAGE_BYTES = L::STAGE_BYTES;
    constexpr int ACC_BUFS = C::ACC_BUFS;
    constexpr int SF_SLOTS = C::SF_SLOTS;
    constexpr int EPI_COLS = C::EPI_COLS;
    extern __shared__ uint8_t smem_raw[];
    // full:   the leader's; both CTAs' operand tiles and scale atoms of a stage
    //         have landed (the peer's loads signal it through cta_group::2);
    // scaled: the leader's; the stage's scale atoms are in both CTAs' TMEM;
    // empty:  both CTAs'; the MMAs of a stage have completed;
    // accf:   both CTAs'; an accumulator holds a finished tile;
    // acce:   the leader's; both CTAs' epilogues have read an accumulator.
    __shared__ __align__(8) uint64_t full_bar[STAGES], scaled_bar[STAGES], empty_bar[STAGES];
    __shared__ __align__(8) uint64_t accf_bar[ACC_BUFS], acce_bar[ACC_BUFS], drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = (int)cluster_id_x();
    const int npairs = (int)nclusters_x();
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    WaitCtx wc{&abort_sh, g.dev_status};

    if (threadIdx.x == 0) {
        abort_sh = 0;
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&scaled_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < ACC_BUFS; ++b) {
            mbar_init(&accf_bar[b], 1);
            mbar_init(&acce_bar[b], 2 * C::EPI_WARPS);
        }
        mbar_init(&drain_bar, 1);
        fence_barrier_init();
        for (int i = 0; i < g.count; ++i)
            for (int m = 0; m < 5; ++m) tma_prefetch_desc(&g.map[i][m]);
    }
    // scale regions start as zeros (finite) so rows that are never loaded
    // (beyond M or N) multiply zero codes by a finite scale
    for (int s = 0; s < STAGES; ++s) {
        uint32_t* z = reinterpret_cast<uint32_t*>(smem + s * STAGE_BYTES + A_BYTES + L::B_BYTES);
        for (int i = threadIdx.x; i < (L::SFA_BYTES + L::SFB_BYTES) / 4; i += kThreads) z[i] = 0u;
    }
    fence_proxy_async_smem();
    cluster_sync_all();                       // barriers initialised in both CTAs
    if (warp == 0) {
        tmem_alloc2(&tmem_base_sh, 512);
        tmem_relinquish2();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;

    const uint32_t sf_base = tmem_base + ACC_BUFS * BN;
    // one register-budget change per warpgroup, before the roles diverge
    // (the epilogue code sits under the same branch as its increase, so that
    // ptxas allocates it against the raised budget)
    if (warp < C::EPI_WARP0) {
        if (warp < 4 || C::EPI_WARP0 == 8) regs_dec<C::REGS_LOW>();   // whole warpgroups: 0 (and 1)
        if (warp == 0) {
            // ------------------------------------------------------------ producer (both CTAs)
            const uint64_t pol_a = policy_evict_normal();
            const uint64_t pol_b = policy_evict_last();
            int stage = 0;
            uint32_t phase = 0, issued = 0, issued_any = 0;
            bool ok = true;
            for (int t = pair; t < g.num_tiles && ok; t += npairs) {
                const int pi = problem_of(g, t);
                const PairProblem& P = g.prob[pi];
                const CUtensorMap* maps = g.map[pi];
                const int num_kt = (P.K + 255) / 256, k_atoms = P.K / L::K_ATOM;
                int mb2, nb;
                tile_coords(t - P.first_tile, P.num_mb2, P.num_nb, mb2, nb);
                const int arow = mb2 * 256 + (int)rank * 128;
                const int brow = nb * BN + (int)rank * L::B_ROWS;
                const int sfa_row = (mb2 * 2 + (int)rank) * k_atoms;
                const int sfb_blk = (nb * BN) >> 7;          // first 128-row atom block of the tile's B rows
                const int sfb_row0 = sfb_blk * k_atoms, sfb_row1 = (sfb_blk + 1) * k_atoms;
                for (int kt = 0; kt < num_kt; ++kt) {
                    if (!__all_sync(0xffffffffu, mbar_wait(&empty_bar[stage], phase ^ 1u, wc) ? 1 : 0)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sb = smem + stage * STAGE_BYTES;
                    if (elect_one()) {
                        // every load of the pair completes on the leader's barrier,
                        // which the leader arms with the bytes of both CTAs
                        if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * STAGE_BYTES);
                        const uint32_t fb = mapa_shared(smem_u32(&full_bar[stage]), 0);
                        uint8_t* sfs = sb + A_BYTES + L::B_BYTES;
                        tma_load_2d_pair(sfs, &maps[2], fb, 0, sfa_row + kt * L::SF_PER, pol_a);
                        tma_load_2d_pair(sfs + L::SFA_BYTES, &maps[3], fb, 0, sfb_row0 + kt * L::SF_PER, pol_b);
                        tma_load_2d_pair(sfs + L::SFA_BYTES + L::SF_PER * SF_ATOM, &maps[3], fb, 0,
                                         sfb_row1 + kt * L::SF_PER, pol_b);
                        tma_load_2d_pair(sb, &maps[0], fb, kt * BK_BYTES, arow, pol_a);
                        tma_load_2d_pair(sb + A_BYTES, &maps[1], fb, kt * BK_BYTES, brow, pol_b);
                    }
                    __syncwarp();
                    issued = (issued & ~(1u << stage)) | (phase << stage);
                    issued_any |= 1u << stage;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            // loads in flight land before the CTAs may exit; the leader sees both
            // CTAs' loads complete and the peer is held at the final cluster
            // barrier until then
            if (lane == 0 && rank == 0) {
                int no_abort = 0;
                WaitCtx w2{&no_abort, g.dev_status};
                for (int s = 0; s < STAGES; ++s)
                    if (issued_any & (1u << s)) mbar_wait(&full_bar[s], (issued >> s) & 1u, w2);
            }
        } else if (warp == 2) {
            if (rank == 0 && !C::COPY_IN_MMA) {
                // -------------------------------------------------------- scale copier (leader)
                // Per stage: wait for the operands (and, with fewer scale slots
                // than stages, for the MMAs that last read the slot), copy the
                // stage's scale atoms of both CTAs into the slot, commit to the
                // stage's "scaled" barrier.  (From the MMA warp the twelve copies
                // per stage cost issue slots that the four MMAs need: ~626 cycles
                // per stage against ~533.)
                const uint32_t smem0 = smem_u32(smem);
                // ring positions: this stage (stage, phase), its scale slot, and
                // the stage SF_SLOTS back, whose MMAs last read that slot
                int stage = 0, slot = 0, wstage = 0;
                uint32_t phase = 0, wphase = 0, done = 0;
                bool ok = true;
                for (int t = pair; t < g.num_tiles && ok; t += npairs) {
                    const PairProblem& P = g.prob[problem_of(g, t)];
                    const int num_kt = (P.K + 255) / 256, k_atoms = P.K / L::K_ATOM;
                    for (int kt = 0; kt < num_kt; ++kt) {
                        bool got = mbar_wait(&full_bar[stage], phase, wc);
                        if (SF_SLOTS < STAGES && done >= (uint32_t)SF_SLOTS && got) {
                            // that stage's barrier cannot have moved on since: its
                            // next completion needs this stage's MMAs
                            got = mbar_wait(&empty_bar[wstage], wphase, wc);
                        }
                        if (!__all_sync(0xffffffffu, got ? 1 : 0)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t sfs = smem0 + stage * STAGE_BYTES + A_BYTES + L::B_BYTES;
                        const uint32_t sf_col = sf_base + slot * L::SF_COLS_STAGE;
                        const int nat = k_atoms - kt * L::SF_PER;
                        if (elect_one()) {
                            if (nat >= L::SF_PER) {
#pragma unroll
                                for (int at = 0; at < L::SF_PER; ++at) k_copy_scales<BN, MXS>(sfs, sf_col, at);
                            } else {
                                for (int at = 0; at < nat; ++at) k_copy_scales<BN, MXS>(sfs, sf_col, at);
                            }
                            tc_commit2_mc(&scaled_bar[stage], 0x1);
                        }
                        __syncwarp();
                        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                        if (++slot == SF_SLOTS) slot = 0;
                        if (++done > (uint32_t)SF_SLOTS) {
                            if (++wstage == STAGES) { wstage = 0; wphase ^= 1u; }
                        }
                    }
                }
            }
        } else if (warp == 1) {
            if (rank == 0) {
                // -------------------------------------------------------- MMA issuer (leader)
                // The whole warp runs the loop so that descriptors and addresses
                // stay warp-uniform; one elected lane issues four MMAs per stage.
                constexpr uint32_t idesc = MXS ? idesc_mxf4(256, BN) : idesc_nvf4(256, BN);
                const uint32_t smem0 = smem_u32(smem);
                int stage = 0, slot = 0, buf = 0;
                uint32_t phase = 0, acc_phase = 0;
                bool ok = true;
                for (int t = pair; t < g.num_tiles && ok; t += npairs) {
                    const PairProblem& P = g.prob[problem_of(g, t)];
                    const int num_kt = (P.K + 255) / 256, k_atoms = P.K / L::K_ATOM, k_steps = P.K / 64;
                    (void)k_atoms;
                    int mb2, nb;
                    tile_coords(t - P.first_tile, P.num_mb2, P.num_nb, mb2, nb);
                    const uint32_t sfb_off = (uint32_t)(((nb * BN) & 127) >> 5);
                    // the accumulator's previous tile has been read out by both epilogues
                    if (!__all_sync(0xffffffffu, mbar_wait_cluster(&acce_bar[buf], acc_phase ^ 1u, wc) ? 1 : 0)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t tmem_acc = tmem_base + buf * BN;
                    for (int kt = 0; kt < num_kt; ++kt) {
                        // operands landed (and, from the copier, the stage's scales are in TMEM)
                        uint64_t* ready = C::COPY_IN_MMA ? &full_bar[stage] : &scaled_bar[stage];
                        if (!__all_sync(0xffffffffu, mbar_wait(ready, phase, wc) ? 1 : 0)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t sb = smem0 + stage * STAGE_BYTES;
                        const uint32_t sf_col = sf_base + slot * L::SF_COLS_STAGE;
                        const int nks = k_steps - kt * 4;
                        if (C::COPY_IN_MMA && elect_one()) {
                            const uint32_t sfs = sb + A_BYTES + L::B_BYTES;
                            const int nat = k_atoms - kt * L::SF_PER;
                            if (nat >= L::SF_PER) {
#pragma unroll
                                for (int at = 0; at < L::SF_PER; ++at) k_copy_scales<BN, MXS>(sfs, sf_col, at);
                            } else {
                                for (int at = 0; at < nat; ++at) k_copy_scales<BN, MXS>(sfs, sf_col, at);
                            }
                        }
                        if (elect_one()) {
                            if (nks >= 4) {
#pragma unroll
                                for (int ks = 0; ks < 4; ++ks)
                                    k_mma<BN, MXS>(tmem_acc, sb, sf_col, sfb_off, ks, idesc, (kt | ks) != 0);
                            } else {
                                for (int ks = 0; ks < nks; ++ks)
                                    k_mma<BN, MXS>(tmem_acc, sb, sf_col, sfb_off, ks, idesc, (kt | ks) != 0);
                            }
                            tc_commit2_mc(&empty_bar[stage], 0x3);
                        }
                        __syncwarp();
                        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                        if (++slot == SF_SLOTS) slot = 0;
                    }
                    if (!ok) break;
                    if (elect_one()) tc_commit2_mc(&accf_bar[buf], 0x3);
                    __syncwarp();
                    if (++buf == ACC_BUFS) { buf = 0; acc_phase ^= 1u; }
                }
                if (elect_one()) tc_commit2_mc(&drain_bar, 0x1);
                __syncwarp();
                int no_abort = 0;
                WaitCtx w2{&no_abort, g.dev_status};
                mbar_wait(&drain_bar, 0, w2);
            }
        }
    } else {
        regs_inc<C::REGS_HIGH>();
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;                       // TMEM lane quarter
        const int h = (warp - C::EPI_WARP0) >> 2;     // column part: [h EPI_COLS, (h + 1) EPI_COLS) of BN
        const int row_t = (int)rank * 128 + q * 32 + lane;    // row inside the pair tile
        // per-problem constants, refreshed when the tile sequence enters
        // another problem (MX operands have no tensor scale: a null scale
        // reads as 1)
        int cur = -1;
        float alpha = 0.0f, g_y = 0.0f;
        ScaleConsts sc_y = scale_consts(0.0f);
        uint8_t* ebuf = smem + STAGES * STAGE_BYTES + (warp - C::EPI_WARP0) * 2 * C::EPI_BUF;
        // the output is written once and not read again by this kernel: evict
        // it from L2 first, so that its write-back to DRAM happens while the
        // tensor cores run rather than in whatever kernel comes next
        const uint64_t pol_y = policy_evict_first();
        int nstore = 0, buf = 0;
        uint32_t acc_phase = 0;
        float amax_run = 0.0f;
        for (int t = pair; t < g.num_tiles; t += npairs) {
            const int pi = problem_of(g, t);
            const PairProblem& P = g.prob[pi];
            if (pi != cur) {
                if (OUT == OUT_NVFP4 && cur >= 0) flush_amax(amax_run, g.prob[cur].y_amax, lane);
                cur = pi;
                alpha = __fmul_rn(P.a_scale ? *P.a_scale : 1.0f, P.b_scale ? *P.b_scale : 1.0f);
                if (OUT == OUT_NVFP4) {
                    g_y = *P.y_scale;
                    sc_y = scale_consts(g_y);
                }
            }
            int mb2, nb;
            tile_coords(t - P.first_tile, P.num_mb2, P.num_nb, mb2, nb);
            if (!__all_sync(0xffffffffu, mbar_wait(&accf_bar[buf], acc_phase, wc) ? 1 : 0)) break;
            tc_fence_after();
            uint32_t r[EPI_COLS];
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + buf * BN + h * EPI_COLS;
#pragma unroll
            for (int c = 0; c < EPI_COLS / 32; ++c)
                if (h * EPI_COLS + c * 32 < BN)           // the last part can be narrower
                    tmem_ld_32x32b_x32(tbase + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
            tmem_ld_wait();
            // the accumulator is in registers: hand TMEM back to the MMA issuer
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (rank == 0)
                    mbar_arrive(&acce_bar[buf]);
                else
                    mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(&acce_bar[buf]), 0));
            }
            if (++buf == ACC_BUFS) { buf = 0; acc_phase ^= 1u; }

            const int m0 = mb2 * 256 + (int)rank * 128 + q * 32;
            const int n0 = nb * BN + h * EPI_COLS;
            if (OUT == OUT_NVFP4) {
                // 32 columns (two 16-value blocks) at a time: 16 bytes of codes
                // and two scale bytes (half a scale word) per row
                const int64_t grow = (int64_t)mb2 * 256 + row_t;
                const int kb4 = P.N / 64;
#pragma unroll
                for (int c = 0; c < EPI_COLS / 32; ++c) {
                    const int ncol = n0 + c * 32;
                    if (ncol >= P.N || h * EPI_COLS + c * 32 >= BN) continue;
                    uint32_t sfh = 0u, cw[4];
#pragma unroll
                    for (int b = 0; b < 2; ++b) {
                        float v[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) v[j] = epi_value<ACT>(alpha, r[c * 32 + b * 16 + j]);
                        float ab = 0.0f;
#pragma unroll
                        for (int j = 0; j < 16; ++j) ab = fmaxf(ab, fabsf(v[j]));
                        if (grow < P.M) amax_run = fmaxf(amax_run, ab);
                        const uint32_t sfc = block_scale_code(ab, sc_y);
                        const float s = __fmul_rn(e4m3_to_f32(sfc), g_y);
                        float lo[8], hi[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) { lo[j] = v[j]; hi[j] = v[8 + j]; }
                        cw[2 * b] = quantize8(lo, s);
                        cw[2 * b + 1] = quantize8(hi, s);
                        sfh |= sfc << (8 * b);
                    }
                    if (grow < P.M)
                        *reinterpret_cast<uint4*>(P.y_codes + grow * (P.N / 2) + ncol / 2) =
                            make_uint4(cw[0], cw[1], cw[2], cw[3]);
                    // rows past M inside the padded scale buffer get zero scales
                    if (grow < (int64_t)((P.M + 127) / 128) * 128) {
                        const int rb = (int)(grow >> 7), rr = (int)(grow & 127);
                        const int64_t atom = (int64_t)rb * kb4 + ncol / 64;
                        *reinterpret_cast<uint16_t*>(P.y_sf + atom * SF_ATOM + (rr & 31) * 16 + (rr >> 5) * 4 +
                                                     ((ncol >> 4) & 3)) = (uint16_t)sfh;
                    }
                }
            } else {
#pragma unroll
                for (int c = 0; c < EPI_COLS / 32; ++c) {
                    if (n0 + c * 32 >= P.N || h * EPI_COLS + c * 32 >= BN) continue;
                    uint8_t* buf_s = ebuf + (nstore & 1) * C::EPI_BUF;
                    if (lane == 0) bulk_wait_group_read<1>();
                    __syncwarp();
                    store_chunk<OUT, ACT>(&r[c * 32], alpha, buf_s, lane, &g.map[pi][4], n0 + c * 32, m0, pol_y);
                    ++nstore;
                }
            }
        }
        if (lane == 0) bulk_wait_group<0>();
        if (OUT == OUT_NVFP4 && cur >= 0) flush_amax(amax_run, g.prob[cur].y_amax, lane);
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                       // the leader's MMAs are done with both CTAs' memory
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc2(tmem_base, 512);
    }
}

// Tensor maps of one problem: A and B codes, their scale atoms, and Y (bf16 or
// FP32; with the NVFP4 output the map is unused and a copy of A's is kept).
template <int BN, int OUT, bool MXS>
static bool encode_maps(const GemmW4A4Args& a, CUtensorMap (&m)[5]) {
    using L = Lay<BN, MXS>;
    const uint64_t kh = (uint64_t)(a.K / 2);
    const uint64_t atoms_a = (uint64_t)((a.M + 127) / 128) * (uint64_t)(a.K / L::K_ATOM);
    const uint64_t atoms_b = (uint64_t)((a.N + 127) / 128) * (uint64_t)(a.K / L::K_ATOM);
    if (make_tmap_2d(&m[0], a.a_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kh, (uint64_t)a.M, kh, BK_BYTES, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
        make_tmap_2d(&m[1], a.b_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kh, (uint64_t)a.N, kh, BK_BYTES, L::B_ROWS,
                     CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
        make_tmap_2d(&m[2], a.a_sf, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, 128, atoms_a, SF_ATOM, 128, L::SF_PER,
                     CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS ||
        make_tmap_2d(&m[3], a.b_sf, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, 128, atoms_b, SF_ATOM, 128, L::SF_PER,
                     CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
        return false;
    CUresult r = CUDA_SUCCESS;
    if (OUT == OUT_BF16)
        r = make_tmap_2d(&m[4], a.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.N, (uint64_t)a.M,
                         (uint64_t)a.N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
    else if (OUT == OUT_F32)
        r = make_tmap_2d(&m[4], a.y, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)a.N, (uint64_t)a.M,
                         (uint64_t)a.N * 4, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B);
    else
        m[4] = m[0];
    return r == CUDA_SUCCESS;
}

template <int G, int BN, int OUT, int ACT, bool MXS>
cudaError_t launch_out(const GemmW4A4Args* probs, int count, int num_sms, cudaStream_t stream) {
    using C = Cfg<BN, OUT, MXS>;
    if (count < 1 || count > G) return cudaErrorInvalidValue;
    PairGroup<G> g;
    int tiles = 0;
    for (int i = 0; i < count; ++i) {
        const GemmW4A4Args& a = probs[i];
        if (!encode_maps<BN, OUT, MXS>(a, g.map[i])) return cudaErrorInvalidValue;
        PairProblem& P = g.prob[i];
        P.a_scale = a.a_scale;
        P.b_scale = a.b_scale;
        P.M = (int)a.M;
        P.N = (int)a.N;
        P.K = (int)a.K;
        P.num_mb2 = (int)((a.M + 255) / 256);
        P.num_nb = (int)(a.N / BN);
        P.first_tile = tiles;
        P.y_codes = a.y_codes;
        P.y_sf = a.y_sf;
        P.y_scale = a.y_scale;
        P.y_amax = a.y_amax;
        tiles += P.num_mb2 * P.num_nb;
    }
    for (int i = count; i < G; ++i) {
        g.prob[i] = g.prob[0];
        g.prob[i].first_tile = tiles;            // never reached
        for (int m = 0; m < 5; ++m) g.map[i][m] = g.map[0][m];
    }
    g.count = count;
    g.num_tiles = tiles;
    g.dev_status = probs[0].dev_status;
    if (tiles == 0) return cudaSuccess;

    auto kern = gemm2_kernel<G, BN, OUT, ACT, MXS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // as many pairs as can be resident at once (persistent over tiles)
    int max_clusters = 0;
    cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
    if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg) != cudaSuccess || max_clusters < 1)
        max_clusters = num_sms / 2;
    const int pairs = tiles < max_clusters ? tiles : max_clusters;
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    e = cudaLaunchKernelEx(&cfg, kern, g);
    count_launch(1);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int G, int BN>
cudaError_t launch_bn(const GemmW4A4Args* probs, int count, int num_sms, cudaStream_t stream) {
    const GemmW4A4Args& a = probs[0];
    const bool gelu = a.act == ACT_GELU_TANH;
    if (a.mx) {
        // MX operands: bf16 or FP32 output (no NVFP4 output of an MX product),
        // plain calls only
        if (G != 1 || a.y == nullptr) return cudaErrorInvalidValue;
        if (a.y_dtype == 1)
            return gelu ? launch_out<1, BN, OUT_F32, ACT_GELU_TANH, true>(probs, count, num_sms, stream)
                        : launch_out<1, BN, OUT_F32, ACT_NONE, true>(probs, count, num_sms, stream);
        return gelu ? launch_out<1, BN, OUT_BF16, ACT_GELU_TANH, true>(probs, count, num_sms, stream)
                    : launch_out<1, BN, OUT_BF16, ACT_NONE, true>(probs, count, num_sms, stream);
    }
    if (a.y != nullptr) {
        if (a.y_dtype == 1)
            return gelu ? launch_out<G, BN, OUT_F32, ACT_GELU_TANH, false>(probs, count, num_sms, stream)
                        : launch_out<G, BN, OUT_F32, ACT_NONE, false>(probs, count, num_sms, stream);
        return gelu ? launch_out<G, BN, OUT_BF16, ACT_GELU_TANH, false>(probs, count, num_sms, stream)
                    : launch_out<G, BN, OUT_BF16, ACT_NONE, false>(probs, count, num_sms, stream);
    }
    return gelu ? launch_out<G, BN, OUT_NVFP4, ACT_GELU_TANH, false>(probs, count, num_sms, stream)
                : launch_out<G, BN, OUT_NVFP4, ACT_NONE, false>(probs, count, num_sms, stream);
}

}  // namespace w4a4_2sm

// The pair kernel's tile width for a set of problems: 256 when every N is a
// multiple of 256, else 192 when every N is a multiple of 192, else 0 (not
// supported).  A pair MMA (M = 256, K = 64) takes about 120 cycles whatever
// its N up to 192 and 128 at N = 256, so only the 256-wide tile runs the
// tensor cores at full rate.  NVFP4_PAIR_TILE_N (192 or 256) picks the width
// for measurements, where the shapes allow it.
int gemm_w4a4_2sm_tile_n(const GemmW4A4Args* probs, int count) {
    bool all256 = true, all192 = true;
    for (int i = 0; i < count; ++i) {
        all256 = all256 && probs[i].N % 256 == 0;
        all192 = all192 && probs[i].N % 192 == 0;
    }
    const char* env = getenv("NVFP4_PAIR_TILE_N");
    const int forced = env ? atoi(env) : 0;
    if (all256 && (forced != 192 || !all192)) return 256;
    if (all192) return 192;
    return 0;
}

cudaError_t launch_gemm_w4a4_2sm(const GemmW4A4Args& a, int num_sms, cudaStream_t stream) {
    using namespace w4a4_2sm;
    const int bn = gemm_w4a4_2sm_tile_n(&a, 1);
    if (bn == 256) return launch_bn<1, 256>(&a, 1, num_sms, stream);
    if (bn == 192) return launch_bn<1, 192>(&a, 1, num_sms, stream);
    return cudaErrorInvalidValue;
}

// Up to kPairGroup problems with one output kind and activation in one launch
// of the pair kernel (one tile space).
cudaError_t launch_gemm_w4a4_2sm_grouped(const GemmW4A4Args* probs, int count, int num_sms, cudaStream_t stream) {
    using namespace w4a4_2sm;
    const int bn = gemm_w4a4_2sm_tile_n(probs, count);
    if (bn == 256) return launch_bn<kPairGroup, 256>(probs, count, num_sms, stream);
    if (bn == 192) return launch_bn<kPairGroup, 192>(probs, count, num_sms, stream);
    return cudaErrorInvalidValue;
}

bool gemm_w4a4_2sm_supports(int64_t N) { return N % 192 == 0 || N % 256 == 0; }

}  // namespace nvfp4
