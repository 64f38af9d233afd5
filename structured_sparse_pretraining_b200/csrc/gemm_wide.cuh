// gemm_wide.cuh -- the 2:4 sparse products (forward and input gradient) for
// long reduction dimensions, on pairs of SMs with two row blocks per CTA.
//
// Why a second kernel.  A pair tile of sp_pair_kernel (256 rows x BN tokens)
// consumes ~46 KB of operands per CTA for every 448 cycles of sparse MMA at
// BN = 224, about 103 B/clk.  The operand ring can hold 4 such stages
// (184 KB).  A stage returns to the producer only after its MMAs have
// completed, the release has reached the producer, the refill has come back
// from L2 and the consumer has woken: measured on B200 at about 2k cycles
// without the load and 3-4k with it.  Four stages hide about 1.8k cycles at
// that rate, so the tensor pipe idles about half the time.  Here each CTA
// holds two 128-row blocks of the sparse operand against the same token rows:
// a pair tile is 512 rows x 224 tokens, a k-tile is 2 x 4 sparse MMAs (896
// cycles) for 60 KB per CTA, about 69 B/clk, and three stages hide ~2.6k
// cycles (measured: 80% of the MMA rate with L2-resident operands against
// 57% for one block).  The price is a single accumulator per block (2 x 224
// TMEM columns, next to a 64-column code ring): the epilogue of a tile is
// not hidden behind the next tile's mainloop, except that each block is
// released as soon as it is drained, so the next tile's first MMAs on
// block 0 overlap the draining of block 1.  The planner takes this kernel
// for reduction dimensions long enough that the epilogue is a small part.
//
// Roles (352 threads), as in sp_pair_kernel: warp 0 operand producer, warp 1
// TMEM owner and (pair leader) MMA issuer, warps 2..5 epilogue, warps 6..9
// code writers, warp 10 code-tile producer.  Position codes: one 2 KB code
// tile per block and k-tile, brought by TMA, rearranged in place into the
// TMEM lane image by the writers and copied into TMEM by tcgen05.cp (see
// gemm_pair.cuh).  The rank-r adapter runs as dense MMAs through the operand
// ring after the sparse k-tiles of each tile.  No TMA multicast.
//
// Fused rank product (p.tok_units > 0).  The adapter's down-projection
// (XL = X . L before the forward, G = dY . R^T before the input gradient) is
// computed by the same launch: the first tok_units work units each multiply
// 256 token rows (128 per CTA, as the MMA's M) by the rank factor over the
// whole reduction dimension into the accumulator of block 0, and the epilogue
// writes the bf16 rows and publishes them with a release add on the unit's
// flag.  These units come first in every pair's work list and wait on
// nothing, and the launch is fully resident, so a tile whose adapter phase
// needs them (its producer waits on the flags of the units covering its
// tokens before loading XL or G) can always proceed.  The last CTA to finish
// resets the flags for the next launch.  With fewer units than SM pairs, each
// unit is split into tok_split pieces over consecutive ranges of the
// reduction (so that the units' work is spread over more pairs instead of
// adding a whole unit to the makespan of a few): a piece writes its fp32
// partial rows to a workspace slot and counts itself in per (unit, CTA,
// warp); the warp that arrives last sums the slots in piece order (the same
// order whichever arrives last), writes the bf16 rows and publishes them.
#pragma once
#include <cstdint>
#include "gemm_pair.cuh"

namespace slope {

struct WideCfg {
    static constexpr int BN = 224, BNH = 112;    // token columns of a pair tile / rows held per CTA
    static constexpr int NBLK = 2;               // 256-row blocks per pair tile (128 rows per CTA each)
    static constexpr int TILE_M = 256 * NBLK;
    static constexpr int A_BYTES = 16384;        // one block: 128 rows x 64 stored values (128 logical K)
    static constexpr int B_PANEL = BNH * 128;    // BNH rows x 64 K, 128-byte swizzle
    static constexpr int B_BYTES = 2 * B_PANEL;
    static constexpr int STAGE_BYTES = NBLK * A_BYTES + B_BYTES;
    static constexpr int NS = 3;
    static constexpr int E_BYTES = 2048;         // one block's code tile: 128 rows x 16 bytes
    static constexpr int ESLOT_BYTES = NBLK * E_BYTES;
    static constexpr int NE = 8;                 // code slots (k-tiles), 4 TMEM columns per block each
    static constexpr int CB = 4;                 // slots handed over per batch
    static constexpr int STAGING_BYTES = 4 * 2048;
    static constexpr int META_COL = NBLK * BN;   // 448
    static constexpr int TMEM_COLS = 512;
    static constexpr int BAR_BYTES = 512;
    static constexpr int SMEM_BYTES = NS * STAGE_BYTES + NE * ESLOT_BYTES + STAGING_BYTES + BAR_BYTES + 1024;
    static_assert(META_COL + 4 * NBLK * NE <= TMEM_COLS, "TMEM budget");
    static_assert(NE % CB == 0, "code batches");
    static_assert(BAR_BYTES >= 8 * (2 * NS + NE + 2 * (NE / CB) + 1 + NBLK) + 8, "barrier area");
    static_assert(STAGE_BYTES % 1024 == 0 && B_PANEL % 1024 == 0 && ESLOT_BYTES % 1024 == 0, "alignment");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Unit w of the wide kernel: its 512-row m tile and token tile (grouped order).
__device__ __forceinline__ void wide_unit(const GemmParams &p, int w, int &mt, int &nt) {
    grouped_tile(w, p.num_m_tiles, p.num_n_tiles, p.raster_g, mt, nt);
}

// Rank-product item w (< tok_items): its unit u, piece h and range of
// 64-wide k-slices [k0, k1) (every piece non-empty: tok_split <= tok_k_tiles).
__device__ __forceinline__ void tok_piece(const GemmParams &p, int w, int &u, int &h, int &k0, int &k1) {
    u = w / p.tok_split;
    h = w % p.tok_split;
    const int per = (p.tok_k_tiles + p.tok_split - 1) / p.tok_split;
    k0 = h * per;
    k1 = min(p.tok_k_tiles, k0 + per);
}

template <bool A2_MN>
__global__ void __launch_bounds__(352, 1)
    sp_wide_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                   const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmTA,
                   const __grid_constant__ CUtensorMap tmTB, const __grid_constant__ GemmParams p) {
    using C = WideCfg;
    constexpr int NS = C::NS, NE = C::NE, CB = C::CB, NBAT = NE / CB, BN = C::BN, BNH = C::BNH, NBLK = C::NBLK;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ering = smem + NS * C::STAGE_BYTES;
    uint8_t *staging = ering + NE * C::ESLOT_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(staging + C::STAGING_BYTES);  // leader: both CTAs' bytes
    uint64_t *empty = full + NS;          // each CTA: stage s may be refilled
    uint64_t *efull = empty + NS;         // each CTA: both raw code tiles of slot e are in shared memory
    uint64_t *eempty = efull + NE;        // each CTA: code batch b may be refilled
    uint64_t *mfull = eempty + NBAT;      // leader: both CTAs' lane images of batch b are ready (8 arrivals)
    uint64_t *acc_full = mfull + NBAT;    // each CTA: the tile's accumulators are complete
    uint64_t *acc_empty = acc_full + 1;   // leader, per block: both CTAs drained it (8 arrivals)
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(acc_empty + NBLK);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int e = 0; e < NE; ++e) mbar_init(&efull[e], 1);
        for (int b = 0; b < NBAT; ++b) {
            mbar_init(&eempty[b], 1);
            mbar_init(&mfull[b], 8);
        }
        mbar_init(acc_full, 1);
        for (int b = 0; b < NBLK; ++b) mbar_init(&acc_empty[b], 8);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmE);
        if (p.r > 0) {
            tma_prefetch_desc(&tmA2);
            tma_prefetch_desc(&tmB2);
        }
        if (p.tok_units > 0) {
            tma_prefetch_desc(&tmTA);
            tma_prefetch_desc(&tmTB);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_holder, C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the peer's barriers are initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    grid_dep_wait();
    grid_dep_launch();
    int my_tiles = 0;  // sparse tiles (not rank-product units) in this pair's work list
    for (int w = pair; w < p.num_work; w += num_pairs) my_tiles += w >= p.tok_items ? 1 : 0;
    const int my_ktiles = my_tiles * p.k_tiles_total;

    if (warp == 0) {
        // ------------------------------------------------------------ operand producer (both CTAs)
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            for (int w = pair; w < p.num_work; w += num_pairs) {
                if (w < p.tok_items) {  // rank-product piece: 128 token rows of this CTA x the rank factor
                    // a stage holds tok_nsl k-slices of 64: token rows [128 x 64] (16 KB), then the factor's
                    // 64 K rows (MN-major L) or tok_bc rows of 64 K (K-major R)
                    int u, h, k0, k1;
                    tok_piece(p, w, u, h, k0, k1);
                    const int t0 = u * 256 + 128 * rank;
                    const uint32_t b_bytes = 128u * (uint32_t)p.tok_bc;
                    for (int kt0 = k0; kt0 < k1; kt0 += p.tok_nsl) {
                        const int nsl = min(p.tok_nsl, k1 - kt0);
                        if (!mbar_wait(&empty[s], ph ^ 1, abort_flag)) goto done;
                        const uint32_t lead_full = cluster_addr(&full[s], 0);
                        if (rank == 0) mbar_arrive_expect_tx(&full[s], 2u * (uint32_t)nsl * (C::A_BYTES + b_bytes));
                        for (int i = 0; i < nsl; ++i) {
                            uint8_t *a = smem + s * C::STAGE_BYTES + i * p.tok_slice_bytes;
                            const int kt = kt0 + i;
                            tma_load_2d_pair(a, &tmTA, lead_full, kt * 64, t0);
                            if (p.tok_b_mn) tma_load_2d_pair(a + C::A_BYTES, &tmTB, lead_full, (int)rank * p.tok_bc, kt * 64);
                            else tma_load_2d_pair(a + C::A_BYTES, &tmTB, lead_full, kt * 64, (int)rank * p.tok_bc);
                        }
                        if (++s == NS) { s = 0; ph ^= 1; }
                    }
                    continue;
                }
                int mt, nt;
                wide_unit(p, w - p.tok_items, mt, nt);
                const int m0 = mt * C::TILE_M + 128 * rank;  // this CTA's rows of block 0 (block 1: + 256)
                const int n0 = nt * BN + BNH * rank;         // this CTA's token rows of B
                for (int kt = 0; kt < p.k_tiles_total; ++kt) {
                    if (!mbar_wait(&empty[s], ph ^ 1, abort_flag)) goto done;
                    uint8_t *a = smem + s * C::STAGE_BYTES;
                    uint8_t *b = a + NBLK * C::A_BYTES;
                    const uint32_t lead_full = cluster_addr(&full[s], 0);
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * C::STAGE_BYTES);
#pragma unroll
                    for (int blk = 0; blk < NBLK; ++blk)
                        tma_load_2d_pair(a + blk * C::A_BYTES, &tmA, lead_full, kt * 64, m0 + 256 * blk);
                    tma_load_2d_pair(b, &tmB, lead_full, kt * 128, n0);
                    tma_load_2d_pair(b + C::B_PANEL, &tmB, lead_full, kt * 128 + 64, n0);
                    if (++s == NS) { s = 0; ph ^= 1; }
                }
                // adapter: A2 (R^T MN-major, or L K-major) for both blocks, B2 (XL or G) k-tiles of 64 rank
                if (p.tok_units > 0 && p.adp_k_tiles > 0) {
                    // B2 is this launch's own rank product: wait for the units covering the tile's tokens
                    const int u0 = (nt * BN) / 256, u1 = min(nt * BN + BN, p.N) - 1;
                    for (int u = u0; u <= u1 / 256; ++u)
                        if (in_bounds(u, 1, p.ext.tok_flags) && !flag_wait(p.tok_flags + u, 8, abort_flag)) goto done;
                    fence_proxy_async_global();
                }
                for (int kt = 0; kt < p.adp_k_tiles; ++kt) {
                    if (!mbar_wait(&empty[s], ph ^ 1, abort_flag)) goto done;
                    uint8_t *a = smem + s * C::STAGE_BYTES;
                    uint8_t *b = a + NBLK * C::A_BYTES;
                    const uint32_t lead_full = cluster_addr(&full[s], 0);
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * (NBLK * C::A_BYTES + C::B_PANEL));
#pragma unroll
                    for (int blk = 0; blk < NBLK; ++blk) {
                        uint8_t *ab = a + blk * C::A_BYTES;
                        if (A2_MN) {
                            tma_load_2d_pair(ab, &tmA2, lead_full, m0 + 256 * blk, kt * 64);
                            tma_load_2d_pair(ab + 8192, &tmA2, lead_full, m0 + 256 * blk + 64, kt * 64);
                        } else {
                            tma_load_2d_pair(ab, &tmA2, lead_full, kt * 64, m0 + 256 * blk);
                        }
                    }
                    tma_load_2d_pair(b, &tmB2, lead_full, kt * 64, n0);
                    if (++s == NS) { s = 0; ph ^= 1; }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader only)
        if (rank == 0 && lane == 0) {
            constexpr uint32_t IDESC_SP = instr_desc(256, BN, 0, 0, 1);
            constexpr uint32_t IDESC_AD = instr_desc(256, BN, A2_MN ? 1 : 0, 0, 0);
            const uint32_t base = smem_addr(smem);
            const uint64_t a_desc0 = smem_desc(base, 16, 1024, SWZ_128B);
            const uint64_t b_desc0 = smem_desc(base + NBLK * C::A_BYTES, 16, 1024, SWZ_128B);
            const uint64_t a2_desc0 = A2_MN ? smem_desc(base, 8192, 1024, SWZ_128B) : a_desc0;
            const uint64_t e_desc0 = smem_desc(smem_addr(ering), 128, 128, SWZ_NONE);
            const uint32_t e_col0 = tmem_base + C::META_COL;
            // rank-product units: A = token rows (K-major), B = L (MN-major) or R (K-major)
            const uint32_t tok_rowb = 2u * (uint32_t)p.tok_bc;  // bytes per K row of an MN-major B
            const uint64_t tb_desc0 =
                p.tok_b_mn ? smem_desc(base + C::A_BYTES, 8192, 8 * tok_rowb,
                                       tok_rowb == 32 ? SWZ_32B : tok_rowb == 64 ? SWZ_64B : SWZ_128B)
                           : smem_desc(base + C::A_BYTES, 16, 1024, SWZ_128B);
            const uint32_t IDESC_TOK = instr_desc(256, p.tok_n, 0, p.tok_b_mn, 0);
            int s = 0, e = 0, j = 0;   // j: main k-tiles consumed so far
            uint32_t ph = 0, bph = 0;  // bph: per-batch phase bits of mfull
            int fills[NBLK] = {0};     // times each block's accumulator was filled
            for (int w = pair; w < p.num_work; w += num_pairs) {
                if (w < p.tok_items) {  // the rank product into block 0's accumulator
                    int u, h, k0, k1;
                    tok_piece(p, w, u, h, k0, k1);
                    if (!mbar_wait(&acc_empty[0], (fills[0] & 1) ^ 1, abort_flag)) goto done;
                    tc_fence_after();
                    for (int kt0 = k0; kt0 < k1; kt0 += p.tok_nsl) {
                        const int nsl = min(p.tok_nsl, k1 - kt0);
                        if (!mbar_wait(&full[s], ph, abort_flag)) goto done;
                        tc_fence_after();
                        for (int i = 0; i < nsl; ++i) {
                            const uint32_t off = (uint32_t)(s * C::STAGE_BYTES + i * p.tok_slice_bytes) >> 4;
                            const uint64_t ad = a_desc0 + (uint64_t)off;
                            const uint64_t bd = tb_desc0 + (uint64_t)off;
#pragma unroll
                            for (int c = 0; c < 4; ++c)
                                mma_bf16_pair(tmem_base, ad + (uint64_t)(2 * c),
                                              bd + (uint64_t)(p.tok_b_mn ? tok_rowb * c : 2 * c), IDESC_TOK,
                                              (kt0 + i > k0 || c > 0) ? 1u : 0u);
                        }
                        mma_commit_pair_both(&empty[s]);
                        if (++s == NS) { s = 0; ph ^= 1; }
                    }
                    mma_commit_pair_both(acc_full);
                    ++fills[0];
                    continue;
                }
                // Lead-in of a tile: the first `lead` k-tiles run on block 0
                // alone (its accumulator is drained first), then the same
                // stages, still in shared memory, on block 1 once the epilogue
                // has drained it; the stages and the code batches are released
                // after both.  Block 1's draining thus overlaps `lead` k-tiles
                // of block-0 MMAs instead of one, at the price of a refill
                // bubble (all stages are held until block 1 has used them).
                // Measured on B200 (fused forward, one CUDA graph per call):
                // 2-7% faster from 32 k-tiles on (K >= 4096), 5% slower at 8
                // (K = 1024), no change at 6 and 24; so one k-tile (the plain
                // order) below 32.
                static_assert(NBLK == 2, "the lead-in is written for two blocks");
                const int lead = p.k_tiles_total >= 32 ? min(NS, p.k_tiles_total) : 1;
                int lead_s[NS], lead_e[NS];
                if (!mbar_wait(&acc_empty[0], (fills[0] & 1) ^ 1, abort_flag)) goto done;
                tc_fence_after();
                for (int kt = 0; kt < lead; ++kt) {
                    const int bb = e / CB;
                    if (e % CB == 0) {  // first slot of a batch: its lane images must be ready
                        if (!mbar_wait(&mfull[bb], (bph >> bb) & 1u, abort_flag)) goto done;
                        bph ^= 1u << bb;
                    }
                    if (!mbar_wait(&full[s], ph, abort_flag)) goto done;
                    tc_fence_after();
                    const uint32_t ecol = e_col0 + e * 4 * NBLK;
#pragma unroll
                    for (int blk = 0; blk < NBLK; ++blk)
                        tmem_cp_128x128b_pair(ecol + 4 * blk,
                                              e_desc0 + (uint64_t)((e * C::ESLOT_BYTES + blk * C::E_BYTES) >> 4));
                    const uint64_t bd = b_desc0 + (uint64_t)((s * C::STAGE_BYTES) >> 4);
                    const uint64_t ad = a_desc0 + (uint64_t)((s * C::STAGE_BYTES) >> 4);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        mma_sp_bf16_pair(tmem_base, ad + (uint64_t)(2 * c),
                                         bd + (uint64_t)(((c >> 1) * C::B_PANEL + (c & 1) * 64) >> 4), (ecol + c) & ~1u,
                                         IDESC_SP | ((ecol + c) & 1u), (kt > 0 || c > 0) ? 1u : 0u);
                    lead_s[kt] = s;
                    lead_e[kt] = e;
                    if (++s == NS) { s = 0; ph ^= 1; }
                    if (++e == NE) e = 0;
                }
                if (!mbar_wait(&acc_empty[1], (fills[1] & 1) ^ 1, abort_flag)) goto done;
                tc_fence_after();
                for (int kt = 0; kt < lead; ++kt, ++j) {
                    const int ls = lead_s[kt], le = lead_e[kt];
                    const uint32_t eb = e_col0 + le * 4 * NBLK + 4;
                    const uint64_t bd = b_desc0 + (uint64_t)((ls * C::STAGE_BYTES) >> 4);
                    const uint64_t ad = a_desc0 + (uint64_t)((ls * C::STAGE_BYTES + C::A_BYTES) >> 4);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        mma_sp_bf16_pair(tmem_base + BN, ad + (uint64_t)(2 * c),
                                         bd + (uint64_t)(((c >> 1) * C::B_PANEL + (c & 1) * 64) >> 4), (eb + c) & ~1u,
                                         IDESC_SP | ((eb + c) & 1u), (kt > 0 || c > 0) ? 1u : 0u);
                    mma_commit_pair_both(&empty[ls]);
                    if (le % CB == CB - 1 || j == my_ktiles - 1) mma_commit_pair_both(&eempty[le / CB]);
                }
                for (int kt = lead; kt < p.k_tiles_total; ++kt, ++j) {
                    const int bb = e / CB;
                    if (e % CB == 0) {  // first slot of a batch: its lane images must be ready
                        if (!mbar_wait(&mfull[bb], (bph >> bb) & 1u, abort_flag)) goto done;
                        bph ^= 1u << bb;
                    }
                    if (!mbar_wait(&full[s], ph, abort_flag)) goto done;
                    tc_fence_after();
                    const uint32_t ecol = e_col0 + e * 4 * NBLK;
#pragma unroll
                    for (int blk = 0; blk < NBLK; ++blk)
                        tmem_cp_128x128b_pair(ecol + 4 * blk,
                                              e_desc0 + (uint64_t)((e * C::ESLOT_BYTES + blk * C::E_BYTES) >> 4));
                    const uint64_t bd = b_desc0 + (uint64_t)((s * C::STAGE_BYTES) >> 4);
#pragma unroll
                    for (int blk = 0; blk < NBLK; ++blk) {
                        const uint32_t d = tmem_base + blk * BN;
                        const uint64_t ad = a_desc0 + (uint64_t)((s * C::STAGE_BYTES + blk * C::A_BYTES) >> 4);
                        const uint32_t eb = ecol + 4 * blk;
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            mma_sp_bf16_pair(d, ad + (uint64_t)(2 * c),
                                             bd + (uint64_t)(((c >> 1) * C::B_PANEL + (c & 1) * 64) >> 4), (eb + c) & ~1u,
                                             IDESC_SP | ((eb + c) & 1u), (kt > 0 || c > 0) ? 1u : 0u);
                    }
                    mma_commit_pair_both(&empty[s]);
                    if (e % CB == CB - 1 || j == my_ktiles - 1) mma_commit_pair_both(&eempty[bb]);
                    if (++s == NS) { s = 0; ph ^= 1; }
                    if (++e == NE) e = 0;
                }
                for (int kt = 0; kt < p.adp_k_tiles; ++kt) {
                    if (!mbar_wait(&full[s], ph, abort_flag)) goto done;
                    tc_fence_after();
                    const uint64_t bd = b_desc0 + (uint64_t)((s * C::STAGE_BYTES) >> 4);
                    const int nblk = min(4, (p.r - kt * 64 + 15) / 16);
#pragma unroll
                    for (int blk = 0; blk < NBLK; ++blk) {
                        const uint64_t ad = a2_desc0 + (uint64_t)((s * C::STAGE_BYTES + blk * C::A_BYTES) >> 4);
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            if (c < nblk)
                                mma_bf16_pair(tmem_base + blk * BN, ad + (uint64_t)(A2_MN ? 128 * c : 2 * c),
                                              bd + (uint64_t)(2 * c), IDESC_AD, 1u);
                    }
                    mma_commit_pair_both(&empty[s]);
                    if (++s == NS) { s = 0; ph ^= 1; }
                }
                mma_commit_pair_both(acc_full);
#pragma unroll
                for (int blk = 0; blk < NBLK; ++blk) ++fills[blk];
            }
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;
        uint8_t *tile = staging + q * 2048;  // [32 tokens][32 features] bf16
        const int seg = lane & 3;            // 16-byte segment of a token's 32 features
        const int rsub = lane >> 2;          // token row within a group of 8
        const int odd = lane & 1;
        uint16_t *out = reinterpret_cast<uint16_t *>(p.out);
        constexpr int NCH = BN / 32;  // 7 chunks of 32 token columns
        int it = 0;
        for (int w = pair; w < p.num_work; w += num_pairs) {
            if (!mbar_wait_warp(acc_full, it & 1, abort_flag)) break;
            tc_fence_after();
            ++it;
            if (w < p.tok_items) {
                // rank product: TMEM lane = token row, column = rank; bf16 rows of tok_r values
                int u, h, k0, k1;
                tok_piece(p, w, u, h, k0, k1);
                const int rloc = 128 * rank + 32 * q + lane;  // row within the unit
                const int row = u * 256 + rloc;
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
                uint16_t *dst = p.tok_out + (int64_t)row * p.tok_r;
                const bool piece = p.tok_split > 1;
                float *slot = p.tok_ws + (((int64_t)u * p.tok_split + h) * 256 + rloc) * p.tok_r;
                for (int c0 = 0; c0 < p.tok_r; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld_32x32(taddr + c0, v);
                    tmem_ld_wait();
                    if (piece) {  // this piece's fp32 partial row
#pragma unroll
                        for (int j4 = 0; j4 < 32; j4 += 4)
                            if (c0 + j4 < p.tok_r && in_buf(slot + c0 + j4, p.tok_ws, 4, p.ext.tok_ws))
                                *reinterpret_cast<uint4 *>(slot + c0 + j4) = make_uint4(v[j4], v[j4 + 1], v[j4 + 2], v[j4 + 3]);
                    } else if (row < p.N) {
#pragma unroll
                        for (int j8 = 0; j8 < 32; j8 += 8) {
                            if (c0 + j8 < p.tok_r && in_bounds((int64_t)row * p.tok_r + c0 + j8, 8, p.ext.tok_out)) {
                                uint32_t pk[4];
#pragma unroll
                                for (int u = 0; u < 4; ++u)
                                    pk[u] = static_cast<uint32_t>(f32_to_bf16_bits(bits_to_f32(v[j8 + 2 * u]))) |
                                            (static_cast<uint32_t>(f32_to_bf16_bits(bits_to_f32(v[j8 + 2 * u + 1]))) << 16);
                                *reinterpret_cast<uint4 *>(dst + c0 + j8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                            }
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (rank == 0) mbar_arrive(&acc_empty[0]);
                    else mbar_arrive_cluster(cluster_addr(&acc_empty[0], 0));
                }
                if (piece) {
                    // count this piece in; the last of the unit's pieces for these 32 rows sums them
                    __threadfence();
                    __syncwarp();
                    int last = 0;
                    if (lane == 0) {
                        int *cnt = p.tok_cnt + (int64_t)u * 8 + 4 * rank + q;
                        if (in_buf(cnt, p.tok_cnt, 1, p.ext.tok_cnt)) {
                            last = atomicAdd(cnt, 1) == p.tok_split - 1;
                            if (last) *cnt = 0;  // every piece has arrived: ready for the next launch
                        }
                    }
                    last = __shfl_sync(0xFFFFFFFFu, last, 0);
                    if (!last) continue;
                    __threadfence();
                    const float *base = p.tok_ws + ((int64_t)u * p.tok_split * 256 + rloc) * p.tok_r;
                    const int64_t pstride = (int64_t)256 * p.tok_r;  // one piece's slot to the next
                    if (row < p.N && in_buf(base + (int64_t)(p.tok_split - 1) * pstride, p.tok_ws, p.tok_r, p.ext.tok_ws)) {
                        for (int c0 = 0; c0 < p.tok_r; c0 += 8) {
                            float4 a0 = __ldcg(reinterpret_cast<const float4 *>(base + c0));
                            float4 a1 = __ldcg(reinterpret_cast<const float4 *>(base + c0 + 4));
                            for (int k = 1; k < p.tok_split; ++k) {  // in piece order
                                const float4 b0 = __ldcg(reinterpret_cast<const float4 *>(base + k * pstride + c0));
                                const float4 b1 = __ldcg(reinterpret_cast<const float4 *>(base + k * pstride + c0 + 4));
                                a0.x += b0.x; a0.y += b0.y; a0.z += b0.z; a0.w += b0.w;
                                a1.x += b1.x; a1.y += b1.y; a1.z += b1.z; a1.w += b1.w;
                            }
                            if (in_bounds((int64_t)row * p.tok_r + c0, 8, p.ext.tok_out)) {
                                const uint32_t w0 = static_cast<uint32_t>(f32_to_bf16_bits(a0.x)) |
                                                    (static_cast<uint32_t>(f32_to_bf16_bits(a0.y)) << 16);
                                const uint32_t w1 = static_cast<uint32_t>(f32_to_bf16_bits(a0.z)) |
                                                    (static_cast<uint32_t>(f32_to_bf16_bits(a0.w)) << 16);
                                const uint32_t w2 = static_cast<uint32_t>(f32_to_bf16_bits(a1.x)) |
                                                    (static_cast<uint32_t>(f32_to_bf16_bits(a1.y)) << 16);
                                const uint32_t w3 = static_cast<uint32_t>(f32_to_bf16_bits(a1.z)) |
                                                    (static_cast<uint32_t>(f32_to_bf16_bits(a1.w)) << 16);
                                *reinterpret_cast<uint4 *>(dst + c0) = make_uint4(w0, w1, w2, w3);
                            }
                        }
                    }
                }
                // publish the rows to the tiles of other CTAs, which read them by TMA
                fence_proxy_async_global();
                __threadfence();
                __syncwarp();
                if (lane == 0 && in_bounds(u, 1, p.ext.tok_flags)) red_release_gpu_add(p.tok_flags + u, 1);
                continue;
            }
            int mt, nt;
            wide_unit(p, w - p.tok_items, mt, nt);
            __syncwarp();  // the previous tile's reads of the staging tile are done
#pragma unroll 1
            for (int blk = 0; blk < NBLK; ++blk) {
                const int m0 = mt * C::TILE_M + 256 * blk + 128 * rank + 32 * q;  // first output feature of this warp
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + blk * BN;
                const bool m_ok = m0 + 8 * seg < p.M;  // M is a multiple of 8: a segment is all in or all out
                uint32_t v[2][32];
                tmem_ld_32x32(taddr, v[0]);
#pragma unroll
                for (int cc = 0; cc < NCH; ++cc) {
                    tmem_ld_wait();  // chunk cc has landed
                    if (cc + 1 < NCH) {
                        tmem_ld_32x32(taddr + 32 * (cc + 1), v[(cc + 1) & 1]);
                    } else {
                        // the block is drained: the next tile's MMAs on it may start
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            if (rank == 0) mbar_arrive(&acc_empty[blk]);
                            else mbar_arrive_cluster(cluster_addr(&acc_empty[blk], 0));
                        }
                    }
                    // transpose to [token][feature] two tokens at a time (see sp_pair_kernel)
#pragma unroll
                    for (int jj = 0; jj < 32; jj += 2) {
                        const float mine_lo = bits_to_f32(v[cc & 1][jj]), mine_hi = bits_to_f32(v[cc & 1][jj + 1]);
                        const float other = __shfl_xor_sync(0xffffffffu, odd ? mine_lo : mine_hi, 1);
                        const __nv_bfloat162 pr = odd ? __floats2bfloat162_rn(other, mine_hi) : __floats2bfloat162_rn(mine_lo, other);
                        *reinterpret_cast<__nv_bfloat162 *>(tile + ((jj + odd) * 32 + (lane & ~1)) * 2) = pr;
                    }
                    __syncwarp();
                    const int n0 = nt * BN + 32 * cc;
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int r = 8 * g + rsub;
                        const uint4 val = *reinterpret_cast<const uint4 *>(tile + (r * 32 + seg * 8) * 2);
                        if (m_ok && n0 + r < p.N && in_bounds((int64_t)(n0 + r) * p.ld_out + m0 + seg * 8, 8, p.ext.out))
                            *reinterpret_cast<uint4 *>(out + (int64_t)(n0 + r) * p.ld_out + m0 + seg * 8) = val;
                    }
                    __syncwarp();  // every lane has read the tile before the next chunk overwrites it
                }
            }
        }
    } else if (warp < 10) {
        // ------------------------------------------------------------ code writers (both CTAs)
        // The lane image of each block's code tile, built in place (see sp_pair_kernel).
        const int q = warp & 3;
        const int L = 32 * q + lane;
        const int mm = 16 * (L >> 4) + (L & 7);
        const int h = (L >> 3) & 1;
        int e = 0, j = 0;
        uint32_t eph = 0;
        for (int w = pair; w < p.num_work; w += num_pairs) {
            if (w < p.tok_items) continue;
            int mt, nt;
            wide_unit(p, w - p.tok_items, mt, nt);
            for (int kt = 0; kt < p.k_tiles_total; ++kt, ++j) {
                if (!mbar_wait_warp(&efull[e], eph, abort_flag)) goto done;
#pragma unroll
                for (int blk = 0; blk < NBLK; ++blk) {
                    uint8_t *et = ering + e * C::ESLOT_BYTES + blk * C::E_BYTES;
                    const int rowA = mt * C::TILE_M + 256 * blk + 128 * rank + mm;
                    const uint4 va = *reinterpret_cast<const uint4 *>(et + mm * 16);
                    const uint4 vb = *reinterpret_cast<const uint4 *>(et + (mm + 8) * 16);
                    uint32_t ca[4] = {va.x, va.y, va.z, va.w}, cb[4] = {vb.x, vb.y, vb.z, vb.w};
                    const uint32_t fill = 0x44444444u;  // rows past M: positions 0, 1 of zero-filled values
                    if (rowA >= p.M) ca[0] = ca[1] = ca[2] = ca[3] = fill;
                    if (rowA + 8 >= p.M) cb[0] = cb[1] = cb[2] = cb[3] = fill;
                    uint4 img;
                    img.x = word16(ca, 0 + h) | (word16(cb, 0 + h) << 16);
                    img.y = word16(ca, 2 + h) | (word16(cb, 2 + h) << 16);
                    img.z = word16(ca, 4 + h) | (word16(cb, 4 + h) << 16);
                    img.w = word16(ca, 6 + h) | (word16(cb, 6 + h) << 16);
                    __syncwarp();  // this warp's 32 image rows come from its own 32 raw rows: all read
                    *reinterpret_cast<uint4 *>(et + L * 16) = img;
                }
                fence_proxy_async_smem();  // visible to tcgen05.cp
                if (e % CB == CB - 1 || j == my_ktiles - 1) {  // batch complete: publish it to the MMA issuer
                    __syncwarp();
                    if (lane == 0) {
                        if (rank == 0) mbar_arrive(&mfull[e / CB]);
                        else mbar_arrive_cluster(cluster_addr(&mfull[e / CB], 0));
                    }
                }
                if (++e == NE) { e = 0; eph ^= 1; }
            }
        }
    } else {
        // ------------------------------------------------------------ code-tile producer (both CTAs)
        if (lane == 0) {
            int e = 0;
            uint32_t bph = 0;
            for (int w = pair; w < p.num_work; w += num_pairs) {
                if (w < p.tok_items) continue;
                int mt, nt;
                wide_unit(p, w - p.tok_items, mt, nt);
                const int m0 = mt * C::TILE_M + 128 * rank;
                for (int kt = 0; kt < p.k_tiles_total; ++kt) {
                    if (e % CB == 0) {
                        const int bb = e / CB;
                        if (!mbar_wait(&eempty[bb], ((bph >> bb) & 1u) ^ 1u, abort_flag)) goto done;
                        bph ^= 1u << bb;
                    }
                    mbar_arrive_expect_tx(&efull[e], C::ESLOT_BYTES);
#pragma unroll
                    for (int blk = 0; blk < NBLK; ++blk)
                        tma_load_2d(ering + e * C::ESLOT_BYTES + blk * C::E_BYTES, &tmE, &efull[e], kt * 8, m0 + 256 * blk);
                    if (++e == NE) e = 0;
                }
            }
        }
    }
done:
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // neither CTA leaves while its peer may still signal it
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
    if (p.tok_units > 0 && threadIdx.x == 0 && in_bounds(0, p.tok_units + 1, p.ext.tok_flags)) {
        // every role of this CTA is done with the flags; the last CTA resets them
        __threadfence();
        if (atomicAdd(p.tok_flags + p.tok_units, 1) == (int)gridDim.x - 1) {
            for (int u = 0; u < p.tok_units; ++u) p.tok_flags[u] = 0;
            p.tok_flags[p.tok_units] = 0;
            __threadfence();
        }
    }
}

}  // namespace slope
