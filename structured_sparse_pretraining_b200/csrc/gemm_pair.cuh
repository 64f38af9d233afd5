// gemm_pair.cuh -- the 2:4 sparse products (forward and input gradient) on
// pairs of SMs: tcgen05 with cta_group::2.
//
// A cluster of two CTAs computes one 256 x BN output tile.  CTA r of the pair
// holds A rows [128 r, 128 r + 128) of the tile (compressed values + position
// codes) and token rows [BN/2 r, BN/2 r + BN/2) of B; the pair leader (rank 0)
// issues tcgen05.mma.sp.cta_group::2, which reads A and B from both CTAs'
// shared memory and writes each CTA's 128 accumulator rows into its own TMEM.
// Per SM this halves the operand bytes one MMA needs compared with a 1-SM
// 128 x BN tile, which is what a 2:4 sparse MMA (twice the dense rate) needs
// to be fed from L2.
//
// Roles per CTA: see sp_pair_kernel below.
// Synchronisation across the pair goes through the leader's barriers, named
// by their shared::cluster address; MMA completion is signalled to both CTAs
// by one tcgen05.commit with a CTA mask (two separate commits per k-tile cost
// the tensor pipe about 20 cycles each).  No TMA multicast is used.
#pragma once
#include <cstdint>
#include "gemm.cuh"
#include "ptx.cuh"

namespace slope {

// Eight consecutive 16-bit code words of one row of A (words w0..w0+7),
// returned as four 32-bit pairs.  Words past the row, and rows past M, read
// as 0x4444 (positions 0 and 1: a legal pattern whose values are zero-filled).
__device__ __forceinline__ void load_codes8(const uint16_t *meta, int row, int M, int words_per_row, int w0,
                                            uint32_t (&out)[4], int64_t extent) {
    const uint32_t fill = 0x44444444u;
    out[0] = out[1] = out[2] = out[3] = fill;
    if (row >= M) return;
    const uint16_t *base = meta + (int64_t)row * words_per_row + w0;
    if (!in_bounds((int64_t)row * words_per_row + w0, min(8, words_per_row - w0), extent)) return;
    const uint2 lo = *reinterpret_cast<const uint2 *>(base);
    out[0] = lo.x;
    out[1] = lo.y;
    if (w0 + 8 <= words_per_row) {
        const uint2 hi = *reinterpret_cast<const uint2 *>(base + 4);
        out[2] = hi.x;
        out[3] = hi.y;
    }
}

__device__ __forceinline__ uint32_t word16(const uint32_t (&w)[4], int k) {
    return (w[k >> 1] >> (16 * (k & 1))) & 0xFFFFu;
}

template <int BN>
struct PairCfg {
    static constexpr int BNH = BN / 2;          // token rows of B held by each CTA
    static constexpr int A_BYTES = 16384;       // 128 rows x 64 stored values (128 logical K)
    static constexpr int B_PANEL = BNH * 128;   // BNH rows x 64 K, 128-byte swizzle
    static constexpr int B_BYTES = 2 * B_PANEL;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int E_BYTES = 2048;        // code tile: 128 rows x 16 bytes
    // Depth of the code ring: as deep as TMEM allows (4 columns per slot next
    // to two BN-column accumulators).  A shallow ring starves the MMA: a code
    // tile passes TMA, the writers and a hand-over before the MMA can use it.
    static constexpr int NE = 2 * BN + 48 <= 512 ? 12 : 8;
    static constexpr int CB = 4;                // code slots handed over per batch
    static constexpr int STAGING_BYTES = 4 * 2048;  // epilogue: one 32 x 32 bf16 transpose tile per warp
    // adapter tile of rank <= 32 (padded to 16 or 32): A2 128 x 32 and B2 BNH x 32 bf16
    static constexpr int ADP_A_BYTES = 8192;
    static constexpr int ADP_BYTES = ADP_A_BYTES + 8192;
    static constexpr int NS_RAW = (225 * 1024 - NE * E_BYTES - STAGING_BYTES - ADP_BYTES) / STAGE_BYTES;
    static constexpr int NS = NS_RAW > 8 ? 8 : NS_RAW;
    static constexpr int META_COL = 2 * BN;     // TMEM columns of the code ring: 4 per slot
    static constexpr int TMEM_COLS = 512;
    static constexpr int BAR_BYTES = 1024;
    static constexpr int SMEM_BYTES = NS * STAGE_BYTES + NE * E_BYTES + STAGING_BYTES + ADP_BYTES + BAR_BYTES + 1024;
    static_assert(BAR_BYTES >= 8 * (2 * 8 + NE + 2 * (NE / CB) + 6) + 8, "barrier area");
    static_assert(BNH * 64 <= ADP_BYTES - ADP_A_BYTES, "adapter buffer");
    static_assert(NE % CB == 0, "code batches");
    static_assert(2 * BN + 4 * NE <= TMEM_COLS, "TMEM budget");
    static_assert(B_PANEL % 1024 == 0 && STAGE_BYTES % 1024 == 0, "swizzle-atom alignment");
    static_assert(BN % 16 == 0 && BNH % 8 == 0 && BN <= 256, "tile shape");
    static_assert(NS >= 3, "pipeline depth");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Roles per CTA (352 threads): warp 0 operand producer, warp 1 TMEM owner and
// (pair leader) MMA issuer, warps 2..5 epilogue, warps 6..9 code writers,
// warp 10 code-tile producer.
//
// Position codes.  tcgen05.mma.sp reads them from TMEM: for M = 128 rows per
// CTA, one 32-bit column per MMA of 32 logical K, row m / k-half h in lane
// (m % 8) + 8 h + 16 (m / 16), bits 16 ((m / 8) % 2) .. +15, so each lane packs
// rows m and m + 8.  A code tile (128 rows x 8 code words = 128 logical K) is
// brought to shared memory by TMA, rearranged there in place into that lane
// image (16 bytes per lane) by the code writers, and copied into TMEM by the
// MMA thread with tcgen05.cp, which runs in the tensor pipe in order with the
// MMAs.  (A tcgen05.st of the codes by other warps, the alternative, completes
// only after the MMAs queued ahead of it, and so drains the pipe.)  The code
// ring has NE slots of shared memory and 4 TMEM columns each; slots move
// between roles in batches of CB.
//
// Epilogue.  The accumulator lane is an output feature and the column a token,
// while the output is token-major: each warp transposes 32 x 32 tiles through
// shared memory and writes whole 64-byte row segments with plain stores.
// Epilogue of a product split over K (kept out of line: the unsplit path's
// code stays as it is).  The warp's 32 features x BN tokens of fp32 partial
// sums go to its split's workspace slot ([token][lane], coalesced); it then
// releases the accumulator and counts itself in on the counter of (tile, CTA,
// warp).  The last of the splits to arrive sums all slots in split order (the
// same order whichever arrives last), rounds once to bf16 and writes the tile
// through the staging tile like the unsplit path.
template <int BN>
__device__ __noinline__ void pair_split_epilogue(uint32_t taddr, uint8_t *tile, int lane, bool m_ok, int m0, int nt,
                                                 int sp, int64_t unit, uint64_t *acc_empty, uint32_t rank,
                                                 const GemmParams &p) {
    constexpr int NCH = (BN + 31) / 32;
    float *slots = p.ws + unit * p.num_splits * (BN * 32);
    uint32_t v[32];
#pragma unroll 1
    for (int cc = 0; cc < NCH; ++cc) {
        const int ncols = (BN % 32 != 0 && cc == NCH - 1) ? 16 : 32;
        if (ncols == 16) tmem_ld_32x32_x16(taddr + 32 * cc, v);
        else tmem_ld_32x32(taddr + 32 * cc, v);
        tmem_ld_wait();
        float *dst = slots + (int64_t)sp * (BN * 32) + 32 * 32 * cc + lane;
#pragma unroll
        for (int jj = 0; jj < 32; ++jj)
            if (jj < ncols && in_buf(dst + 32 * jj, p.ws, 1, p.ext.ws)) __stcg(dst + 32 * jj, bits_to_f32(v[jj]));
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {  // the accumulator is drained: release it to the pair leader's MMA issuer
        if (rank == 0) mbar_arrive(acc_empty);
        else mbar_arrive_cluster(cluster_addr(acc_empty, 0));
    }
    __threadfence();
    __syncwarp();
    int last = 0;
    if (lane == 0 && in_bounds(unit, 1, p.ext.ws_count)) {
        int *cnt = p.ws_count + unit;
        last = atomicAdd(cnt, 1) == p.num_splits - 1;
        if (last) *cnt = 0;  // every split has arrived: ready for the next launch
    }
    last = __shfl_sync(0xFFFFFFFFu, last, 0);
    if (!last) return;
    if (!in_buf(slots, p.ws, (int64_t)p.num_splits * (BN * 32), p.ext.ws)) return;
    __threadfence();
    const int odd = lane & 1;
    const int seg = lane & 3;    // 16-byte segment of a token's 32 features
    const int rsub = lane >> 2;  // token row within a group of 8
    uint16_t *out = reinterpret_cast<uint16_t *>(p.out);
#pragma unroll 1
    for (int cc = 0; cc < NCH; ++cc) {
        const int ncols = (BN % 32 != 0 && cc == NCH - 1) ? 16 : 32;
        // splits outermost: each pass has its 32 (16) loads in flight at once
        const float *src = slots + 32 * 32 * cc + lane;
        float a[32];
#pragma unroll
        for (int jj = 0; jj < 32; ++jj)
            if (jj < ncols) a[jj] = __ldcg(src + 32 * jj);
        int k = 1;
#pragma unroll 1
        for (; k + 2 <= p.num_splits; k += 2) {  // two slots' loads in flight per pass
            float t[2][32];
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int jj = 0; jj < 32; ++jj)
                    if (jj < ncols) t[u][jj] = __ldcg(src + (int64_t)(k + u) * (BN * 32) + 32 * jj);
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int jj = 0; jj < 32; ++jj)
                    if (jj < ncols) a[jj] += t[u][jj];
        }
        if (k < p.num_splits) {
#pragma unroll
            for (int jj = 0; jj < 32; ++jj)
                if (jj < ncols) a[jj] += __ldcg(src + (int64_t)k * (BN * 32) + 32 * jj);
        }
#pragma unroll
        for (int jj = 0; jj < 32; ++jj)
            if (jj < ncols) v[jj] = __float_as_uint(a[jj]);
        // transpose through the staging tile (see the unsplit path)
#pragma unroll
        for (int jj = 0; jj < 32; jj += 2) {
            if (jj < ncols) {
                const float mine_lo = bits_to_f32(v[jj]), mine_hi = bits_to_f32(v[jj + 1]);
                const float other = __shfl_xor_sync(0xffffffffu, odd ? mine_lo : mine_hi, 1);
                const __nv_bfloat162 pr = odd ? __floats2bfloat162_rn(other, mine_hi) : __floats2bfloat162_rn(mine_lo, other);
                *reinterpret_cast<__nv_bfloat162 *>(tile + ((jj + odd) * 32 + (lane & ~1)) * 2) = pr;
            }
        }
        __syncwarp();
        const int n0 = nt * BN + 32 * cc;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const int r = 8 * g + rsub;
            if (r < ncols) {
                const uint4 val = *reinterpret_cast<const uint4 *>(tile + (r * 32 + seg * 8) * 2);
                if (m_ok && n0 + r < p.N && in_bounds((int64_t)(n0 + r) * p.ld_out + m0 + seg * 8, 8, p.ext.out))
                    *reinterpret_cast<uint4 *>(out + (int64_t)(n0 + r) * p.ld_out + m0 + seg * 8) = val;
            }
        }
        __syncwarp();
    }
}

// Work unit w of the pair kernel: its m tile, n tile, split and k-tile range.
// Without SPLIT (a launch with one split) the unit is a whole tile, computed
// without the split bookkeeping.
template <bool SPLIT>
__device__ __forceinline__ void pair_unit(const GemmParams &p, int w, int &mt, int &nt, int &sp, int &k0, int &k1) {
    if (SPLIT) {
        decode_work(p, w, mt, nt, sp);
        k_range(p, sp, k0, k1);
    } else {
        mt = w % p.num_m_tiles;
        nt = w / p.num_m_tiles;
        sp = 0;
        k0 = 0;
        k1 = p.k_tiles_total;
    }
}

template <bool A2_MN, int BN, bool SPLIT>
__global__ void __launch_bounds__(352, 1)
    sp_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                   const __grid_constant__ CUtensorMap tmE, const __grid_constant__ GemmParams p) {
    using C = PairCfg<BN>;
    constexpr int NS = C::NS;
    constexpr int NE = C::NE;
    constexpr int CB = C::CB;
    constexpr int NB = NE / CB;  // batches in the code ring
    constexpr int BNH = C::BNH;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ering = smem + NS * C::STAGE_BYTES;
    uint8_t *staging = ering + NE * C::E_BYTES;
    uint8_t *adp = staging + C::STAGING_BYTES;  // adapter tile (rank <= 32): A2 at 0, B2 at ADP_A_BYTES
    uint64_t *full = reinterpret_cast<uint64_t *>(adp + C::ADP_BYTES);  // leader: A,B bytes of both CTAs
    uint64_t *empty = full + NS;        // each CTA: operand stage s may be refilled
    uint64_t *efull = empty + NS;       // each CTA: raw code tile of slot e is in shared memory
    uint64_t *eempty = efull + NE;      // each CTA: code batch b (shared memory + TMEM) may be refilled
    uint64_t *mfull = eempty + NB;      // leader: both CTAs' lane images of batch b are ready (8 arrivals)
    uint64_t *acc_full = mfull + NB;    // each CTA: accumulator ready
    uint64_t *acc_empty = acc_full + 2;  // leader: both CTAs drained the accumulator (8 arrivals)
    uint64_t *adp_full = acc_empty + 2;  // leader: both CTAs' adapter tiles are in shared memory
    uint64_t *adp_empty = adp_full + 1;  // each CTA: the adapter buffer may be refilled
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(adp_empty + 1);
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
        for (int bb = 0; bb < NB; ++bb) {
            mbar_init(&eempty[bb], 1);
            mbar_init(&mfull[bb], 8);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 8);
        }
        mbar_init(adp_full, 1);
        mbar_init(adp_empty, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (p.r > 0) {
            tma_prefetch_desc(&tmA2);
            tma_prefetch_desc(&tmB2);
        }
        if (p.meta_tma) tma_prefetch_desc(&tmE);
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
    // total main k-tiles of this pair's work list (both CTAs count the same)
    int my_ktiles = 0;
    for (int w = pair; w < p.num_work; w += num_pairs) {
        int mt, nt, sp, k0, k1;
        pair_unit<SPLIT>(p, w, mt, nt, sp, k0, k1);
        my_ktiles += k1 - k0;
    }

    if (warp == 0) {
        // ------------------------------------------------------------ operand producer (both CTAs)
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            for (int w = pair; w < p.num_work; w += num_pairs) {
                int mt, nt, sp, k0, k1;
                pair_unit<SPLIT>(p, w, mt, nt, sp, k0, k1);
                const int m0 = mt * 256 + 128 * rank;  // this CTA's A rows
                const int n0 = nt * BN + BNH * rank;   // this CTA's token rows of B
                for (int kt = k0; kt < k1; ++kt) {
                    if (!mbar_wait(&empty[s], ph ^ 1, abort_flag)) goto done;
                    uint8_t *a = smem + s * C::STAGE_BYTES;
                    uint8_t *b = a + C::A_BYTES;
                    const uint32_t lead_full = cluster_addr(&full[s], 0);
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * C::STAGE_BYTES);
                    tma_load_2d_pair(a, &tmA, lead_full, kt * 64, m0);
                    tma_load_2d_pair(b, &tmB, lead_full, kt * 128, n0);
                    tma_load_2d_pair(b + C::B_PANEL, &tmB, lead_full, kt * 128 + 64, n0);
                    if (++s == NS) { s = 0; ph ^= 1; }
                }
                const int adp_kt = sp == 0 ? p.adp_k_tiles : 0;  // the adapter term goes with split 0
                for (int kt = 0; kt < adp_kt; ++kt) {
                    if (!mbar_wait(&empty[s], ph ^ 1, abort_flag)) goto done;
                    uint8_t *a = smem + s * C::STAGE_BYTES;
                    uint8_t *b = a + C::A_BYTES;
                    const uint32_t lead_full = cluster_addr(&full[s], 0);
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * (C::A_BYTES + C::B_PANEL));
                    if (A2_MN) {
                        tma_load_2d_pair(a, &tmA2, lead_full, m0, kt * 64);
                        tma_load_2d_pair(a + 8192, &tmA2, lead_full, m0 + 64, kt * 64);
                    } else {
                        tma_load_2d_pair(a, &tmA2, lead_full, kt * 64, m0);
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
            // Descriptors of stage 0 and code slot 0; a stage, a slot or a
            // k-block only adds a constant to the start-address field.
            const uint32_t base = smem_addr(smem);
            const uint64_t a_desc0 = smem_desc(base, 16, 1024, SWZ_128B);
            const uint64_t b_desc0 = smem_desc(base + C::A_BYTES, 16, 1024, SWZ_128B);
            const uint64_t a2_desc0 = A2_MN ? smem_desc(base, 8192, 1024, SWZ_128B) : a_desc0;
            const uint64_t b2_desc0 = b_desc0;
            // lane image: 128 rows of 16 bytes, no swizzle (both strides one 8-row core matrix)
            const uint64_t e_desc0 = smem_desc(smem_addr(ering), 128, 128, SWZ_NONE);
            const uint32_t e_col0 = tmem_base + C::META_COL;
            // adapter buffer (rank <= 32, padded to rp): A2 MN-major in panels of
            // 64 features x rp rows, or K-major 128 rows x rp; B2 K-major BNH x rp.
            // K-major rows of 2 rp bytes use the matching 32- or 64-byte swizzle.
            const int rp = p.adp_buf;
            const uint32_t kswz = rp == 16 ? SWZ_32B : SWZ_64B;
            const uint32_t abase = smem_addr(adp);
            const uint64_t a3_desc = A2_MN ? smem_desc(abase, (uint32_t)rp * 128u, 1024, SWZ_128B)
                                           : smem_desc(abase, 16, (uint32_t)rp * 16u, kswz);
            const uint64_t b3_desc = smem_desc(abase + C::ADP_A_BYTES, 16, (uint32_t)rp * 16u, kswz);
            int s = 0, e = 0, j = 0;   // j: main k-tiles consumed so far
            uint32_t ph = 0, bph = 0;  // bph: per-batch phase bits of mfull
            uint32_t aph = 0;          // phase of adp_full
            int it = 0;
            for (int w = pair; w < p.num_work; w += num_pairs) {
                int mt, nt, sp, k0, k1;
                pair_unit<SPLIT>(p, w, mt, nt, sp, k0, k1);
                const int acc = it & 1;
                const uint32_t acc_ph = (it >> 1) & 1;
                if (!mbar_wait(&acc_empty[acc], acc_ph ^ 1, abort_flag)) goto done;
                tc_fence_after();
                const uint32_t d = tmem_base + acc * BN;
                uint32_t accumulate = 0;
                if (rp > 0 && sp == 0) {
                    // adapter first: its buffer is then free for the next tile
                    // while this tile's sparse k-tiles run
                    if (!mbar_wait(adp_full, aph, abort_flag)) goto done;
                    aph ^= 1;
                    tc_fence_after();
                    for (int c = 0; c < rp / 16; ++c)
                        mma_bf16_pair(d, a3_desc + (uint64_t)(A2_MN ? 128 * c : 2 * c), b3_desc + (uint64_t)(2 * c),
                                      IDESC_AD, (uint32_t)c);
                    accumulate = 1;
                    mma_commit_pair_both(adp_empty);
                }
                for (int kt = k0; kt < k1; ++kt, ++j) {
                    const int bb = e / CB;
                    if (e % CB == 0) {  // first slot of a batch: its lane images must be ready
                        if (!mbar_wait(&mfull[bb], (bph >> bb) & 1u, abort_flag)) goto done;
                        bph ^= 1u << bb;
                    }
                    if (!mbar_wait(&full[s], ph, abort_flag)) goto done;
                    tc_fence_after();
                    const uint32_t ecol = e_col0 + e * 4;
                    tmem_cp_128x128b_pair(ecol, e_desc0 + (uint64_t)((e * C::E_BYTES) >> 4));
                    const uint64_t ad = a_desc0 + (uint64_t)((s * C::STAGE_BYTES) >> 4);
                    const uint64_t bd = b_desc0 + (uint64_t)((s * C::STAGE_BYTES) >> 4);
                    const int nblk = min(4, (p.k_logical - kt * 128) / 32);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        if (c < nblk) {
                            mma_sp_bf16_pair(d, ad + (uint64_t)(2 * c), bd + (uint64_t)(((c >> 1) * C::B_PANEL + (c & 1) * 64) >> 4),
                                             (ecol + c) & ~1u, IDESC_SP | ((ecol + c) & 1u), accumulate | (uint32_t)c);
                        }
                    }
                    accumulate = 1;
                    mma_commit_pair_both(&empty[s]);
                    if (e % CB == CB - 1 || j == my_ktiles - 1) {  // last slot of a batch: release the batch
                        mma_commit_pair_both(&eempty[bb]);
                    }
                    if (++s == NS) { s = 0; ph ^= 1; }
                    if (++e == NE) e = 0;
                }
                const int adp_kt = sp == 0 ? p.adp_k_tiles : 0;
                for (int kt = 0; kt < adp_kt; ++kt) {
                    if (!mbar_wait(&full[s], ph, abort_flag)) goto done;
                    tc_fence_after();
                    const uint64_t ad = a2_desc0 + (uint64_t)((s * C::STAGE_BYTES) >> 4);
                    const uint64_t bd = b2_desc0 + (uint64_t)((s * C::STAGE_BYTES) >> 4);
                    const int nblk = min(4, (p.r - kt * 64 + 15) / 16);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        if (c < nblk) {
                            mma_bf16_pair(d, ad + (uint64_t)(A2_MN ? 128 * c : 2 * c), bd + (uint64_t)(2 * c), IDESC_AD,
                                          accumulate | (uint32_t)c);
                        }
                    }
                    accumulate = 1;
                    mma_commit_pair_both(&empty[s]);
                    if (++s == NS) { s = 0; ph ^= 1; }
                }
                mma_commit_pair_both(&acc_full[acc]);
                ++it;
            }
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;
        uint8_t *tile = staging + q * 2048;  // [32 tokens][32 features] bf16
        const int seg = lane & 3;      // 16-byte segment of a token's 32 features
        const int rsub = lane >> 2;    // token row within a group of 8
        int it = 0;
        for (int w = pair; w < p.num_work; w += num_pairs) {
            int mt, nt, sp, k0, k1;
            pair_unit<SPLIT>(p, w, mt, nt, sp, k0, k1);
            const int acc = it & 1;
            const uint32_t acc_ph = (it >> 1) & 1;
            if (!mbar_wait_warp(&acc_full[acc], acc_ph, abort_flag)) break;
            tc_fence_after();
            const int m0 = mt * 256 + 128 * rank + 32 * q;  // first output feature of this warp
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + acc * BN;
            const bool m_ok = m0 + 8 * seg < p.M;  // M is a multiple of 8: a segment is all in or all out
            __syncwarp();  // the previous tile's reads of the staging tile are done
            if (SPLIT && p.num_splits > 1) {
                const int64_t unit = ((int64_t)(mt + p.num_m_tiles * nt) * 2 + rank) * 4 + q;
                pair_split_epilogue<BN>(taddr, tile, lane, m_ok, m0, nt, sp, unit, &acc_empty[acc], rank, p);
                ++it;
                continue;
            }
            uint16_t *out = reinterpret_cast<uint16_t *>(p.out);
            // Chunks of 32 token columns (a BN with BN % 32 == 16 ends with a
            // 16-column chunk).  The loop is unrolled: the TMEM load of chunk
            // cc + 1 is in flight while chunk cc is transposed and stored.
            constexpr int NCH = (BN + 31) / 32;
            uint32_t v[2][32];
            if (NCH == 1 && BN % 32 != 0) tmem_ld_32x32_x16(taddr, v[0]);
            else tmem_ld_32x32(taddr, v[0]);
#pragma unroll
            for (int cc = 0; cc < NCH; ++cc) {
                const int ncols = (BN % 32 != 0 && cc == NCH - 1) ? 16 : 32;
                tmem_ld_wait();  // chunk cc (and every earlier load) has landed
                if (cc + 1 < NCH) {
                    if (BN % 32 != 0 && cc + 1 == NCH - 1) tmem_ld_32x32_x16(taddr + 32 * (cc + 1), v[(cc + 1) & 1]);
                    else tmem_ld_32x32(taddr + 32 * (cc + 1), v[(cc + 1) & 1]);
                } else {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        if (rank == 0) mbar_arrive(&acc_empty[acc]);
                        else mbar_arrive_cluster(cluster_addr(&acc_empty[acc], 0));
                    }
                }
                // v[jj] = D[feature m0 + lane][token n0 + jj].  Transpose to
                // [token][feature] two tokens at a time: neighbouring lanes swap
                // one value so that each writes two adjacent features of one
                // token as a bf16 pair (even lane: token jj, odd lane: jj + 1).
                const int odd = lane & 1;
#pragma unroll
                for (int jj = 0; jj < 32; jj += 2) {
                    if (jj < ncols) {
                        const float mine_lo = bits_to_f32(v[cc & 1][jj]), mine_hi = bits_to_f32(v[cc & 1][jj + 1]);
                        const float other = __shfl_xor_sync(0xffffffffu, odd ? mine_lo : mine_hi, 1);
                        const __nv_bfloat162 pr = odd ? __floats2bfloat162_rn(other, mine_hi) : __floats2bfloat162_rn(mine_lo, other);
                        *reinterpret_cast<__nv_bfloat162 *>(tile + ((jj + odd) * 32 + (lane & ~1)) * 2) = pr;
                    }
                }
                __syncwarp();
                const int n0 = nt * BN + 32 * cc;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int r = 8 * g + rsub;
                    if (r < ncols) {
                        const uint4 val = *reinterpret_cast<const uint4 *>(tile + (r * 32 + seg * 8) * 2);
                        if (m_ok && n0 + r < p.N && in_bounds((int64_t)(n0 + r) * p.ld_out + m0 + seg * 8, 8, p.ext.out))
                            *reinterpret_cast<uint4 *>(out + (int64_t)(n0 + r) * p.ld_out + m0 + seg * 8) = val;
                    }
                }
                __syncwarp();  // every lane has read the tile before the next chunk overwrites it
            }
            ++it;
        }
    } else if (warp < 10) {
        // ------------------------------------------------------------ code writers (both CTAs)
        // Lane image row L of a slot: for k-block c (32 logical K), the code
        // word 2c + h of row mm (low half) and of row mm + 8 (high half), with
        // mm = 16 (L / 16) + L % 8 and h = (L / 8) % 2.  Built in place over
        // the raw tile (row m at byte 16 m): image rows 32 q .. 32 q + 31 take
        // their codes from raw rows 32 q .. 32 q + 31 only, so each warp
        // reads its block, syncs, and writes it.
        const int q = warp & 3;
        const int L = 32 * q + lane;
        const int mm = 16 * (L >> 4) + (L & 7);
        const int h = (L >> 3) & 1;
        const int words_per_row = p.k_logical / 16;
        int e = 0, j = 0;
        uint32_t eph = 0;
        for (int w = pair; w < p.num_work; w += num_pairs) {
            int mt, nt, sp, k0, k1;
            pair_unit<SPLIT>(p, w, mt, nt, sp, k0, k1);
            const int rowA = mt * 256 + 128 * rank + mm;
            for (int kt = k0; kt < k1; ++kt, ++j) {
                if (!mbar_wait_warp(&efull[e], eph, abort_flag)) goto done;
                uint8_t *et = ering + e * C::E_BYTES;
                uint32_t ca[4], cb[4];
                if (p.meta_tma) {
                    const uint4 va = *reinterpret_cast<const uint4 *>(et + mm * 16);
                    const uint4 vb = *reinterpret_cast<const uint4 *>(et + (mm + 8) * 16);
                    ca[0] = va.x; ca[1] = va.y; ca[2] = va.z; ca[3] = va.w;
                    cb[0] = vb.x; cb[1] = vb.y; cb[2] = vb.z; cb[3] = vb.w;
                    const uint32_t fill = 0x44444444u;
                    if (rowA >= p.M) ca[0] = ca[1] = ca[2] = ca[3] = fill;
                    if (rowA + 8 >= p.M) cb[0] = cb[1] = cb[2] = cb[3] = fill;
                    if (kt * 8 + 8 > words_per_row) { ca[2] = ca[3] = cb[2] = cb[3] = fill; }
                } else {
                    load_codes8(p.meta_a, rowA, p.M, words_per_row, kt * 8, ca, p.ext.meta_a);
                    load_codes8(p.meta_a, rowA + 8, p.M, words_per_row, kt * 8, cb, p.ext.meta_a);
                }
                uint4 img;
                img.x = word16(ca, 0 + h) | (word16(cb, 0 + h) << 16);
                img.y = word16(ca, 2 + h) | (word16(cb, 2 + h) << 16);
                img.z = word16(ca, 4 + h) | (word16(cb, 4 + h) << 16);
                img.w = word16(ca, 6 + h) | (word16(cb, 6 + h) << 16);
                __syncwarp();  // this warp's 32 image rows come from its own 32 raw rows: all read
                *reinterpret_cast<uint4 *>(et + L * 16) = img;
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
        // A batch of slots is free once the tcgen05.cp and the MMAs that read
        // it are done (eempty, committed by the MMA issuer).
        if (lane == 0) {
            int e = 0;
            uint32_t bph = 0;  // per-batch phase bits of eempty
            uint32_t aph = 0;  // phase of adp_empty
            const int rp = p.adp_buf;
            // bytes of both CTAs' adapter tiles, counted on the leader's barrier
            const uint32_t adp_tx = 2u * (uint32_t)(128 * rp * 2 + BNH * rp * 2);
            for (int w = pair; w < p.num_work; w += num_pairs) {
                int mt, nt, sp, k0, k1;
                pair_unit<SPLIT>(p, w, mt, nt, sp, k0, k1);
                const int m0 = mt * 256 + 128 * rank;
                if (rp > 0 && sp == 0) {
                    // the adapter tile of this output tile (the previous one's
                    // adapter MMAs, issued first in that tile, have released it)
                    if (!mbar_wait(adp_empty, aph ^ 1, abort_flag)) goto done;
                    aph ^= 1;
                    const uint32_t lead = cluster_addr(adp_full, 0);
                    if (rank == 0) mbar_arrive_expect_tx(adp_full, adp_tx);
                    if (A2_MN) {
                        tma_load_2d_pair(adp, &tmA2, lead, m0, 0);
                        tma_load_2d_pair(adp + rp * 128, &tmA2, lead, m0 + 64, 0);
                    } else {
                        tma_load_2d_pair(adp, &tmA2, lead, 0, m0);
                    }
                    tma_load_2d_pair(adp + C::ADP_A_BYTES, &tmB2, lead, 0, nt * BN + BNH * rank);
                }
                for (int kt = k0; kt < k1; ++kt) {
                    if (e % CB == 0) {
                        const int bb = e / CB;
                        if (!mbar_wait(&eempty[bb], ((bph >> bb) & 1u) ^ 1u, abort_flag)) goto done;
                        bph ^= 1u << bb;
                    }
                    if (p.meta_tma) {
                        mbar_arrive_expect_tx(&efull[e], C::E_BYTES);
                        tma_load_2d(ering + e * C::E_BYTES, &tmE, &efull[e], kt * 8, m0);
                    } else {
                        mbar_arrive(&efull[e]);  // slot free: the writers read the codes from global memory
                    }
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
}

// ---------------------------------------------------------------------------
// Masked weight gradient on SM pairs: dW = (dY^T . X) at the static mask,
// dense tcgen05 cta_group::2 with M = 256 output rows (out) per pair and BN
// columns (in).  A = dY^T and B = X are both read as MN-major operands straight
// from the row-major [T x out] and [T x in] tensors; K = T.  CTA r holds A rows
// [128 r, 128 r + 128) and B columns [BN/2 r, BN/2 r + BN/2).  The epilogue
// keeps the two masked columns of every group of four and writes them in W^R's
// compressed slot order.
//
// Split over tokens (p.num_splits > 1, for layers with fewer tiles than SM
// pairs): a work unit is (tile, token range).  Each epilogue warp writes its
// 32 rows of masked fp32 partials to its split's workspace slot, fences, and
// counts itself on the counter of (tile, CTA, warp); the warp that arrives last
// sums all slots in split order, writes the bf16 values and resets the counter
// to 0.  No warp waits for another.
// Final sum of a token-split masked weight gradient, by the warp that
// arrived last for its 32 rows x BN columns: all NSPL partial slots, summed
// in split order, converted to bf16.  Lanes cover a row's BN / 2 kept values
// four at a time (coalesced 16-byte reads, 8-byte stores); SB steps of rows
// are loaded together, NSPL x SB (about 32) independent loads in flight.
template <int BN, int NSPL>
__device__ __forceinline__ void dw_split_sum(const GemmParams &p, int row0, int nt, int lane) {
    constexpr int FPR = BN / 8;         // float4s per row (BN / 2 kept values)
    constexpr int RPS = 32 / FPR;       // rows per step (1 or 2)
    constexpr int STEPS = 32 / RPS;
    constexpr int SB = NSPL >= 32 ? 1 : 32 / NSPL;  // steps per batch
    const int c4 = lane % FPR;
    const int n = nt * BN + 8 * c4;    // first of the 8 columns (4 kept values) of this lane
    const bool col_ok = n < p.N;
    const size_t slot_stride = (size_t)p.M * (p.N / 2);
#pragma unroll 1
    for (int st0 = 0; st0 < STEPS; st0 += SB) {
        float4 v[SB][NSPL];
#pragma unroll
        for (int b = 0; b < SB; ++b) {
            const int row = row0 + (st0 + b) * RPS + lane / FPR;
            const bool ok = col_ok && row < p.M && st0 + b < STEPS &&
                            in_bounds((int64_t)row * (p.N / 2) + n / 2 + (int64_t)(NSPL - 1) * slot_stride, 4, p.ext.ws);
            const float4 *src = reinterpret_cast<const float4 *>(p.ws + (size_t)row * (p.N / 2) + n / 2);
#pragma unroll
            for (int k = 0; k < NSPL; ++k) v[b][k] = ok ? __ldcg(src + k * (slot_stride / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int b = 0; b < SB; ++b) {
            const int row = row0 + (st0 + b) * RPS + lane / FPR;
            if (!(col_ok && row < p.M && st0 + b < STEPS)) continue;
            if (!in_bounds((int64_t)row * p.ld_out + n / 2, 4, p.ext.out)) continue;
            float4 a = v[b][0];
#pragma unroll
            for (int k = 1; k < NSPL; ++k) {
                a.x += v[b][k].x;
                a.y += v[b][k].y;
                a.z += v[b][k].z;
                a.w += v[b][k].w;
            }
            const uint32_t lo = static_cast<uint32_t>(f32_to_bf16_bits(a.x)) | (static_cast<uint32_t>(f32_to_bf16_bits(a.y)) << 16);
            const uint32_t hi = static_cast<uint32_t>(f32_to_bf16_bits(a.z)) | (static_cast<uint32_t>(f32_to_bf16_bits(a.w)) << 16);
            *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(p.out) + (int64_t)row * p.ld_out + n / 2) = make_uint2(lo, hi);
        }
    }
}

// Unit w of the masked-gradient launch: 0 = a dW tile (mt, nt, sp), 1 = a
// dR^T block (mt = 256-row block of out, sp), 2 = a dL block (mt = 256-row
// block of in, sp).  The dW tiles come first.
__device__ __forceinline__ int dw_unit(const GemmParams &p, int w, int &mt, int &nt, int &sp) {
    const int n_dw = p.num_m_tiles * p.num_n_tiles * p.num_splits;
    if (w < n_dw) {
        if (p.num_splits == 1) {  // unsplit: grouped tile order (L2 reuse of dY and X)
            grouped_tile(w, p.num_m_tiles, p.num_n_tiles, p.raster_g, mt, nt);
            sp = 0;
        } else {
            decode_work(p, w, mt, nt, sp);
        }
        return 0;
    }
    w -= n_dw;
    nt = 0;
    if (w < p.ad_units_r) {
        mt = w % p.num_m_tiles;
        sp = w / p.num_m_tiles;
        return 1;
    }
    w -= p.ad_units_r;
    const int nb = (p.ad_in + 255) / 256;
    mt = w % nb;
    sp = w / nb;
    return 2;
}

// Epilogue of a dR^T or dL unit: this warp's 32 rows (lane = row of out or
// in) x ad_r rank columns.  Unsplit: written straight to dR (transposed:
// dR[j][o], coalesced across lanes) or dL (row-major).  Split over tokens: the
// fp32 partial goes to the unit's slot, and the last split to arrive for
// (block, CTA, warp) sums the slots in split order and writes the result.
__device__ __noinline__ void dw_adapter_epilogue(uint32_t taddr, int lane, int row, int kind, int mt, int sp, int q,
                                                 uint32_t rank, uint64_t *acc_empty, const GemmParams &p) {
    const int Mu = kind == 1 ? p.M : p.ad_in;  // rows of the unit's output
    const bool row_ok = row < Mu;
    const bool split = p.num_splits > 1;
    float *const ws_base = kind == 1 ? p.ws2 : p.ws2 + (int64_t)p.num_splits * p.M * p.ad_r;
    uint32_t v[32];
#pragma unroll 1
    for (int c0 = 0; c0 < p.ad_r; c0 += 32) {
        tmem_ld_32x32(taddr + c0, v);
        tmem_ld_wait();
        if (!row_ok) continue;
        const int nj = min(32, p.ad_r - c0);  // a multiple of 8
        if (split) {
            float *slot = ws_base + ((int64_t)sp * Mu + row) * p.ad_r + c0;
            if (!in_buf(slot, p.ws2, nj, p.ext.ws2)) continue;
#pragma unroll
            for (int j4 = 0; j4 < 32; j4 += 4)
                if (j4 < nj) *reinterpret_cast<uint4 *>(slot + j4) = make_uint4(v[j4], v[j4 + 1], v[j4 + 2], v[j4 + 3]);
        } else if (kind == 1) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (j < nj && in_bounds((int64_t)(c0 + j) * p.M + row, 1, p.ext.dR))
                    p.dR[(int64_t)(c0 + j) * p.M + row] = bits_to_f32(v[j]);
        } else {
#pragma unroll
            for (int j4 = 0; j4 < 32; j4 += 4)
                if (j4 < nj && in_bounds((int64_t)row * p.ad_r + c0 + j4, 4, p.ext.dL))
                    *reinterpret_cast<float4 *>(p.dL + (int64_t)row * p.ad_r + c0 + j4) =
                        make_float4(bits_to_f32(v[j4]), bits_to_f32(v[j4 + 1]), bits_to_f32(v[j4 + 2]), bits_to_f32(v[j4 + 3]));
        }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(cluster_addr(acc_empty, 0));
    if (!split) return;
    __threadfence();
    __syncwarp();
    int last = 0;
    if (lane == 0) {
        const int ublock = kind == 1 ? mt : p.num_m_tiles + mt;
        int *cnt = p.ws2_count + ((int64_t)ublock * 2 + rank) * 4 + q;
        if (in_buf(cnt, p.ws2_count, 1, p.ext.ws2_count)) last = atomicAdd(cnt, 1) == p.num_splits - 1;
        if (last) *cnt = 0;  // every split has arrived: ready for the next launch
    }
    last = __shfl_sync(0xFFFFFFFFu, last, 0);
    if (!last || !row_ok) return;
    __threadfence();
#pragma unroll 1
    for (int c0 = 0; c0 < p.ad_r; c0 += 4) {
        if (!in_buf(ws_base + ((int64_t)(p.num_splits - 1) * Mu + row) * p.ad_r + c0, p.ws2, 4, p.ext.ws2) ||
            !in_bounds(kind == 1 ? (int64_t)(c0 + 3) * p.M + row : (int64_t)row * p.ad_r + c0, kind == 1 ? 1 : 4,
                       kind == 1 ? p.ext.dR : p.ext.dL))
            continue;
        float4 a = __ldcg(reinterpret_cast<const float4 *>(ws_base + (int64_t)row * p.ad_r + c0));
        for (int k = 1; k < p.num_splits; ++k) {  // in split order, the same whichever arrived last
            const float4 b = __ldcg(reinterpret_cast<const float4 *>(ws_base + ((int64_t)k * Mu + row) * p.ad_r + c0));
            a.x += b.x;
            a.y += b.y;
            a.z += b.z;
            a.w += b.w;
        }
        if (kind == 1) {
            p.dR[(int64_t)(c0 + 0) * p.M + row] = a.x;
            p.dR[(int64_t)(c0 + 1) * p.M + row] = a.y;
            p.dR[(int64_t)(c0 + 2) * p.M + row] = a.z;
            p.dR[(int64_t)(c0 + 3) * p.M + row] = a.w;
        } else {
            *reinterpret_cast<float4 *>(p.dL + (int64_t)row * p.ad_r + c0) = a;
        }
    }
}

template <int BN>
struct DwPairCfg {
    static constexpr int BNH = BN / 2;
    static constexpr int A_BYTES = 16384;         // 2 panels [64 t x 64 rows]
    static constexpr int B_BYTES = BNH * 128;     // BNH/64 panels [64 t x 64 cols]
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int NS_RAW = (208 * 1024) / STAGE_BYTES;
    static constexpr int NS = NS_RAW > 8 ? 8 : NS_RAW;
    static constexpr int TMEM_COLS = 2 * BN <= 256 ? 256 : 512;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = NS * STAGE_BYTES + BAR_BYTES + 1024;
    static_assert(BNH % 64 == 0 && BN <= 256, "tile shape");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <int BN>
__global__ void __launch_bounds__(192, 1)
    dw_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmXL, const __grid_constant__ CUtensorMap tmG,
                   const __grid_constant__ GemmParams p) {
    using C = DwPairCfg<BN>;
    constexpr int NS = C::NS;
    constexpr int BNH = C::BNH;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + NS * C::STAGE_BYTES);  // leader: both CTAs' bytes
    uint64_t *empty = full + NS;
    uint64_t *acc_full = empty + NS;
    uint64_t *acc_empty = acc_full + 2;  // leader: 8 arrivals
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(acc_empty + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 8);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (p.ad_units_r > 0) {
            tma_prefetch_desc(&tmXL);
            tma_prefetch_desc(&tmG);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_holder, C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    grid_dep_wait();
    grid_dep_launch();

    if (warp == 0) {
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            for (int w = pair; w < p.num_work; w += num_pairs) {
                int mt, nt, sp, k0, k1;
                const int kind = dw_unit(p, w, mt, nt, sp);
                k_range(p, sp, k0, k1);
                const int m0 = mt * 256 + 128 * rank;
                const int n0 = nt * BN + BNH * rank;
                if (kind != 0) {
                    // dR^T: A = dY^T (as the dW tiles), B = XL; dL: A = X^T (X read as the A operand), B = G;
                    // B MN-major, ad_c rank columns per CTA
                    const uint32_t b_bytes = 128u * (uint32_t)p.ad_c;
                    const CUtensorMap *ma = kind == 1 ? &tmA : &tmB;
                    const CUtensorMap *mb = kind == 1 ? &tmXL : &tmG;
                    for (int kt = k0; kt < k1; ++kt) {
                        if (!mbar_wait(&empty[s], ph ^ 1, abort_flag)) goto done;
                        uint8_t *a = smem + s * C::STAGE_BYTES;
                        uint8_t *b = a + C::A_BYTES;
                        const uint32_t lead_full = cluster_addr(&full[s], 0);
                        if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * (C::A_BYTES + b_bytes));
                        tma_load_2d_pair(a, ma, lead_full, m0, kt * 64);
                        tma_load_2d_pair(a + 8192, ma, lead_full, m0 + 64, kt * 64);
                        tma_load_2d_pair(b, mb, lead_full, (int)rank * p.ad_c, kt * 64);
                        if (++s == NS) { s = 0; ph ^= 1; }
                    }
                    continue;
                }
                for (int kt = k0; kt < k1; ++kt) {
                    if (!mbar_wait(&empty[s], ph ^ 1, abort_flag)) goto done;
                    uint8_t *a = smem + s * C::STAGE_BYTES;
                    uint8_t *b = a + C::A_BYTES;
                    const uint32_t lead_full = cluster_addr(&full[s], 0);
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * C::STAGE_BYTES);
                    tma_load_2d_pair(a, &tmA, lead_full, m0, kt * 64);
                    tma_load_2d_pair(a + 8192, &tmA, lead_full, m0 + 64, kt * 64);
#pragma unroll
                    for (int j = 0; j < BNH / 64; ++j)
                        tma_load_2d_pair(b + j * 8192, &tmB, lead_full, n0 + 64 * j, kt * 64);
                    if (++s == NS) { s = 0; ph ^= 1; }
                }
            }
        }
    } else if (warp == 1) {
        if (rank == 0 && lane == 0) {
            constexpr uint32_t IDESC = instr_desc(256, BN, 1, 1, 0);
            const uint32_t base = smem_addr(smem);
            const uint64_t a_desc0 = smem_desc(base, 8192, 1024, SWZ_128B);
            const uint64_t b_desc0 = smem_desc(base + C::A_BYTES, 8192, 1024, SWZ_128B);
            // adapter-gradient units: B = XL or G, MN-major rows of 2 ad_c bytes
            const uint32_t ad_rowb = 2u * (uint32_t)p.ad_c;
            const uint64_t b2_desc0 = smem_desc(base + C::A_BYTES, 8192, 8 * ad_rowb,
                                                ad_rowb == 32 ? SWZ_32B : ad_rowb == 64 ? SWZ_64B : SWZ_128B);
            const uint32_t IDESC2 = instr_desc(256, p.ad_n > 0 ? p.ad_n : 16, 1, 1, 0);
            int s = 0;
            uint32_t ph = 0;
            int it = 0;
            for (int w = pair; w < p.num_work; w += num_pairs) {
                int mt, nt, sp, k0, k1;
                const int kind = dw_unit(p, w, mt, nt, sp);
                k_range(p, sp, k0, k1);
                const int acc = it & 1;
                const uint32_t acc_ph = (it >> 1) & 1;
                if (!mbar_wait(&acc_empty[acc], acc_ph ^ 1, abort_flag)) goto done;
                tc_fence_after();
                const uint32_t d = tmem_base + acc * BN;
                uint32_t accumulate = 0;
                for (int kt = k0; kt < k1; ++kt) {
                    if (!mbar_wait(&full[s], ph, abort_flag)) goto done;
                    tc_fence_after();
                    const uint64_t ad = a_desc0 + (uint64_t)((s * C::STAGE_BYTES) >> 4);
                    if (kind != 0) {
                        const uint64_t bd = b2_desc0 + (uint64_t)((s * C::STAGE_BYTES) >> 4);
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            mma_bf16_pair(d, ad + (uint64_t)(128 * c), bd + (uint64_t)(ad_rowb * c), IDESC2,
                                          accumulate | (uint32_t)c);
                        accumulate = 1;
                        mma_commit_pair_both(&empty[s]);
                        if (++s == NS) { s = 0; ph ^= 1; }
                        continue;
                    }
                    const uint64_t bd = b_desc0 + (uint64_t)((s * C::STAGE_BYTES) >> 4);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        mma_bf16_pair(d, ad + (uint64_t)(128 * c), bd + (uint64_t)(128 * c), IDESC, accumulate | (uint32_t)c);
                    accumulate = 1;
                    mma_commit_pair_both(&empty[s]);
                    if (++s == NS) { s = 0; ph ^= 1; }
                }
                mma_commit_pair_both(&acc_full[acc]);
                ++it;
            }
        }
    } else {
        // epilogue: this CTA's 128 rows (out) x BN columns (in); lane = row
        const int q = warp & 3;
        const bool split = p.num_splits > 1;
        int it = 0;
        for (int w = pair; w < p.num_work; w += num_pairs) {
            int mt, nt, sp;
            const int kind = dw_unit(p, w, mt, nt, sp);
            const int acc = it & 1;
            const uint32_t acc_ph = (it >> 1) & 1;
            if (kind != 0) {
                if (!mbar_wait_warp(&acc_full[acc], acc_ph, abort_flag)) break;
                tc_fence_after();
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + acc * BN;
                dw_adapter_epilogue(taddr, lane, mt * 256 + 128 * rank + 32 * q + lane, kind, mt, sp, q, rank,
                                    &acc_empty[acc], p);
                ++it;
                continue;
            }
            const int row = mt * 256 + 128 * rank + 32 * q + lane;
            const bool row_ok = row < p.M;
            uint16_t *out_row = reinterpret_cast<uint16_t *>(p.out) + (int64_t)row * p.ld_out;
            // this row's mask codes for the tile (one 32-bit word per 32
            // columns), loaded while the tile's MMAs still run
            const uint32_t *mask_row = reinterpret_cast<const uint32_t *>(p.meta_mask + (int64_t)row * (p.N / 16));
            uint32_t cw[BN / 32];
#pragma unroll
            for (int cc = 0; cc < BN / 32; ++cc) {
                const int n = nt * BN + 32 * cc;
                cw[cc] = (row_ok && n < p.N && in_bounds((int64_t)row * (p.N / 16) + n / 16, 2, p.ext.meta_mask))
                             ? mask_row[n / 32] : 0u;
            }
            if (!mbar_wait_warp(&acc_full[acc], acc_ph, abort_flag)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + acc * BN;
#pragma unroll
            for (int cc = 0; cc < BN / 32; ++cc) {
                uint32_t v[32];
                tmem_ld_32x32(taddr + 32 * cc, v);
                tmem_ld_wait();
                if (cc == BN / 32 - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(cluster_addr(&acc_empty[acc], 0));
                }
                const int n = nt * BN + 32 * cc;
                if (n >= p.N) continue;  // the same for every lane
                const uint32_t codes = cw[cc];
                uint32_t kept[16];  // fp32 bits of the two masked columns of each group
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const uint32_t code = (codes >> (4 * g)) & 0xFu;
                    const uint32_t i0 = code & 3u, i1 = code >> 2;
                    kept[2 * g] = i0 == 0 ? v[4 * g] : (i0 == 1 ? v[4 * g + 1] : v[4 * g + 2]);
                    kept[2 * g + 1] = i1 == 1 ? v[4 * g + 1] : (i1 == 2 ? v[4 * g + 2] : v[4 * g + 3]);
                }
                if (!row_ok) continue;
                if (split) {
                    uint4 *slot = reinterpret_cast<uint4 *>(p.ws + ((int64_t)sp * p.M + row) * (p.N / 2) + n / 2);
                    if (!in_bounds(((int64_t)sp * p.M + row) * (p.N / 2) + n / 2, 16, p.ext.ws)) continue;
#pragma unroll
                    for (int k = 0; k < 4; ++k) slot[k] = make_uint4(kept[4 * k], kept[4 * k + 1], kept[4 * k + 2], kept[4 * k + 3]);
                } else {
                    uint32_t packed[8];
#pragma unroll
                    for (int g = 0; g < 8; ++g)
                        packed[g] = static_cast<uint32_t>(f32_to_bf16_bits(bits_to_f32(kept[2 * g]))) |
                                    (static_cast<uint32_t>(f32_to_bf16_bits(bits_to_f32(kept[2 * g + 1]))) << 16);
                    uint4 *dst = reinterpret_cast<uint4 *>(out_row + n / 2);
                    if (!in_bounds((int64_t)row * p.ld_out + n / 2, 16, p.ext.out)) continue;
                    dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                    dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
                }
            }
            if (split) {
                // count this warp's partial in; the last of the splits reduces
                __threadfence();
                __syncwarp();
                int last = 0;
                if (lane == 0) {
                    int *cnt = p.ws_count + ((int64_t)(mt * p.num_n_tiles + nt) * 2 + rank) * 4 + q;
                    if (in_buf(cnt, p.ws_count, 1, p.ext.ws_count)) {
                        last = atomicAdd(cnt, 1) == p.num_splits - 1;
                        if (last) *cnt = 0;  // every split has arrived: ready for the next launch
                    }
                }
                last = __shfl_sync(0xFFFFFFFFu, last, 0);
                if (last) {
                    __threadfence();
                    const int row0 = mt * 256 + 128 * rank + 32 * q;
                    switch (p.num_splits) {
                        case 2: dw_split_sum<BN, 2>(p, row0, nt, lane); break;
                        case 3: dw_split_sum<BN, 3>(p, row0, nt, lane); break;
                        case 4: dw_split_sum<BN, 4>(p, row0, nt, lane); break;
                        case 5: dw_split_sum<BN, 5>(p, row0, nt, lane); break;
                        case 6: dw_split_sum<BN, 6>(p, row0, nt, lane); break;
                        case 7: dw_split_sum<BN, 7>(p, row0, nt, lane); break;
                        default: dw_split_sum<BN, 8>(p, row0, nt, lane); break;
                    }
                }
            }
            ++it;
        }
    }
done:
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace slope
