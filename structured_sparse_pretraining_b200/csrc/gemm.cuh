// gemm.cuh -- warp-specialised, persistent dense tcgen05 GEMM (1 SM per tile)
// for the adapter's skinny products: XL = X . L, G = dY . R^T,
// dR^T = dY^T . XL and dL = X^T . G (SLoPe technical summary (gist.science),
// §2.B: W_dense = W_sparse + L R; the gradients are the chain rule on it).
//
// Roles (192 threads): warp 0 TMA producer (one thread), warp 1 TMEM owner and
// MMA issuer (one thread), warps 2..5 epilogue (TMEM lanes 32 (warp % 4) ..).
// A and B are each K-major or MN-major (read straight from row-major tensors,
// no transposes in HBM).  Tiles are BM (64 or 128) rows x BN columns; a
// 64-row tile lets the token-dimension products of a few thousand tokens use
// every SM.  Optional split-K: the fp32 epilogues add into zeroed outputs.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace slope {

enum Epi : int {
    EPI_BF16_ROW = 2,     // out[m][n] = bf16(acc)      (XL, G)
    EPI_F32_ADD_ROW = 3,  // out[m][n] += acc (fp32)    (dL, split-K)
    EPI_F32_ADD_T = 4     // out[n][m] += acc (fp32)    (dR, split-K)
};

// Elements of each buffer a launch may touch, stated by the host from the
// sizes of the C ABI call (checked by the debug build's in_bounds).
struct Extents {
    int64_t out, ws, ws_count, meta_a, meta_mask, tok_out, tok_flags, tok_ws, tok_cnt, dR, dL, ws2, ws2_count;
};

struct GemmParams {
    int M, N;              // output extent along MMA M and MMA N
    int num_m_tiles, num_n_tiles, num_splits, num_work;
    int k_tiles_total;     // k-tiles of the main phase
    int k_tiles_per_split; // split-K: k-tiles per split
    int k_logical;         // sparse products: logical K (for the code words' bounds)
    int r;                 // sparse products: adapter rank (0 = no adapter phase)
    int adp_k_tiles;       // sparse products: adapter k-tiles through the operand ring (ceil(r / 64)), or 0
    int adp_buf;           // sparse products: 0, or the padded rank (16, 32) of an adapter tile held in its own buffer
    int meta_tma;          // sparse products: 1 = code tiles by TMA, 0 = from global memory
    const uint16_t *meta_a;     // sparse products: codes of A [M x k_logical/16]
    const uint16_t *meta_mask;  // masked weight gradient: codes of the mask [M x N/16]
    void *out;
    int64_t ld_out;        // leading dimension of `out`, in elements
    float *zero0;          // optional fp32 buffers this launch clears before its own work (outputs of
    int64_t zero_n0;       // later split-K launches, so that they need no separate clearing launch)
    float *zero1;
    int64_t zero_n1;
    float *ws;             // masked weight gradient split over tokens: fp32 partials [split][M][N/2]
    int *ws_count;         // and one arrival counter per (tile, CTA of the pair, epilogue warp), left at 0
    int raster_g;          // grouped tile order: m-tiles per group (0 = m fastest over the whole M)
    // Fused rank product of the sparse products (XL = X . L ahead of the
    // forward, G = dY . R^T ahead of the input gradient): the first tok_units
    // work units each compute it for 256 tokens and publish it with a flag.
    int tok_units;         // 0 = none
    int tok_k_tiles;       // its k-tiles (64 wide) over the reduction dimension
    int tok_n;             // its MMA N (the rank, padded)
    int tok_b_mn;          // 1: B = L [K x r] read MN-major, tok_bc columns per CTA; 0: B = R [r x K], tok_bc rows per CTA
    int tok_bc;
    int tok_r;             // rank columns written
    int tok_nsl;           // 64-wide k-slices per operand stage (a slice: 16 KB of token rows + the factor's rows)
    int tok_slice_bytes;   // bytes from one slice to the next in a stage (multiple of 1024)
    uint16_t *tok_out;     // [tokens x tok_r] bf16 (XL or G), also the adapter phase's B operand
    int *tok_flags;        // per unit: epilogue warps done (8 when complete); [tok_units]: CTAs finished; all left 0
    int tok_split;         // pieces per unit (1 = none): piece h sums the h-th of tok_split ranges of the k-slices
    int tok_items;         // tok_units x tok_split: the first work items of the launch
    float *tok_ws;         // split units: fp32 partials [unit][piece][256 rows][tok_r]
    int *tok_cnt;          // split units: pieces arrived per (unit, CTA, epilogue warp), left at 0
    // Adapter gradients fused into the masked weight gradient: after the dW
    // units come ad_units_r units of dR^T = dY^T . XL (per 256-row block of
    // out and token split) and ad_units_l units of dL = X^T . G (per 256-row
    // block of in and split).  MMA N = ad_n (the rank padded; ad_c columns of
    // XL or G per CTA); ad_r rank columns written; ad_in = in.
    int ad_units_r, ad_units_l, ad_n, ad_c, ad_r, ad_in;
    float *dR, *dL;        // [ad_r x out] and [in x ad_r], fp32
    float *ws2;            // split partials of those units: [split][out][ad_r], then [split][in][ad_r]
    int *ws2_count;        // per (unit block, CTA, epilogue warp), left at 0
    Extents ext;
};

// Grouped order of the output tiles of an unsplit launch (L2 reuse): work unit
// w walks groups of `g` m-tiles; inside a group the m-tile varies fastest, so
// the pairs active at one time share a few weight tiles and a few token tiles,
// which then serve several pairs from L2 instead of being streamed from DRAM
// once per pair.  g = 0: the m-tile varies fastest over the whole M.
__device__ __forceinline__ void grouped_tile(int w, int num_m_tiles, int num_n_tiles, int g, int &mt, int &nt) {
    if (g <= 0 || g >= num_m_tiles) {
        mt = w % num_m_tiles;
        nt = w / num_m_tiles;
        return;
    }
    const int per = g * num_n_tiles;
    const int grp = w / per, i = w % per;
    const int gm = min(g, num_m_tiles - grp * g);  // the last group may hold fewer m-tiles
    mt = grp * g + i % gm;
    nt = i / gm;
}

template <int BM, int BN>
struct GemmCfg {
    static constexpr int A_BYTES = BM * 128;   // BM rows x 64 K (K-major) or BM/64 panels (MN-major)
    // B: BN rows x 64 K (K-major, 128-byte swizzle), or 64 K-rows of BN
    // elements (MN-major): 64-element panels with 128-byte swizzle, or one
    // row of 16 / 32 elements with a 32 / 64-byte swizzle when BN < 64
    static constexpr int B_BYTES = BN * 128;
    static constexpr int B_MN_ROW = (BN < 64 ? BN : 64) * 2;  // bytes per K-row of an MN-major B panel
    static constexpr uint32_t B_MN_SWZ = BN == 16 ? SWZ_32B : BN == 32 ? SWZ_64B : SWZ_128B;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int NS_RAW = (208 * 1024) / STAGE_BYTES;
    static constexpr int NS = NS_RAW > 12 ? 12 : NS_RAW;
    static constexpr int COLS_USED = 2 * BN;
    static constexpr int TMEM_COLS = COLS_USED <= 32 ? 32 : COLS_USED <= 64 ? 64 : COLS_USED <= 128 ? 128
                                     : COLS_USED <= 256 ? 256 : 512;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = NS * STAGE_BYTES + BAR_BYTES + 1024;
    static_assert(BM == 64 || BM == 128, "tile rows");
    static_assert((BN == 16 || BN == 32 || BN % 64 == 0) && BN <= 256, "tile columns");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

__device__ __forceinline__ float bits_to_f32(uint32_t v) { return __uint_as_float(v); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

__device__ __forceinline__ void decode_work(const GemmParams &p, int w, int &m_tile, int &n_tile, int &split) {
    m_tile = w % p.num_m_tiles;
    const int rest = w / p.num_m_tiles;
    n_tile = rest % p.num_n_tiles;
    split = rest / p.num_n_tiles;
}

__device__ __forceinline__ void k_range(const GemmParams &p, int split, int &k0, int &k1) {
    k0 = split * p.k_tiles_per_split;
    k1 = min(p.k_tiles_total, k0 + p.k_tiles_per_split);
}

// bf16 epilogue of a product split over K (out of line, so that the unsplit
// path's code stays as it is).  Each split adds its fp32 partial into a
// per-device accumulator [M x N] (fire-and-forget atomic adds, kept at zero
// between launches), releases the accumulator tile, and counts itself in on
// the counter of (tile, quarter).  The warp that arrives last converts its
// rows of the tile to bf16 and zeroes them again.  Every split's adds are in
// flight at once, so the final step is one read of the tile instead of a
// walk through every split's partial; the order of the adds, and so the last
// bit of a sum, can differ from run to run.
template <int BN>
__device__ __noinline__ void gemm_split_bf16_epilogue(uint32_t taddr, int lane, bool lane_ok, int row, int nt,
                                                      int64_t unit, uint64_t *acc_empty, const GemmParams &p) {
    constexpr int NCH = (BN + 31) / 32;
    constexpr int CW = BN == 16 ? 16 : 32;  // columns per chunk
    const bool row_ok = lane_ok && row < p.M;
    float *acc_row = p.ws + (int64_t)row * p.N;
    uint32_t v[32];
#pragma unroll 1
    for (int cc = 0; cc < NCH; ++cc) {
        if (BN == 16) tmem_ld_32x32_x16(taddr, v);
        else tmem_ld_32x32(taddr + 32 * cc, v);
        tmem_ld_wait();
        const int n = nt * BN + 32 * cc;
        if (row_ok) {
#pragma unroll
            for (int j = 0; j < CW; ++j)
                if (n + j < p.N && in_buf(acc_row + n + j, p.ws, 1, p.ext.ws)) atomicAdd(acc_row + n + j, bits_to_f32(v[j]));
        }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(acc_empty);
    __threadfence();
    __syncwarp();
    int last = 0;
    if (lane == 0 && in_bounds(unit, 1, p.ext.ws_count)) {
        int *cnt = p.ws_count + unit;
        last = atomicAdd(cnt, 1) == p.num_splits - 1;
        if (last) *cnt = 0;  // every split has arrived: ready for the next launch
    }
    last = __shfl_sync(0xFFFFFFFFu, last, 0);
    if (!last || !row_ok) return;
    __threadfence();
    // this lane's row of the tile: columns n0 .. n0 + BN (N and n0 are multiples of 8)
    const int n0 = nt * BN;
    const int nq = min(BN, p.N - n0) / 4;
    uint16_t *out = reinterpret_cast<uint16_t *>(p.out) + (int64_t)row * p.ld_out + n0;
    float4 *src = reinterpret_cast<float4 *>(acc_row + n0);
    if (!in_buf(acc_row + n0, p.ws, 4 * nq, p.ext.ws) ||
        !in_buf(out, reinterpret_cast<uint16_t *>(p.out), 4 * nq, p.ext.out))
        return;
#pragma unroll 1
    for (int q0 = 0; q0 < nq; q0 += 8) {
        float4 x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (q0 + u < nq) x[u] = __ldcg(src + q0 + u);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (q0 + u < nq) {
                const uint32_t lo = static_cast<uint32_t>(f32_to_bf16_bits(x[u].x)) |
                                    (static_cast<uint32_t>(f32_to_bf16_bits(x[u].y)) << 16);
                const uint32_t hi = static_cast<uint32_t>(f32_to_bf16_bits(x[u].z)) |
                                    (static_cast<uint32_t>(f32_to_bf16_bits(x[u].w)) << 16);
                *reinterpret_cast<uint2 *>(out + 4 * (q0 + u)) = make_uint2(lo, hi);
                __stcg(src + q0 + u, make_float4(0.f, 0.f, 0.f, 0.f));  // zero again for the next launch
            }
        }
    }
}

template <bool A_MN, bool B_MN, int EPI, int BM, int BN>
__global__ void __launch_bounds__(192, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ GemmParams p) {
    using C = GemmCfg<BM, BN>;
    constexpr int NS = C::NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + NS * C::STAGE_BYTES);
    uint64_t *empty = full + NS;
    uint64_t *acc_full = empty + NS;
    uint64_t *acc_empty = acc_full + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(acc_empty + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    grid_dep_wait();
    grid_dep_launch();
    {
        const int64_t i0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x, step = (int64_t)gridDim.x * blockDim.x;
        for (int64_t i = i0; i < p.zero_n0; i += step) p.zero0[i] = 0.0f;
        for (int64_t i = i0; i < p.zero_n1; i += step) p.zero1[i] = 0.0f;
    }

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            for (int w = blockIdx.x; w < p.num_work; w += gridDim.x) {
                int mt, nt, sp, k0, k1;
                decode_work(p, w, mt, nt, sp);
                k_range(p, sp, k0, k1);
                const int m0 = mt * BM, n0 = nt * BN;
                for (int kt = k0; kt < k1; ++kt) {
                    if (!mbar_wait(&empty[s], ph ^ 1, abort_flag)) goto done;
                    uint8_t *a = smem + s * C::STAGE_BYTES;
                    uint8_t *b = a + C::A_BYTES;
                    mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
                    if (A_MN) {
#pragma unroll
                        for (int j = 0; j < BM / 64; ++j) tma_load_2d(a + j * 8192, &tmA, &full[s], m0 + 64 * j, kt * 64);
                    } else {
                        tma_load_2d(a, &tmA, &full[s], kt * 64, m0);
                    }
                    if (B_MN) {
#pragma unroll
                        for (int j = 0; j < (BN + 63) / 64; ++j)
                            tma_load_2d(b + j * 8192, &tmB, &full[s], n0 + 64 * j, kt * 64);
                    } else {
                        tma_load_2d(b, &tmB, &full[s], kt * 64, n0);
                    }
                    if (++s == NS) { s = 0; ph ^= 1; }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC = instr_desc(BM, BN, A_MN ? 1 : 0, B_MN ? 1 : 0, 0);
            // Descriptors of stage 0; stages and k-blocks only add constants to
            // the start-address field.
            const uint32_t base = smem_addr(smem);
            const uint64_t a_desc0 = A_MN ? smem_desc(base, 8192, 1024, SWZ_128B) : smem_desc(base, 16, 1024, SWZ_128B);
            const uint64_t b_desc0 = B_MN ? smem_desc(base + C::A_BYTES, 8192, 8 * C::B_MN_ROW, C::B_MN_SWZ)
                                          : smem_desc(base + C::A_BYTES, 16, 1024, SWZ_128B);
            int s = 0;
            uint32_t ph = 0;
            int it = 0;
            for (int w = blockIdx.x; w < p.num_work; w += gridDim.x) {
                int mt, nt, sp, k0, k1;
                decode_work(p, w, mt, nt, sp);
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
                    const uint64_t bd = b_desc0 + (uint64_t)((s * C::STAGE_BYTES) >> 4);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        mma_bf16(d, ad + (uint64_t)(A_MN ? 128 * c : 2 * c), bd + (uint64_t)(B_MN ? C::B_MN_ROW * c : 2 * c),
                                 IDESC, accumulate | (uint32_t)c);
                    accumulate = 1;
                    mma_commit(&empty[s]);
                    if (++s == NS) { s = 0; ph ^= 1; }
                }
                mma_commit(&acc_full[acc]);
                ++it;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // An M = 128 accumulator has row m in TMEM lane m; an M = 64 one has
        // rows 16 q .. 16 q + 15 in lanes 32 q .. 32 q + 15 of quarter q.
        const int q = warp & 3;
        const bool lane_ok = BM == 128 || lane < 16;
        int it = 0;
        for (int w = blockIdx.x; w < p.num_work; w += gridDim.x) {
            int mt, nt, sp;
            decode_work(p, w, mt, nt, sp);
            const int acc = it & 1;
            const uint32_t acc_ph = (it >> 1) & 1;
            if (!mbar_wait_warp(&acc_full[acc], acc_ph, abort_flag)) break;
            tc_fence_after();
            const int row = mt * BM + (BM == 128 ? 32 * q + lane : 16 * q + lane);
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + acc * BN;
            if (EPI == EPI_BF16_ROW && p.num_splits > 1) {
                const int64_t unit = (int64_t)(mt * p.num_n_tiles + nt) * 4 + q;
                gemm_split_bf16_epilogue<BN>(taddr, lane, lane_ok, row, nt, unit, &acc_empty[acc], p);
                ++it;
                continue;
            }
            // chunks of 32 columns; BN = 16 is a single 16-column chunk
            constexpr int NCH = (BN + 31) / 32;
#pragma unroll 1
            for (int cc = 0; cc < NCH; ++cc) {
                uint32_t v[32];
                if (BN == 16) tmem_ld_32x32_x16(taddr, v);
                else tmem_ld_32x32(taddr + 32 * cc, v);
                tmem_ld_wait();
                if (cc == NCH - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acc_empty[acc]);
                }
                const int n = nt * BN + 32 * cc;  // first column of this chunk
                if (!lane_ok || row >= p.M || n >= p.N) continue;
                const int nmax = min(BN == 16 ? 16 : 32, p.N - n);
                if (EPI == EPI_BF16_ROW) {
                    uint16_t *out = reinterpret_cast<uint16_t *>(p.out) + (int64_t)row * p.ld_out;
                    if (!in_bounds((int64_t)row * p.ld_out + n, nmax, p.ext.out)) continue;
#pragma unroll
                    for (int j8 = 0; j8 < 32; j8 += 8) {
                        if (j8 + 8 <= nmax) {
                            uint32_t pk[4];
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                pk[u] = static_cast<uint32_t>(f32_to_bf16_bits(bits_to_f32(v[j8 + 2 * u]))) |
                                        (static_cast<uint32_t>(f32_to_bf16_bits(bits_to_f32(v[j8 + 2 * u + 1]))) << 16);
                            *reinterpret_cast<uint4 *>(out + n + j8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        } else {
#pragma unroll
                            for (int u = 0; u < 8; ++u)
                                if (j8 + u < nmax) out[n + j8 + u] = f32_to_bf16_bits(bits_to_f32(v[j8 + u]));
                        }
                    }
                } else if (EPI == EPI_F32_ADD_ROW) {
                    float *out = reinterpret_cast<float *>(p.out) + (int64_t)row * p.ld_out;
                    if (!in_bounds((int64_t)row * p.ld_out + n, nmax, p.ext.out)) continue;
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (j < nmax) atomicAdd(out + n + j, bits_to_f32(v[j]));
                } else {  // EPI_F32_ADD_T
                    float *out = reinterpret_cast<float *>(p.out);
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (j < nmax && in_bounds((int64_t)(n + j) * p.ld_out + row, 1, p.ext.out))
                            atomicAdd(out + (int64_t)(n + j) * p.ld_out + row, bits_to_f32(v[j]));
                }
            }
            ++it;
        }
    }
done:
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace slope
