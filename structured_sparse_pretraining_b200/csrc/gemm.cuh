// gemm.cuh -- warp-specialised, persistent tcgen05 GEMM for the SLoPe layer.
//
// One CTA per SM.  Roles:
//   warp 0      TMA producer (one thread): fills a ring of shared-memory stages.
//   warp 1      MMA issuer (one thread) and TMEM owner.
//   warps 2..5  epilogue: TMEM -> registers -> global (quarter = warp % 4).
//   warps 6..9  (sparse modes only) metadata loaders: read the 2:4 position
//               codes of the A tile from global memory and write them into
//               TMEM with tcgen05.st in the layout tcgen05.mma.sp reads.
//
// Modes (template parameters):
//   SPARSE   A is a compressed 2:4 matrix (values K-major in smem, codes in
//            TMEM); each MMA covers 32 logical K (16 stored values).  Used for
//            the forward product Y^T = W^R . X^T and the input gradient
//            dX^T = (W^{R,C})^T . dY^T (SLoPe technical summary (gist.science),
//            §2.A).  An optional second phase accumulates the rank-r adapter
//            term (R^T . XL^T, or L . G^T) into the same fp32 tile (§2.B, §2.C:
//            the sparse product and the low-rank product in one kernel).
//   dense    plain bf16 x bf16 -> fp32, with A and B each K-major or MN-major,
//            optional split-K; used for the masked weight gradient and the
//            adapter products.
//
// Tiles: BM = 128 rows of the output (MMA M) x BN columns (MMA N).  Stage:
// A 16 KB (128 rows x 128 B, 128-byte swizzle) + B (sparse: BN rows x 256 B as
// two 128-byte-swizzled panels; dense: BN x 128 B).  Two fp32 accumulators in
// TMEM let the epilogue of tile i overlap the main loop of tile i+1.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace slope {

enum Epi : int {
    EPI_BF16_T = 0,       // out[n][m] = bf16(acc)      (Y, dX: rows are tokens)
    EPI_DW_COMPRESS = 1,  // keep the masked slots of row m, write compressed bf16
    EPI_BF16_ROW = 2,     // out[m][n] = bf16(acc)      (XL, G)
    EPI_F32_ADD_ROW = 3,  // out[m][n] += acc (fp32)    (dL, split-K)
    EPI_F32_ADD_T = 4     // out[n][m] += acc (fp32)    (dR, split-K)
};

struct GemmParams {
    int M, N;              // output extent along MMA M and MMA N
    int num_m_tiles, num_n_tiles, num_splits, num_work;
    int k_tiles_total;     // k-tiles of the main phase
    int k_tiles_per_split; // dense split-K: k-tiles per split
    int k_logical;         // sparse: logical K (for the code words' bounds)
    int r;                 // sparse modes: adapter rank (0 = no adapter phase)
    int adp_k_tiles;       // ceil(r / 64)
    const uint16_t *meta_a;     // sparse: codes of A [M x k_logical/16]
    const uint16_t *meta_mask;  // EPI_DW_COMPRESS: codes of the mask [M x N/16]
    void *out;
    int64_t ld_out;        // leading dimension of `out`, in elements
};

template <bool SPARSE, int BN>
struct GemmCfg {
    static constexpr int BM = 128;
    static constexpr int A_BYTES = 16384;
    static constexpr int B_BYTES = SPARSE ? BN * 256 : BN * 128;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int NS_RAW = (200 * 1024) / STAGE_BYTES;
    static constexpr int NS = NS_RAW > 8 ? 8 : NS_RAW;
    static constexpr int NUM_WARPS = SPARSE ? 10 : 6;
    static constexpr int META_COL = 2 * BN;
    static constexpr int COLS_USED = 2 * BN + (SPARSE ? 4 * NS : 0);
    static constexpr int TMEM_COLS = COLS_USED <= 32 ? 32 : COLS_USED <= 64 ? 64 : COLS_USED <= 128 ? 128
                                     : COLS_USED <= 256 ? 256 : 512;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = NS * STAGE_BYTES + BAR_BYTES + 1024;
    static_assert(COLS_USED <= 512, "TMEM budget");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(NS >= 2, "pipeline depth");
    static_assert(BN % 64 == 0 || !SPARSE, "sparse tiles are multiples of 64 tokens");
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

// Eight consecutive 16-bit code words of one row of A (words w0..w0+7),
// returned as four 32-bit pairs.  Words past the row, and rows past M, read
// as 0x4444 (positions 0 and 1: a legal pattern whose values are zero-filled).
__device__ __forceinline__ void load_codes8(const uint16_t *meta, int row, int M, int words_per_row, int w0,
                                            uint32_t (&out)[4]) {
    const uint32_t fill = 0x44444444u;
    out[0] = out[1] = out[2] = out[3] = fill;
    if (row >= M) return;
    const uint16_t *base = meta + (int64_t)row * words_per_row + w0;
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

template <bool SPARSE, bool A_MN, bool B_MN, bool A2_MN, int EPI, int BN>
__global__ void __launch_bounds__(GemmCfg<SPARSE, BN>::NUM_WARPS * 32, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                const GemmParams p) {
    using C = GemmCfg<SPARSE, BN>;
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
            mbar_init(&full[s], SPARSE ? 5 : 1);
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
        if (SPARSE && p.r > 0) {
            tma_prefetch_desc(&tmA2);
            tma_prefetch_desc(&tmB2);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            for (int w = blockIdx.x; w < p.num_work; w += gridDim.x) {
                int mt, nt, sp, k0, k1;
                decode_work(p, w, mt, nt, sp);
                k_range(p, sp, k0, k1);
                const int m0 = mt * C::BM, n0 = nt * BN;
                for (int kt = k0; kt < k1; ++kt) {
                    if (!mbar_wait(&empty[s], ph ^ 1, abort_flag)) goto done;
                    uint8_t *a = smem + s * C::STAGE_BYTES;
                    uint8_t *b = a + C::A_BYTES;
                    if (SPARSE) {
                        mbar_arrive_expect_tx(&full[s], C::A_BYTES + 2 * BN * 128);
                        tma_load_2d(a, &tmA, &full[s], kt * 64, m0);
                        tma_load_2d(b, &tmB, &full[s], kt * 128, n0);
                        tma_load_2d(b + BN * 128, &tmB, &full[s], kt * 128 + 64, n0);
                    } else {
                        mbar_arrive_expect_tx(&full[s], C::A_BYTES + BN * 128);
                        if (A_MN) {
                            tma_load_2d(a, &tmA, &full[s], m0, kt * 64);
                            tma_load_2d(a + 8192, &tmA, &full[s], m0 + 64, kt * 64);
                        } else {
                            tma_load_2d(a, &tmA, &full[s], kt * 64, m0);
                        }
                        if (B_MN) {
#pragma unroll
                            for (int j = 0; j < BN / 64; ++j) tma_load_2d(b + j * 8192, &tmB, &full[s], n0 + 64 * j, kt * 64);
                        } else {
                            tma_load_2d(b, &tmB, &full[s], kt * 64, n0);
                        }
                    }
                    if (++s == NS) { s = 0; ph ^= 1; }
                }
                if (SPARSE && p.r > 0) {
                    for (int kt = 0; kt < p.adp_k_tiles; ++kt) {
                        if (!mbar_wait(&empty[s], ph ^ 1, abort_flag)) goto done;
                        uint8_t *a = smem + s * C::STAGE_BYTES;
                        uint8_t *b = a + C::A_BYTES;
                        mbar_arrive_expect_tx(&full[s], C::A_BYTES + BN * 128);
                        if (A2_MN) {
                            tma_load_2d(a, &tmA2, &full[s], m0, kt * 64);
                            tma_load_2d(a + 8192, &tmA2, &full[s], m0 + 64, kt * 64);
                        } else {
                            tma_load_2d(a, &tmA2, &full[s], kt * 64, m0);
                        }
                        tma_load_2d(b, &tmB2, &full[s], kt * 64, n0);
                        if (++s == NS) { s = 0; ph ^= 1; }
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_SP = instr_desc(128, BN, 0, 0, 1);
            constexpr uint32_t IDESC_DN = instr_desc(128, BN, A_MN ? 1 : 0, B_MN ? 1 : 0, 0);
            constexpr uint32_t IDESC_AD = instr_desc(128, BN, A2_MN ? 1 : 0, 0, 0);
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
                    const uint32_t a_addr = smem_addr(smem + s * C::STAGE_BYTES);
                    const uint32_t b_addr = a_addr + C::A_BYTES;
                    if (SPARSE) {
                        const int nblk = min(4, (p.k_logical - kt * 128) / 32);
                        for (int c = 0; c < nblk; ++c) {
                            const uint64_t ad = smem_desc(a_addr + 32 * c, 16, 1024, SWZ_128B);
                            const uint64_t bd = smem_desc(b_addr + (c >> 1) * (BN * 128) + (c & 1) * 64, 16, 1024, SWZ_128B);
                            const uint32_t e = tmem_base + C::META_COL + s * 4 + c;
                            mma_sp_bf16(d, ad, bd, e & ~1u, IDESC_SP | (e & 1u), accumulate);
                            accumulate = 1;
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const uint64_t ad = A_MN ? smem_desc(a_addr + c * 2048, 8192, 1024, SWZ_128B)
                                                     : smem_desc(a_addr + 32 * c, 16, 1024, SWZ_128B);
                            const uint64_t bd = B_MN ? smem_desc(b_addr + c * 2048, 8192, 1024, SWZ_128B)
                                                     : smem_desc(b_addr + 32 * c, 16, 1024, SWZ_128B);
                            mma_bf16(d, ad, bd, IDESC_DN, accumulate);
                            accumulate = 1;
                        }
                    }
                    mma_commit(&empty[s]);
                    if (++s == NS) { s = 0; ph ^= 1; }
                }
                if (SPARSE && p.r > 0) {
                    for (int kt = 0; kt < p.adp_k_tiles; ++kt) {
                        if (!mbar_wait(&full[s], ph, abort_flag)) goto done;
                        tc_fence_after();
                        const uint32_t a_addr = smem_addr(smem + s * C::STAGE_BYTES);
                        const uint32_t b_addr = a_addr + C::A_BYTES;
                        const int nblk = min(4, (p.r - kt * 64 + 15) / 16);
                        for (int c = 0; c < nblk; ++c) {
                            const uint64_t ad = A2_MN ? smem_desc(a_addr + c * 2048, 8192, 1024, SWZ_128B)
                                                      : smem_desc(a_addr + 32 * c, 16, 1024, SWZ_128B);
                            const uint64_t bd = smem_desc(b_addr + 32 * c, 16, 1024, SWZ_128B);
                            mma_bf16(d, ad, bd, IDESC_AD, accumulate);
                            accumulate = 1;
                        }
                        mma_commit(&empty[s]);
                        if (++s == NS) { s = 0; ph ^= 1; }
                    }
                }
                mma_commit(&acc_full[acc]);
                ++it;
            }
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        int it = 0;
        for (int w = blockIdx.x; w < p.num_work; w += gridDim.x) {
            int mt, nt, sp;
            decode_work(p, w, mt, nt, sp);
            const int acc = it & 1;
            const uint32_t acc_ph = (it >> 1) & 1;
            if (!mbar_wait(&acc_full[acc], acc_ph, abort_flag)) break;
            tc_fence_after();
            const int row = mt * C::BM + 32 * q + lane;
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + acc * BN;
#pragma unroll 1
            for (int cc = 0; cc < BN / 32; ++cc) {
                uint32_t v[32];
                tmem_ld_32x32(taddr + 32 * cc, v);
                tmem_ld_wait();
                if (cc == BN / 32 - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acc_empty[acc]);
                }
                const int n = nt * BN + 32 * cc;  // first column of this chunk
                if (row >= p.M || n >= p.N) continue;
                if (EPI == EPI_BF16_T) {
                    uint16_t *out = reinterpret_cast<uint16_t *>(p.out);
                    const int nmax = min(32, p.N - n);
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (j < nmax) out[(int64_t)(n + j) * p.ld_out + row] = f32_to_bf16_bits(bits_to_f32(v[j]));
                } else if (EPI == EPI_DW_COMPRESS) {
                    // 32 columns = 8 groups = 2 code words of this row of the mask
                    const uint32_t codes =
                        *reinterpret_cast<const uint32_t *>(p.meta_mask + (int64_t)row * (p.N / 16) + n / 16);
                    uint32_t packed[8];
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        const uint32_t code = (codes >> (4 * g)) & 0xFu;
                        const uint32_t i0 = code & 3u, i1 = code >> 2;
                        const uint32_t x0 = i0 == 0 ? v[4 * g] : (i0 == 1 ? v[4 * g + 1] : v[4 * g + 2]);
                        const uint32_t x1 = i1 == 1 ? v[4 * g + 1] : (i1 == 2 ? v[4 * g + 2] : v[4 * g + 3]);
                        packed[g] = static_cast<uint32_t>(f32_to_bf16_bits(bits_to_f32(x0))) |
                                    (static_cast<uint32_t>(f32_to_bf16_bits(bits_to_f32(x1))) << 16);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(p.out) +
                                                           (int64_t)row * p.ld_out + n / 2);
                    dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                    dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
                } else if (EPI == EPI_BF16_ROW) {
                    uint16_t *out = reinterpret_cast<uint16_t *>(p.out) + (int64_t)row * p.ld_out;
                    const int nmax = min(32, p.N - n);
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
                    const int nmax = min(32, p.N - n);
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (j < nmax) atomicAdd(out + n + j, bits_to_f32(v[j]));
                } else {  // EPI_F32_ADD_T
                    float *out = reinterpret_cast<float *>(p.out);
                    const int nmax = min(32, p.N - n);
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (j < nmax) atomicAdd(out + (int64_t)(n + j) * p.ld_out + row, bits_to_f32(v[j]));
                }
            }
            ++it;
        }
    } else if (SPARSE) {
        // ------------------------------------------------------------ code loaders
        // TMEM layout of the position codes read by tcgen05.mma.sp (M = 128,
        // one 32-bit column per MMA of 32 logical K): row m, k-half h of the
        // column lives in lane (m % 8) + 8 h + 16 (m / 16), bits
        // 16 ((m / 8) % 2) .. +15, i.e. each lane packs rows m and m + 8.
        const int q = warp & 3;
        const int L = 32 * q + lane;
        const int mm = 16 * (L >> 4) + (L & 7);
        const int h = (L >> 3) & 1;
        const int words_per_row = p.k_logical / 16;
        int s = 0;
        uint32_t ph = 0;
        for (int w = blockIdx.x; w < p.num_work; w += gridDim.x) {
            int mt, nt, sp, k0, k1;
            decode_work(p, w, mt, nt, sp);
            k_range(p, sp, k0, k1);
            const int rowA = mt * C::BM + mm;
            for (int kt = k0; kt < k1; ++kt) {
                if (!mbar_wait(&empty[s], ph ^ 1, abort_flag)) goto done;
                uint32_t ca[4], cb[4];
                load_codes8(p.meta_a, rowA, p.M, words_per_row, kt * 8, ca);
                load_codes8(p.meta_a, rowA + 8, p.M, words_per_row, kt * 8, cb);
                uint32_t col[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) col[c] = word16(ca, 2 * c + h) | (word16(cb, 2 * c + h) << 16);
                tmem_st_32x32_x4(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + C::META_COL + s * 4, col[0],
                                 col[1], col[2], col[3]);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&full[s]);
                if (++s == NS) { s = 0; ph ^= 1; }
            }
            if (p.r > 0) {
                for (int kt = 0; kt < p.adp_k_tiles; ++kt) {
                    if (!mbar_wait(&empty[s], ph ^ 1, abort_flag)) goto done;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full[s]);
                    if (++s == NS) { s = 0; ph ^= 1; }
                }
            }
        }
    }
done:
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace slope
