// prune.cuh -- row-wise 2:4 magnitude pruning (prune24) and the second 2:4
// pruning of the transposed sparse weight (double_prune).
//
// SLoPe technical summary (gist.science), §1 "Structured Sparsity (N:M)" and
// §2.A "Double-Pruned Backward Pass": W^R keeps two of every four
// consecutive weights of a row; W^{R,C} is W^R transposed and pruned 2:4
// again.  Both kernels are memory-bound: they move 3.125 (prune24) and 2.25
// (double_prune) bytes per dense weight and do integer compares only.
#pragma once
#include <cstdint>
#include "ptx.cuh"

namespace slope {

// Kept positions of one group of four bf16 patterns: the two largest
// magnitudes, ties to the lower position (+0 == -0).  Returns the 4-bit code
// i0 | i1 << 2 (i0 < i1).
__device__ __forceinline__ uint32_t top2_code(uint32_t v0, uint32_t v1, uint32_t v2, uint32_t v3) {
    const uint32_t a0 = v0 & 0x7FFFu, a1 = v1 & 0x7FFFu, a2 = v2 & 0x7FFFu, a3 = v3 & 0x7FFFu;
    // element k is beaten by m when a_m > a_k, or a_m == a_k and m < k
    const uint32_t b0 = (a1 > a0) + (a2 > a0) + (a3 > a0);
    const uint32_t b1 = (a0 >= a1) + (a2 > a1) + (a3 > a1);
    const uint32_t b2 = (a0 >= a2) + (a1 >= a2) + (a3 > a2);
    const uint32_t b3 = (a0 >= a3) + (a1 >= a3) + (a2 >= a3);
    const uint32_t keep = (b0 < 2u) | ((b1 < 2u) << 1) | ((b2 < 2u) << 2) | ((b3 < 2u) << 3);
    const uint32_t i0 = __ffs(keep) - 1;
    const uint32_t i1 = 31 - __clz(keep);
    return i0 | (i1 << 2);
}

__device__ __forceinline__ uint32_t pick4(uint32_t v0, uint32_t v1, uint32_t v2, uint32_t v3, uint32_t i) {
    return i == 0 ? v0 : (i == 1 ? v1 : (i == 2 ? v2 : v3));
}

__device__ __forceinline__ bool nonfinite_bf16(uint32_t v) { return (v & 0x7F80u) == 0x7F80u; }

// One thread per 16 consecutive weights of a row (four groups): two 16-byte
// loads, one 16-byte store of the eight kept values, one 16-bit code word.
// Consecutive threads take consecutive 16-weight chunks, so every access of
// a warp is contiguous.  Grid-stride over all chunks.
__global__ void __launch_bounds__(256) prune24_kernel(const uint16_t *__restrict__ W, uint16_t *__restrict__ vals,
                                                      uint16_t *__restrict__ meta, int64_t n_chunks) {
    grid_dep_wait();
    grid_dep_launch();
    bool bad = false;
    for (int64_t c = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; c < n_chunks;
         c += (int64_t)gridDim.x * blockDim.x) {
        const uint4 *src = reinterpret_cast<const uint4 *>(W) + 2 * c;
        const uint4 lo = __ldcs(src), hi = __ldcs(src + 1);
        const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
        uint32_t out[4];
        uint32_t word = 0;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const uint32_t e0 = w[2 * g] & 0xFFFFu, e1 = w[2 * g] >> 16;
            const uint32_t e2 = w[2 * g + 1] & 0xFFFFu, e3 = w[2 * g + 1] >> 16;
            bad |= nonfinite_bf16(e0) | nonfinite_bf16(e1) | nonfinite_bf16(e2) | nonfinite_bf16(e3);
            const uint32_t code = top2_code(e0, e1, e2, e3);
            const uint32_t k0 = pick4(e0, e1, e2, e3, code & 3u);
            const uint32_t k1 = pick4(e0, e1, e2, e3, code >> 2);
            out[g] = k0 | (k1 << 16);
            word |= code << (4 * g);
        }
        reinterpret_cast<uint4 *>(vals)[c] = make_uint4(out[0], out[1], out[2], out[3]);
        meta[c] = static_cast<uint16_t>(word);
    }
    if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) atomicOr(&g_status, ST_NONFINITE);
}

// double_prune: tiles of 64 out-rows x 64 in-columns of W^R.  The compressed
// rows are expanded into a dense 64x64 bf16 tile in shared memory (pruned
// positions = +0), then each thread prunes one (column i, 16 out-rows) strip:
// four groups along out -> eight kept values (one 16-byte store into row i of
// vals_t) and one 16-bit code word of meta_t.  Four consecutive threads write
// 64 contiguous bytes of a vals_t row.
constexpr int DP_TILE = 64;

__global__ void __launch_bounds__(256) double_prune_kernel(const uint16_t *__restrict__ vals,
                                                           const uint16_t *__restrict__ meta, int out, int in,
                                                           uint16_t *__restrict__ vals_t,
                                                           uint16_t *__restrict__ meta_t) {
    __shared__ uint16_t tile[DP_TILE][DP_TILE + 2];  // +2 keeps column reads off one bank
    grid_dep_wait();
    grid_dep_launch();
    const int n_in_tiles = in / DP_TILE;
    const int tiles = (out / DP_TILE) * n_in_tiles;
    const int tid = threadIdx.x;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int o0 = (t / n_in_tiles) * DP_TILE;
        const int i0 = (t % n_in_tiles) * DP_TILE;
        // expand: each thread takes one row o and 16 columns (4 groups):
        // 8 kept values (16 B) + one code word
        {
            const int r = tid >> 2, q = tid & 3;  // 64 rows x 4 chunks of 16 columns
            const int o = o0 + r;
            const uint4 v = *reinterpret_cast<const uint4 *>(vals + (int64_t)o * (in / 2) + i0 / 2 + q * 8);
            const uint32_t word = meta[(int64_t)o * (in / 16) + i0 / 16 + q];
            const uint32_t kv[4] = {v.x, v.y, v.z, v.w};
            uint32_t dense[8];
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const uint32_t code = (word >> (4 * g)) & 0xFu;
                const uint32_t p0 = code & 3u, p1 = code >> 2;
                const uint32_t x0 = kv[g] & 0xFFFFu, x1 = kv[g] >> 16;
                uint32_t e[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) e[k] = (k == (int)p0) ? x0 : ((k == (int)p1) ? x1 : 0u);
                dense[2 * g] = e[0] | (e[1] << 16);
                dense[2 * g + 1] = e[2] | (e[3] << 16);
            }
            uint32_t *row = reinterpret_cast<uint32_t *>(&tile[r][q * 16]);
#pragma unroll
            for (int k = 0; k < 8; ++k) row[k] = dense[k];
        }
        __syncthreads();
        // prune down the columns: thread -> (column c, strip w of 16 out-rows)
        {
            const int c = tid >> 2, w = tid & 3;
            uint32_t kept[4];
            uint32_t word = 0;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const int rb = w * 16 + g * 4;
                const uint32_t e0 = tile[rb][c], e1 = tile[rb + 1][c], e2 = tile[rb + 2][c], e3 = tile[rb + 3][c];
                const uint32_t code = top2_code(e0, e1, e2, e3);
                kept[g] = pick4(e0, e1, e2, e3, code & 3u) | (pick4(e0, e1, e2, e3, code >> 2) << 16);
                word |= code << (4 * g);
            }
            const int i = i0 + c;
            *reinterpret_cast<uint4 *>(vals_t + (int64_t)i * (out / 2) + o0 / 2 + w * 8) =
                make_uint4(kept[0], kept[1], kept[2], kept[3]);
            meta_t[(int64_t)i * (out / 16) + o0 / 16 + w] = static_cast<uint16_t>(word);
        }
        __syncthreads();
    }
}

}  // namespace slope
