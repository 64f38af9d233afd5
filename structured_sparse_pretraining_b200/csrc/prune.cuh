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

// Top two of one group of four bf16 patterns, given as two words (w01 holds
// elements 0 | 1 << 16, w23 elements 2 | 3 << 16).  Each element gets the key
// (magnitude << 2) | (3 - position): keys are distinct, and a larger key is a
// larger magnitude or, on equal magnitudes (+0 == -0), the lower position.
// The kept pair is the two largest keys.  Returns the pair's values as one
// word (lower position in the low half), the 4-bit code i0 | i1 << 2
// (i0 < i1), and the group's largest key (>= 0x1FE00 iff the group holds an
// Inf or NaN, whose magnitude bits are >= 0x7F80).
__device__ __forceinline__ uint32_t top2_of4(uint32_t w01, uint32_t w23, uint32_t &code, uint32_t &maxkey) {
    const uint32_t k0 = ((w01 << 2) & 0x1FFFCu) | 3u;
    const uint32_t k1 = ((w01 >> 14) & 0x1FFFCu) | 2u;
    const uint32_t k2 = ((w23 << 2) & 0x1FFFCu) | 1u;
    const uint32_t k3 = (w23 >> 14) & 0x1FFFCu;
    const uint32_t hi01 = max(k0, k1), lo01 = min(k0, k1);
    const uint32_t hi23 = max(k2, k3), lo23 = min(k2, k3);
    const uint32_t first = max(hi01, hi23);
    const uint32_t second = max(min(hi01, hi23), max(lo01, lo23));
    const uint32_t ia = 3u - (first & 3u), ib = 3u - (second & 3u);
    const uint32_t i0 = min(ia, ib), i1 = max(ia, ib);
    code = i0 | (i1 << 2);
    maxkey = first;
    // byte selector over the group's 8 bytes (w01: bytes 0..3, w23: 4..7):
    // element i is bytes 2i, 2i+1
    return __byte_perm(w01, w23, (i0 * 0x22u + 0x10u) | ((i1 * 0x22u + 0x10u) << 8));
}

constexpr uint32_t kNonfiniteKey = 0x7F80u << 2;

// Four groups of a row (16 weights, two 16-byte words) -> eight kept values
// and one 16-bit code word.
__device__ __forceinline__ uint4 prune16(const uint4 lo, const uint4 hi, uint32_t &word, bool &bad) {
    const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    uint32_t out[4];
    uint32_t mk = 0;
    word = 0;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        uint32_t code, maxkey;
        out[g] = top2_of4(w[2 * g], w[2 * g + 1], code, maxkey);
        word |= code << (4 * g);
        mk = max(mk, maxkey);
    }
    bad |= mk >= kNonfiniteKey;
    return make_uint4(out[0], out[1], out[2], out[3]);
}

// One thread per 16 consecutive weights of a row (a chunk: four groups): two
// 16-byte loads, one 16-byte store of the eight kept values, one 16-bit code
// word.  Consecutive threads take consecutive chunks, so every access of a
// warp is contiguous.  Each thread takes PR_UNROLL chunks a grid-stride apart
// per pass and issues all their loads before any compute, which keeps enough
// bytes in flight per SM to run at HBM speed.
constexpr int PR_UNROLL = 4;

__global__ void __launch_bounds__(256) prune24_kernel(const uint16_t *__restrict__ W, uint16_t *__restrict__ vals,
                                                      uint16_t *__restrict__ meta, int64_t n_chunks) {
    grid_dep_wait();
    grid_dep_launch();
    bool bad = false;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const uint4 *src = reinterpret_cast<const uint4 *>(W);
    for (int64_t base = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; base < n_chunks; base += PR_UNROLL * stride) {
        uint4 lo[PR_UNROLL], hi[PR_UNROLL];
#pragma unroll
        for (int u = 0; u < PR_UNROLL; ++u) {
            const int64_t c = base + u * stride;
            if (c < n_chunks) {
                lo[u] = __ldcs(src + 2 * c);
                hi[u] = __ldcs(src + 2 * c + 1);
            }
        }
#pragma unroll
        for (int u = 0; u < PR_UNROLL; ++u) {
            const int64_t c = base + u * stride;
            if (c < n_chunks) {
                uint32_t word;
                reinterpret_cast<uint4 *>(vals)[c] = prune16(lo[u], hi[u], word, bad);
                meta[c] = static_cast<uint16_t>(word);
            }
        }
    }
    if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) atomicOr(&g_status, ST_NONFINITE);
}

// double_prune: tiles of ROWS out-rows (64 or 128) x 64 in-columns of W^R.
//
// Expand: each thread takes one compressed row chunk (16 columns: eight kept
// values and one code word) and writes the dense bf16 row chunk (pruned
// positions = +0) into a shared tile of 32-bit words, each holding two
// adjacent columns.  A group's dense words are two byte permutes of its kept
// pair, with selectors from a 16-entry table indexed by the group's code.
//
// Prune: thread (column c, strip w of ROWS / 4 out-rows) reads its column
// down the strip, ROWS / 16 groups of four, and keeps the top two of each:
// ROWS / 8 kept values (16-byte stores into row i of vals_t) and ROWS / 64
// code words of meta_t.  Four consecutive threads cover one vals_t row
// segment (contiguous bytes).  The word index of a tile row is XORed with 8 x
// its strip, so the four strips' reads of a warp fall in different banks.
//
// The tile is double-buffered and the next tile's compressed rows are loaded
// into registers while the current one is pruned: one barrier per tile.
constexpr int DP_TILE = 64;     // columns of W^R per tile
constexpr int DP_WSTRIDE = 36;  // words per tile row: 32 column pairs + 4 pad (16-byte aligned rows)

template <int ROWS>
__device__ __forceinline__ int dp_word(int row, int word) {
    return row * DP_WSTRIDE + (word ^ (8 * (row / (ROWS / 4))));
}

template <int ROWS>
__device__ __forceinline__ void dp_load(const uint16_t *__restrict__ vals, const uint16_t *__restrict__ meta, int in,
                                        int o0, int i0, int tid, uint4 (&v)[ROWS / 64], uint32_t (&word)[ROWS / 64]) {
    const int r = tid >> 2, q = tid & 3;  // 64 rows x 4 chunks of 16 columns per pass
#pragma unroll
    for (int h = 0; h < ROWS / 64; ++h) {
        const int o = o0 + r + 64 * h;
        v[h] = *reinterpret_cast<const uint4 *>(vals + (int64_t)o * (in / 2) + i0 / 2 + q * 8);
        word[h] = meta[(int64_t)o * (in / 16) + i0 / 16 + q];
    }
}

template <int ROWS>
__device__ __forceinline__ void dp_expand(uint32_t *tilew, const uint32_t *lut, int tid, const uint4 (&v)[ROWS / 64],
                                          const uint32_t (&word)[ROWS / 64]) {
    const int r = tid >> 2, q = tid & 3;
#pragma unroll
    for (int h = 0; h < ROWS / 64; ++h) {
        const uint32_t kv[4] = {v[h].x, v[h].y, v[h].z, v[h].w};
        uint32_t d[8];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const uint32_t sel = lut[(word[h] >> (4 * g)) & 0xFu];
            d[2 * g] = __byte_perm(kv[g], 0u, sel & 0xFFFFu);
            d[2 * g + 1] = __byte_perm(kv[g], 0u, sel >> 16);
        }
        // words q*8 .. q*8+7 of the row; the swizzle keeps each half 4-word aligned
        const int row = r + 64 * h;
        *reinterpret_cast<uint4 *>(tilew + dp_word<ROWS>(row, q * 8)) = make_uint4(d[0], d[1], d[2], d[3]);
        *reinterpret_cast<uint4 *>(tilew + dp_word<ROWS>(row, q * 8 + 4)) = make_uint4(d[4], d[5], d[6], d[7]);
    }
}

template <int ROWS>
__global__ void __launch_bounds__(256) double_prune_kernel(const uint16_t *__restrict__ vals,
                                                           const uint16_t *__restrict__ meta, int out, int in,
                                                           uint16_t *__restrict__ vals_t,
                                                           uint16_t *__restrict__ meta_t) {
    __shared__ __align__(16) uint32_t tilew[2][ROWS * DP_WSTRIDE];
    __shared__ uint32_t lut[16];
    const int tid = threadIdx.x;
    if (tid < 16) {
        // code c keeps positions p0 = c & 3 and p1 = c >> 2: dense element k
        // takes bytes 0-1 (x0) if k == p0, 2-3 (x1) if k == p1, else 4-5 (zero)
        const uint32_t p0 = tid & 3u, p1 = (uint32_t)tid >> 2;
        uint32_t sel = 0;
#pragma unroll
        for (uint32_t k = 0; k < 4; ++k) {
            const uint32_t src = k == p0 ? 0u : (k == p1 ? 2u : 4u);
            sel |= (src * 0x11u + 0x10u) << (8 * k);
        }
        lut[tid] = sel;
    }
    __syncthreads();
    grid_dep_wait();
    grid_dep_launch();
    const int n_in_tiles = in / DP_TILE;
    const int tiles = (out / ROWS) * n_in_tiles;
    uint4 v[ROWS / 64];
    uint32_t word[ROWS / 64];
    int t = blockIdx.x;
    if (t < tiles) dp_load<ROWS>(vals, meta, in, (t / n_in_tiles) * ROWS, (t % n_in_tiles) * DP_TILE, tid, v, word);
    const int c = tid >> 2, w = tid & 3;  // prune phase: column c, strip w
    constexpr int SR = ROWS / 4;          // rows per strip
    constexpr int G = SR / 4;             // groups per strip
    for (int buf = 0; t < tiles; t += gridDim.x, buf ^= 1) {
        const int o0 = (t / n_in_tiles) * ROWS;
        const int i0 = (t % n_in_tiles) * DP_TILE;
        dp_expand<ROWS>(tilew[buf], lut, tid, v, word);
        const int tn = t + gridDim.x;  // prefetch the next tile's compressed rows
        if (tn < tiles) dp_load<ROWS>(vals, meta, in, (tn / n_in_tiles) * ROWS, (tn % n_in_tiles) * DP_TILE, tid, v, word);
        __syncthreads();
        // the column's half-words: word (c / 2) ^ 8 w of each strip row, half c % 2
        const uint16_t *colp = reinterpret_cast<const uint16_t *>(tilew[buf] + w * SR * DP_WSTRIDE + ((c >> 1) ^ (8 * w))) + (c & 1);
        uint32_t kept[G];
        uint32_t words[G / 4];
#pragma unroll
        for (int k = 0; k < G / 4; ++k) words[k] = 0;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const uint16_t *e = colp + (4 * g) * DP_WSTRIDE * 2;
            const uint32_t w01 = (uint32_t)e[0] | ((uint32_t)e[DP_WSTRIDE * 2] << 16);
            const uint32_t w23 = (uint32_t)e[DP_WSTRIDE * 4] | ((uint32_t)e[DP_WSTRIDE * 6] << 16);
            uint32_t code, mk;
            kept[g] = top2_of4(w01, w23, code, mk);
            words[g / 4] |= code << (4 * (g % 4));
        }
        const int i = i0 + c;
        uint16_t *vrow = vals_t + (int64_t)i * (out / 2) + o0 / 2 + w * (SR / 2);
#pragma unroll
        for (int k = 0; k < G / 4; ++k)
            reinterpret_cast<uint4 *>(vrow)[k] = make_uint4(kept[4 * k], kept[4 * k + 1], kept[4 * k + 2], kept[4 * k + 3]);
        uint16_t *mrow = meta_t + (int64_t)i * (out / 16) + o0 / 16 + w * (SR / 16);
#pragma unroll
        for (int k = 0; k < G / 4; ++k) mrow[k] = static_cast<uint16_t>(words[k]);
    }
}

}  // namespace slope
