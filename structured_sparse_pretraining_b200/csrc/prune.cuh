// prune.cuh -- row-wise 2:4 magnitude pruning (prune24) and the second 2:4
// pruning of the transposed sparse weight (double_prune).
//
// SLoPe technical summary (gist.science), §1 "Structured Sparsity (N:M)" and
// §2.A "Double-Pruned Backward Pass": W^R keeps two of every four
// consecutive weights of a row; W^{R,C} is W^R transposed and pruned 2:4
// again.  Both kernels are memory-bound: they move 3.125 (prune24) and 2.25
// (double_prune) bytes per dense weight and do integer compares only.  The
// double_prune kernel has two fused modes: one AdamW step on the kept values
// ahead of the second pruning (the compressed optimizer step), and the row
// pruning of dense W ahead of it (both prunings in one pass, 4.25 bytes per
// weight).
#pragma once
#include <cuda_bf16.h>
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
            lo[u] = hi[u] = make_uint4(0u, 0u, 0u, 0u);
            if (c < n_chunks && in_bounds(16 * c, 16, 16 * n_chunks)) {
                lo[u] = __ldcs(src + 2 * c);
                hi[u] = __ldcs(src + 2 * c + 1);
            }
        }
#pragma unroll
        for (int u = 0; u < PR_UNROLL; ++u) {
            const int64_t c = base + u * stride;
            if (c < n_chunks && in_bounds(8 * c, 8, 8 * n_chunks)) {
                uint32_t word;
                reinterpret_cast<uint4 *>(vals)[c] = prune16(lo[u], hi[u], word, bad);
                meta[c] = static_cast<uint16_t>(word);
            }
        }
    }
    if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) atomicOr(&g_status, ST_NONFINITE);
}

// General row-wise N:M magnitude pruning (N < M, M = 4, 8 or 16), the form
// without tensor-core support: each kept value's position within its group is
// stored in a byte.  One thread per group of M consecutive weights: each
// element gets the key (magnitude << 4) | (15 - position) (keys are distinct;
// a larger key is a larger magnitude or, on equal magnitudes, the lower
// position), is kept iff fewer than N keys exceed its own, and the kept ones
// are written in ascending position.  A block takes 256 consecutive groups
// per pass: loads are contiguous per warp.  For M = 8 and 16 the block's
// kept values and positions (256 N of each, one contiguous span of both
// outputs) are gathered in shared memory and written out with 16-byte
// stores; for M = 4 each thread writes its group's outputs directly.
constexpr int NM_GROUPS = 256;  // groups per block pass (one per thread)

template <int M>
__global__ void __launch_bounds__(NM_GROUPS) prune_nm_kernel(const uint16_t *__restrict__ W,
                                                             uint16_t *__restrict__ vals, uint8_t *__restrict__ pos,
                                                             int64_t n_groups, int N) {
    __shared__ __align__(16) uint16_t sv[NM_GROUPS * (M - 1)];
    __shared__ __align__(16) uint8_t sp[NM_GROUPS * (M - 1)];
    grid_dep_wait();
    grid_dep_launch();
    bool bad = false;
    const int tid = threadIdx.x;
    for (int64_t g0 = (int64_t)blockIdx.x * NM_GROUPS; g0 < n_groups; g0 += (int64_t)gridDim.x * NM_GROUPS) {
        const int64_t gi = g0 + tid;
        if (gi < n_groups && in_bounds(gi * M, M, n_groups * M) && in_bounds(gi * N, N, n_groups * N)) {
            uint32_t w[M / 2];
            const uint32_t *src = reinterpret_cast<const uint32_t *>(W + gi * M);
            if (M == 4) {
                const uint2 t = *reinterpret_cast<const uint2 *>(src);
                w[0] = t.x;
                w[1] = t.y;
            } else {
#pragma unroll
                for (int q = 0; q < M / 8; ++q) {
                    const uint4 t = reinterpret_cast<const uint4 *>(src)[q];
                    w[4 * q] = t.x;
                    w[4 * q + 1] = t.y;
                    w[4 * q + 2] = t.z;
                    w[4 * q + 3] = t.w;
                }
            }
            uint32_t key[M];
#pragma unroll
            for (int k = 0; k < M; ++k) {
                const uint32_t e = (w[k / 2] >> (16 * (k & 1))) & 0xFFFFu;
                key[k] = ((e & 0x7FFFu) << 4) | (15u - k);
                bad |= (e & 0x7F80u) == 0x7F80u;
            }
            // M = 4: the group's few outputs go straight to global memory
            // (measured faster than staging: a pass moves only 2 KB of input)
            uint16_t *dv = M == 4 ? vals + gi * N : sv + tid * N;
            uint8_t *dp = M == 4 ? pos + gi * N : sp + tid * N;
            int n = 0;
#pragma unroll
            for (int k = 0; k < M; ++k) {
                int above = 0;
#pragma unroll
                for (int j = 0; j < M; ++j) above += key[j] > key[k];
                if (above < N) {
                    dv[n] = static_cast<uint16_t>((w[k / 2] >> (16 * (k & 1))) & 0xFFFFu);
                    dp[n] = static_cast<uint8_t>(k);
                    ++n;
                }
            }
        }
        if (M == 4) continue;
        __syncthreads();
        // the block's span: groups g0 .. g0 + ng of the outputs, contiguous
        const int ng = (int)min((int64_t)NM_GROUPS, n_groups - g0);
        const int64_t o0 = g0 * N;  // first output element of the span
        const int len = ng * N;
        if (!in_bounds(o0, len, n_groups * N)) {
            __syncthreads();
            continue;
        }
        // values: 16-byte stores (8 values) when the span starts on a 16-byte boundary
        if ((o0 & 7) == 0) {
            const int n8 = len / 8;
            for (int i = tid; i < n8; i += NM_GROUPS)
                reinterpret_cast<uint4 *>(vals + o0)[i] = reinterpret_cast<const uint4 *>(sv)[i];
            for (int i = 8 * n8 + tid; i < len; i += NM_GROUPS) vals[o0 + i] = sv[i];
        } else {
            for (int i = tid; i < len; i += NM_GROUPS) vals[o0 + i] = sv[i];
        }
        // positions: 16-byte stores (16 bytes) when the span starts on a 16-byte boundary
        if ((o0 & 15) == 0) {
            const int n16 = len / 16;
            for (int i = tid; i < n16; i += NM_GROUPS)
                reinterpret_cast<uint4 *>(pos + o0)[i] = reinterpret_cast<const uint4 *>(sp)[i];
            for (int i = 16 * n16 + tid; i < len; i += NM_GROUPS) pos[o0 + i] = sp[i];
        } else {
            for (int i = tid; i < len; i += NM_GROUPS) pos[o0 + i] = sp[i];
        }
        __syncthreads();  // the span is written out before the next pass refills it
    }
    if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) atomicOr(&g_status, ST_NONFINITE);
}

// double_prune: tiles of ROWS out-rows (64 or 128) x 64 in-columns of W^R.
//
// Expand: each thread takes one compressed row chunk (16 columns: eight kept
// values and one code word; from dense W, the 16 weights, pruned row-wise
// first as prune24 does and written out as W^R) and writes the dense bf16 row
// chunk (pruned positions = +0) into a shared tile of 32-bit words, each
// holding two adjacent columns.  A group's dense words are two byte permutes of its kept
// pair, with selectors from a 16-entry table indexed by the group's code.
//
// Prune: thread (column pair cp, strip w of 16 out-rows) reads its two
// columns down the strip as 32-bit words, four groups of four rows.  For each
// group the six pairwise magnitude comparisons of both columns come from
// packed 16-bit subtractions: with x_i the word of row i, (x_i | 0x80008000)
// - (x_j & 0x7FFF7FFF) holds 0x8000 + |x_i| - |x_j| in each half (never
// negative, so no borrow crosses halves), whose top bit is |x_i| >= |x_j|.
// For i < j that bit says i beats j (ties go to the lower position), so the
// six bits fix the order of the group, and a 64-entry table maps them to the
// byte selector of the kept pair and its 4-bit code.  Each column gives
// four kept pairs (one 16-byte store into its vals_t row) and one code word.
// Eight consecutive threads are the eight strips of one column pair: their
// stores cover 128 contiguous bytes of two vals_t rows.  The word index of a
// tile row is XORed with 4 x its strip, so a warp's 32 reads (4 column pairs
// x 8 strips) fall in 32 different banks.
//
// The tile is double-buffered in shared memory, and the compressed rows of
// the tile after next are loaded into registers while the current one is
// pruned (two register sets): one barrier per tile.
constexpr int DP_TILE = 64;     // columns of W^R per tile
constexpr int DP_WSTRIDE = 36;  // words per tile row: 32 column pairs + 4 pad (16-byte aligned rows)

__device__ __forceinline__ int dp_word(int row, int word) { return row * DP_WSTRIDE + (word ^ (4 * (row >> 4))); }

// One thread's share of a tile, loaded two tiles ahead: per 64-row half h,
// eight kept values and their code word.  From dense W (the row and column
// prunings in one pass), v holds the row chunk's first eight weights and hi
// its last eight instead.
template <int ROWS, bool ADAM, bool DENSE = false>
struct DpRegs {
    uint4 v[ROWS / 64];
    uint4 hi[DENSE ? ROWS / 64 : 1];
    uint32_t word[ROWS / 64];
};

struct DpAdam;

// One AdamW step on the kept values, fused into the expand phase of the
// second pruning (the tile's kept values are updated, written back with their
// states, and the updated values are what gets pruned again).  The states are
// fp32, one pair per kept value, in the slots of vals.  Every operation is a
// single correctly rounded binary32 operation (no fused multiply-add), in the
// order of the decoupled-decay AdamW step:
//     w <- w * (1 - lr * wd)
//     m <- b1 * m + (1 - b1) * g,   v <- b2 * v + (1 - b2) * (g * g)
//     w <- w - step_size * (m / (sqrt(v) * inv_sqrt_bc2 + eps))
// with step_size = lr / (1 - b1^t) and inv_sqrt_bc2 = 1 / sqrt(1 - b2^t)
// computed on the host in binary64; w is rounded once to bf16.
struct DpAdam {
    uint16_t *vals;        // the kept values, updated in place (the kernel's input)
    const uint16_t *grad;  // compressed gradient, same slots (bf16)
    float *m, *v;          // fp32 states, same slots
    float lr, b1, b2, eps, wd, step_size, inv_sqrt_bc2;
    int64_t n_vals;        // elements of vals, grad, m and v (debug bounds checks)
};

// The row pruning fused ahead of the column pruning: the dense weights it
// reads and the compressed rows (W^R) it writes.
struct DpRowPrune {
    const uint16_t *W;  // [out x in] bf16
    uint16_t *vals;     // [out x in/2]
    uint16_t *meta;     // [out x in/16]
};

template <int ROWS, bool ADAM, bool DENSE>
__device__ __forceinline__ void dp_load(const uint16_t *vals, const uint16_t *__restrict__ meta, int out, int in,
                                        int o0, int i0, int tid, DpRegs<ROWS, ADAM, DENSE> &R, const DpAdam &ad,
                                        const DpRowPrune &rp) {
    const int r = tid >> 2, q = tid & 3;  // 64 rows x 4 chunks of 16 columns per pass
#pragma unroll
    for (int h = 0; h < ROWS / 64; ++h) {
        const int o = o0 + r + 64 * h;
        const int64_t e = (int64_t)o * (in / 2) + i0 / 2 + q * 8;
        R.v[h] = make_uint4(0u, 0u, 0u, 0u);
        R.word[h] = 0x4444u;
        if (DENSE) {  // 16 dense weights of row o (streamed once: bypass L1)
            const int64_t dw = (int64_t)o * in + i0 + 16 * q;
            R.hi[DENSE ? h : 0] = make_uint4(0u, 0u, 0u, 0u);
            if (!in_bounds(dw, 16, (int64_t)out * in)) continue;
            const uint4 *src = reinterpret_cast<const uint4 *>(rp.W + dw);
            R.v[h] = __ldcs(src);
            R.hi[DENSE ? h : 0] = __ldcs(src + 1);
            continue;
        }
        if (!in_bounds(e, 8, (int64_t)out * (in / 2))) continue;
        R.v[h] = *reinterpret_cast<const uint4 *>(vals + e);
        R.word[h] = meta[(int64_t)o * (in / 16) + i0 / 16 + q];
    }
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t adamw_pair(uint32_t w2, uint32_t g2, float *m, float *v, const DpAdam &a) {
    const float decay = __fsub_rn(1.0f, __fmul_rn(a.lr, a.wd));
    const float omb1 = __fsub_rn(1.0f, a.b1), omb2 = __fsub_rn(1.0f, a.b2);
    uint32_t out = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const float g = h ? bf16_hi(g2) : bf16_lo(g2);
        float w = __fmul_rn(h ? bf16_hi(w2) : bf16_lo(w2), decay);
        const float mk = __fadd_rn(__fmul_rn(a.b1, m[h]), __fmul_rn(omb1, g));
        const float vk = __fadd_rn(__fmul_rn(a.b2, v[h]), __fmul_rn(omb2, __fmul_rn(g, g)));
        const float denom = __fadd_rn(__fmul_rn(__fsqrt_rn(vk), a.inv_sqrt_bc2), a.eps);
        w = __fsub_rn(w, __fmul_rn(a.step_size, __fdiv_rn(mk, denom)));
        m[h] = mk;
        v[h] = vk;
        out |= static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(w))) << (16 * h);
    }
    return out;
}

// The AdamW step on one thread's 8 kept values (row chunk at element offset e of vals).
__device__ __forceinline__ void dp_adamw8(uint32_t (&kv)[4], int64_t e, const DpAdam &a) {
    const uint4 g = *reinterpret_cast<const uint4 *>(a.grad + e);
    float4 *mp = reinterpret_cast<float4 *>(a.m + e);
    float4 *vp = reinterpret_cast<float4 *>(a.v + e);
    const float4 m0 = mp[0], m1 = mp[1], v0 = vp[0], v1 = vp[1];
    float m[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
    float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) kv[k] = adamw_pair(kv[k], gw[k], m + 2 * k, v + 2 * k, a);
    *reinterpret_cast<uint4 *>(a.vals + e) = make_uint4(kv[0], kv[1], kv[2], kv[3]);
    mp[0] = make_float4(m[0], m[1], m[2], m[3]);
    mp[1] = make_float4(m[4], m[5], m[6], m[7]);
    vp[0] = make_float4(v[0], v[1], v[2], v[3]);
    vp[1] = make_float4(v[4], v[5], v[6], v[7]);
}

template <int ROWS, bool ADAM, bool DENSE>
__device__ __forceinline__ void dp_expand(uint32_t *tilew, const uint32_t *lut, int tid,
                                          const DpRegs<ROWS, ADAM, DENSE> &R, const DpAdam &ad, const DpRowPrune &rp,
                                          int out, int in, int o0, int i0, bool &bad) {
    const int r = tid >> 2, q = tid & 3;
#pragma unroll
    for (int h = 0; h < ROWS / 64; ++h) {
        uint4 kept = R.v[h];
        uint32_t word = R.word[h];
        if (DENSE) {
            // the row pruning of these 16 weights: kept pair and code of each group, written out as W^R
            kept = prune16(R.v[h], R.hi[DENSE ? h : 0], word, bad);
            const int o = o0 + r + 64 * h;
            const int64_t e = (int64_t)o * (in / 2) + i0 / 2 + q * 8;
            if (in_bounds(e, 8, (int64_t)out * (in / 2))) {
                *reinterpret_cast<uint4 *>(rp.vals + e) = kept;
                rp.meta[(int64_t)o * (in / 16) + i0 / 16 + q] = static_cast<uint16_t>(word);
            }
        }
        uint32_t kv[4] = {kept.x, kept.y, kept.z, kept.w};
        if (ADAM && in_bounds((int64_t)(o0 + r + 64 * h) * (in / 2) + i0 / 2 + q * 8, 8, ad.n_vals))
            dp_adamw8(kv, (int64_t)(o0 + r + 64 * h) * (in / 2) + i0 / 2 + q * 8, ad);
        uint32_t d[8];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const uint32_t sel = lut[(word >> (4 * g)) & 0xFu];
            d[2 * g] = __byte_perm(kv[g], 0u, sel & 0xFFFFu);
            d[2 * g + 1] = __byte_perm(kv[g], 0u, sel >> 16);
        }
        // words q*8 .. q*8+7 of the row; the swizzle keeps each half 4-word aligned
        const int row = r + 64 * h;
        *reinterpret_cast<uint4 *>(tilew + dp_word(row, q * 8)) = make_uint4(d[0], d[1], d[2], d[3]);
        *reinterpret_cast<uint4 *>(tilew + dp_word(row, q * 8 + 4)) = make_uint4(d[4], d[5], d[6], d[7]);
    }
}

// Table entry for the comparison bits p of a group (bit 0: |x0| >= |x1|,
// then 0-2, 0-3, 1-2, 1-3, 2-3; for i < j the bit says position i beats j):
// the byte selector of the two kept values over the group's words (w01 =
// elements 0 | 1 << 16, w23 = 2 | 3 << 16) in the low half, the code
// i0 | i1 << 2 (i0 < i1) above it.  Element i beats as many others as the
// rank count says; the two with fewer than two winners over them are kept.
// Patterns that no order produces (cycles) get positions 0 and 1.
__device__ __forceinline__ uint32_t dp_rank_entry(uint32_t pat) {
    const uint32_t b01 = pat & 1u, b02 = (pat >> 1) & 1u, b03 = (pat >> 2) & 1u;
    const uint32_t b12 = (pat >> 3) & 1u, b13 = (pat >> 4) & 1u, b23 = (pat >> 5) & 1u;
    const uint32_t beaten[4] = {(1u - b01) + (1u - b02) + (1u - b03), b01 + (1u - b12) + (1u - b13),
                                b02 + b12 + (1u - b23), b03 + b13 + b23};
    uint32_t i0 = 4, i1 = 4;
    for (uint32_t i = 0; i < 4; ++i) {
        if (beaten[i] < 2) {
            if (i0 == 4) i0 = i;
            else if (i1 == 4) i1 = i;
        }
    }
    if (i1 == 4) {
        i0 = 0;
        i1 = 1;
    }
    const uint32_t sel = (i0 * 0x22u + 0x10u) | ((i1 * 0x22u + 0x10u) << 8);
    return sel | ((i0 | (i1 << 2)) << 16);
}

template <int ROWS, bool ADAM, bool DENSE = false>
__global__ void __launch_bounds__(256) double_prune_kernel(const uint16_t *vals, const uint16_t *__restrict__ meta,
                                                           int out, int in, uint16_t *__restrict__ vals_t,
                                                           uint16_t *__restrict__ meta_t, const DpAdam ad,
                                                           const DpRowPrune rp) {
    static_assert(!(ADAM && DENSE), "the AdamW step and the row pruning are separate modes");
    __shared__ __align__(16) uint32_t tilew[2][ROWS * DP_WSTRIDE];
    __shared__ uint32_t lut[16];
    __shared__ uint32_t rank_lut[4 * 64];  // one copy per group of a strip, the code placed for it
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
    {
        const uint32_t e = dp_rank_entry((uint32_t)(tid & 63));
        const int g = tid >> 6;  // 256 threads: four tables of 64
        rank_lut[tid] = (e & 0xFFFFu) | ((e >> 16) << (16 + 4 * g));
    }
    __syncthreads();
    grid_dep_wait();
    grid_dep_launch();
    const int n_in_tiles = in / DP_TILE;
    const int tiles = (out / ROWS) * n_in_tiles;
    constexpr int STRIPS = ROWS / 16;            // strips of 16 rows (four groups)
    const int cp = tid >> 3, w = tid & 7;        // prune phase: column pair, strip
    // Prune tile t from shared buffer buf (after the barrier that follows its expand).
    auto prune_tile = [&](const uint32_t *tw, int t) {
        if (w >= STRIPS) return;
        const int o0 = (t / n_in_tiles) * ROWS;
        const int i0 = (t % n_in_tiles) * DP_TILE;
        const uint32_t *col = tw + dp_word(16 * w, cp);  // rows 16 w .. 16 w + 15, word cp
        uint32_t kept_lo[4], kept_hi[4];
        uint32_t code_lo = 0, code_hi = 0;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const uint32_t *e = col + 4 * g * DP_WSTRIDE;
            const uint32_t x0 = e[0], x1 = e[DP_WSTRIDE], x2 = e[2 * DP_WSTRIDE], x3 = e[3 * DP_WSTRIDE];
            const uint32_t h0 = x0 | 0x80008000u, h1 = x1 | 0x80008000u, h2 = x2 | 0x80008000u;
            const uint32_t m1 = x1 & 0x7FFF7FFFu, m2 = x2 & 0x7FFF7FFFu, m3 = x3 & 0x7FFF7FFFu;
            const uint32_t pat = ((h0 - m1) >> 15 & 0x00010001u) | ((h0 - m2) >> 14 & 0x00020002u) |
                                 ((h0 - m3) >> 13 & 0x00040004u) | ((h1 - m2) >> 12 & 0x00080008u) |
                                 ((h1 - m3) >> 11 & 0x00100010u) | ((h2 - m3) >> 10 & 0x00200020u);
            // entry: byte selector in bits 0-15 (a byte permute reads only
            // those), the code in bits 16 + 4 g .. 19 + 4 g of table g
            const uint32_t ent_lo = rank_lut[g * 64 + (pat & 0x3Fu)], ent_hi = rank_lut[g * 64 + (pat >> 16)];
            kept_lo[g] = __byte_perm(__byte_perm(x0, x1, 0x5410u), __byte_perm(x2, x3, 0x5410u), ent_lo);
            kept_hi[g] = __byte_perm(__byte_perm(x0, x1, 0x7632u), __byte_perm(x2, x3, 0x7632u), ent_hi);
            code_lo |= ent_lo & (0xF0000u << (4 * g));
            code_hi |= ent_hi & (0xF0000u << (4 * g));
        }
        code_lo >>= 16;
        code_hi >>= 16;
        const int i = i0 + 2 * cp;  // the low column; the high one is i + 1
        uint16_t *vrow = vals_t + (int64_t)i * (out / 2) + o0 / 2 + 8 * w;
        if (!in_bounds((int64_t)i * (out / 2) + o0 / 2 + 8 * w + out / 2, 8, (int64_t)in * (out / 2)) ||
            !in_bounds((int64_t)i * (out / 16) + o0 / 16 + w + out / 16, 1, (int64_t)in * (out / 16)))
            return;
        *reinterpret_cast<uint4 *>(vrow) = make_uint4(kept_lo[0], kept_lo[1], kept_lo[2], kept_lo[3]);
        *reinterpret_cast<uint4 *>(vrow + out / 2) = make_uint4(kept_hi[0], kept_hi[1], kept_hi[2], kept_hi[3]);
        uint16_t *mrow = meta_t + (int64_t)i * (out / 16) + o0 / 16 + w;
        mrow[0] = static_cast<uint16_t>(code_lo);
        mrow[out / 16] = static_cast<uint16_t>(code_hi);
    };
    auto load_tile = [&](int t, DpRegs<ROWS, ADAM, DENSE> &R) {
        dp_load<ROWS, ADAM, DENSE>(vals, meta, out, in, (t / n_in_tiles) * ROWS, (t % n_in_tiles) * DP_TILE, tid, R, ad,
                                   rp);
    };
    // Two register sets of compressed rows (and AdamW operands): the loads run two tiles ahead.
    DpRegs<ROWS, ADAM, DENSE> ra, rb;
    bool bad = false;
    const int stride = gridDim.x;
    int t = blockIdx.x;
    if (t < tiles) load_tile(t, ra);
    if (t + stride < tiles) load_tile(t + stride, rb);
    for (int buf = 0; t < tiles;) {
        dp_expand<ROWS, ADAM, DENSE>(tilew[buf], lut, tid, ra, ad, rp, out, in, (t / n_in_tiles) * ROWS,
                                     (t % n_in_tiles) * DP_TILE, bad);
        if (t + 2 * stride < tiles) load_tile(t + 2 * stride, ra);
        __syncthreads();
        prune_tile(tilew[buf], t);
        t += stride;
        buf ^= 1;
        if (t >= tiles) break;
        dp_expand<ROWS, ADAM, DENSE>(tilew[buf], lut, tid, rb, ad, rp, out, in, (t / n_in_tiles) * ROWS,
                                     (t % n_in_tiles) * DP_TILE, bad);
        if (t + 2 * stride < tiles) load_tile(t + 2 * stride, rb);
        __syncthreads();
        prune_tile(tilew[buf], t);
        t += stride;
        buf ^= 1;
    }
    if (DENSE && __any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) atomicOr(&g_status, ST_NONFINITE);
}

}  // namespace slope
