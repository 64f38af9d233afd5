// skinny.cuh -- the rank-r token products (XL = X . L, G = dY . R^T) at few
// tokens, on CUDA cores.
//
// With a handful of tokens these products are tiny (T x K x r multiply-adds)
// and bound by reading the rank-r factor once; a tensor-core tile would idle
// on 64 or 128 token rows that do not exist.  Each CTA takes a block of 4 or
// 16 tokens and a set of K chunks: it stages the chunk of A (block x kc) and
// of B (kc x r,
// transposed on the way in when B is stored [r x K]) in shared memory,
// accumulates its 16 x r fp32 partial with every thread owning two columns
// and a stride of k, sums the k-groups in order, and writes the partial to
// its split's workspace slot.  The CTA that arrives last for its 16 tokens
// sums the slots in split order and rounds once to bf16.  Every sum runs in a
// fixed order, so results do not depend on timing.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "ptx.cuh"

namespace slope {

struct SkinnyParams {
    const uint16_t *A;  // [T x K] bf16, row-major
    const uint16_t *B;  // K x r bf16 as [K x r] (B_MN) or [r x K], row-major
    int T, K, r;
    int kc;             // K per chunk (multiple of 64)
    int chunks;         // ceil(K / kc)
    int splits;         // CTAs per token block; CTA s takes chunks s, s + splits, ...
    int tok;            // tokens per block (4 or 16)
    uint16_t *out;      // [T x r] bf16
    float *ws;          // partials [token block][split][16][r] fp32 (the first tok rows used)
    int *count;         // arrivals per token block, left at 0
    float *zero0;       // optional fp32 buffers cleared before any work (outputs
    int64_t zero_n0;    // of later launches that accumulate)
    float *zero1;
    int64_t zero_n1;
    int64_t ext_A, ext_B, ext_out, ext_ws, ext_count;  // elements of each buffer (debug bounds checks)
};

constexpr int SKINNY_THREADS = 256;

// 16-byte global -> shared copy that does not hold a register (cp.async,
// cached in L2 only); src_bytes = 0 writes 16 zero bytes (src must still be
// a valid address).
__device__ __forceinline__ void cp_async16(void *dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}
constexpr int SKINNY_TOK = 16;

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// Four consecutive outputs (element e = t * r + j of this token block) as bf16.
__device__ __forceinline__ void skinny_store4(const SkinnyParams &p, int t0, int e, float4 v) {
    const int t = e / p.r, j = e % p.r;
    const uint32_t lo = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v.x))) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v.y))) << 16);
    const uint32_t hi = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v.z))) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v.w))) << 16);
    if (in_bounds((int64_t)(t0 + t) * p.r + j, 4, p.ext_out))
        *reinterpret_cast<uint2 *>(p.out + (int64_t)(t0 + t) * p.r + j) = make_uint2(lo, hi);
}

// One staged chunk: k pairs kk, kk + 1 with kk = 2 kg, 2 kg + 2 KG, ...; the
// ROWS token values of a k pair are loaded before their multiply-adds.
template <int ROWS>
__device__ __forceinline__ void skinny_chunk(float (&acc)[SKINNY_TOK][2], const uint32_t *As, const uint32_t *Bs,
                                             int aw, int NP, int KG, int jp, int kg, int kn) {
#pragma unroll 2
    for (int kk = 2 * kg; kk < kn; kk += 2 * KG) {
        const float2 b0 = bf16x2_to_float2(Bs[kk * NP + jp]);
        const float2 b1 = bf16x2_to_float2(Bs[(kk + 1) * NP + jp]);
        uint32_t a[ROWS];
#pragma unroll
        for (int t = 0; t < ROWS; ++t) a[t] = As[t * aw + (kk >> 1)];
#pragma unroll
        for (int t = 0; t < ROWS; ++t) {
            const float2 x = bf16x2_to_float2(a[t]);
            acc[t][0] = fmaf(x.x, b0.x, acc[t][0]);
            acc[t][1] = fmaf(x.x, b0.y, acc[t][1]);
            acc[t][0] = fmaf(x.y, b1.x, acc[t][0]);
            acc[t][1] = fmaf(x.y, b1.y, acc[t][1]);
        }
    }
}

template <bool B_MN>
__global__ void __launch_bounds__(SKINNY_THREADS) skinny_kernel(const SkinnyParams p) {
    extern __shared__ __align__(16) uint8_t skinny_smem[];
    const int tid = threadIdx.x;
    const int sidx = blockIdx.x, tb = blockIdx.y;
    const int t0 = tb * p.tok;
    const int NP = p.r / 2;                     // column pairs
    const int KG = SKINNY_THREADS / NP;         // k groups (r <= 256: at least 2)
    const int aw = p.kc / 2;                    // words per staged A row
    uint32_t *As = reinterpret_cast<uint32_t *>(skinny_smem);     // [16][kc] bf16
    uint32_t *Bs = As + SKINNY_TOK * aw;                          // [kc][r] bf16
    float *red = reinterpret_cast<float *>(Bs + p.kc * NP);       // [KG][16][r] fp32
    __shared__ int is_last;

    // Stage chunk ch's rows of B (the rank factor).  Nothing this library
    // launches writes L or R, so the first chunk's factor rows are staged
    // before waiting on the previous kernel (only its tokens and outputs
    // depend on it): their latency overlaps the previous kernel's tail.
    auto stage_B = [&](int ch) {
        const int k0 = ch * p.kc;
        const int kn = min(p.kc, p.K - k0);  // a multiple of 64 (K is)
        if (B_MN) {
            // rows k0 .. k0 + kn of B stored [K x r], as they are: asynchronous
            // 16-byte copies, all in flight at once
            const int rv = p.r / 8;
            for (int i = tid; i < kn * rv; i += SKINNY_THREADS) {
                const int k = i / rv, c = i % rv;
                const bool ok = in_bounds((int64_t)(k0 + k) * p.r + 8 * c, 8, p.ext_B);
                cp_async16(Bs + k * NP + 4 * c, ok ? p.B + (int64_t)(k0 + k) * p.r + 8 * c : p.B, ok ? 16u : 0u);
            }
        } else {
            // [r x K]: eight consecutive k of row j per load, scattered to Bs[k][j];
            // neighbouring threads take neighbouring j (2-byte shared stores
            // side by side); four loads in flight per thread
            uint16_t *Bh = reinterpret_cast<uint16_t *>(Bs);
            const int kv = kn / 8;
            const int n = p.r * kv;
            for (int i0 = tid; i0 < n; i0 += 4 * SKINNY_THREADS) {
                uint4 v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int i = i0 + u * SKINNY_THREADS;
                    v[u] = make_uint4(0u, 0u, 0u, 0u);
                    if (i < n && in_bounds((int64_t)(i % p.r) * p.K + k0 + 8 * (i / p.r), 8, p.ext_B))
                        v[u] = *reinterpret_cast<const uint4 *>(p.B + (int64_t)(i % p.r) * p.K + k0 + 8 * (i / p.r));
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int i = i0 + u * SKINNY_THREADS;
                    if (i >= n) break;
                    const int j = i % p.r, c = i / p.r;
                    const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        Bh[(8 * c + 2 * e) * p.r + j] = static_cast<uint16_t>(w[e] & 0xFFFFu);
                        Bh[(8 * c + 2 * e + 1) * p.r + j] = static_cast<uint16_t>(w[e] >> 16);
                    }
                }
            }
        }
    };
    if (sidx < p.chunks) stage_B(sidx);

    grid_dep_wait();
    grid_dep_launch();
    {
        const int64_t nb = (int64_t)gridDim.x * gridDim.y;
        const int64_t i0 = ((int64_t)blockIdx.y * gridDim.x + blockIdx.x) * SKINNY_THREADS + tid;
        for (int64_t i = i0; i < p.zero_n0; i += nb * SKINNY_THREADS) p.zero0[i] = 0.0f;
        for (int64_t i = i0; i < p.zero_n1; i += nb * SKINNY_THREADS) p.zero1[i] = 0.0f;
    }

    const int rows = min(p.tok, p.T - t0);  // token rows of this block
    const bool active = tid < KG * NP;
    const int jp = tid % NP, kg = tid / NP;
    float acc[SKINNY_TOK][2];
#pragma unroll
    for (int t = 0; t < SKINNY_TOK; ++t) acc[t][0] = acc[t][1] = 0.0f;

    for (int ch = sidx; ch < p.chunks; ch += p.splits) {
        const int k0 = ch * p.kc;
        const int kn = min(p.kc, p.K - k0);  // a multiple of 64 (K is)
        if (ch != sidx) {
            __syncthreads();  // the previous chunk's reads of As / Bs are done
            stage_B(ch);
        }
        // A rows t0 .. t0 + 15 (zero past T): asynchronous 16-byte copies
        const int av = kn / 8;
        for (int i = tid; i < p.tok * av; i += SKINNY_THREADS) {
            const int t = i / av, c = i % av;
            const bool ok = t0 + t < p.T && in_bounds((int64_t)(t0 + t) * p.K + k0 + 8 * c, 8, p.ext_A);
            cp_async16(As + t * aw + 4 * c, ok ? p.A + (int64_t)(t0 + t) * p.K + k0 + 8 * c : p.A, ok ? 16u : 0u);
        }
        cp_async_wait_all();
        __syncthreads();
        if (active) {
            // token rows rounded up to 1, 2, 4, 8 or 16 (the rows past T are
            // staged as zeros); the same branch for the whole CTA
            if (rows <= 1) skinny_chunk<1>(acc, As, Bs, aw, NP, KG, jp, kg, kn);
            else if (rows <= 2) skinny_chunk<2>(acc, As, Bs, aw, NP, KG, jp, kg, kn);
            else if (rows <= 4) skinny_chunk<4>(acc, As, Bs, aw, NP, KG, jp, kg, kn);
            else if (rows <= 8) skinny_chunk<8>(acc, As, Bs, aw, NP, KG, jp, kg, kn);
            else skinny_chunk<16>(acc, As, Bs, aw, NP, KG, jp, kg, kn);
        }
    }
    // this CTA's partial: the k groups summed in order
    if (active) {
#pragma unroll
        for (int t = 0; t < SKINNY_TOK; ++t) {
            red[(kg * SKINNY_TOK + t) * p.r + 2 * jp] = acc[t][0];
            red[(kg * SKINNY_TOK + t) * p.r + 2 * jp + 1] = acc[t][1];
        }
    }
    __syncthreads();
    const int n_out = SKINNY_TOK * p.r;         // slot size
    const int n_valid = rows * p.r;             // its rows below T
    float *slots = p.ws + (int64_t)tb * p.splits * n_out;
    for (int i = tid; i < n_valid; i += SKINNY_THREADS) {
        float v = red[i];
        for (int g = 1; g < KG; ++g) v += red[g * n_out + i];
        if (in_buf(slots + (int64_t)sidx * n_out + i, p.ws, 1, p.ext_ws)) __stcg(slots + (int64_t)sidx * n_out + i, v);
    }
    __threadfence();
    __syncthreads();
    if (tid == 0 && in_bounds(tb, 1, p.ext_count)) {
        const int prev = atomicAdd(p.count + tb, 1);
        is_last = prev == p.splits - 1;
        if (is_last) p.count[tb] = 0;  // every split has arrived: ready for the next launch
    }
    __syncthreads();
    if (!is_last) return;
    if (!in_buf(slots, p.ws, (int64_t)p.splits * n_out, p.ext_ws)) return;
    __threadfence();
    // The last CTA of this token block sums the slots in split order, four
    // outputs (a float4) at a time, sixteen slots' loads in flight per pass.
    // With fewer float4 outputs than threads, G threads share an output: each
    // sums a contiguous range of slots, and the G range sums are then added
    // in range order (a fixed order either way).
    const int n4 = n_valid / 4;  // r is a multiple of 8
    const int64_t stride = n_out / 4;
    const float4 *base = reinterpret_cast<const float4 *>(slots);
    const int G = n4 >= SKINNY_THREADS ? 1 : min(SKINNY_THREADS / n4, p.splits);
    const int per = (p.splits + G - 1) / G;
    float4 *part = reinterpret_cast<float4 *>(red);  // [G][n4] range sums (G > 1: at most 4 KB)
    for (int i = tid; i < G * n4; i += SKINNY_THREADS) {
        const int g = i / n4, o = i % n4;
        const int s0 = g * per, s1 = min(p.splits, s0 + per);
        const float4 *src = base + o;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        bool first = true;
        for (int sb = s0; sb < s1; sb += 16) {
            float4 x[16];
#pragma unroll
            for (int u = 0; u < 16; ++u)
                if (sb + u < s1) x[u] = __ldcg(src + (sb + u) * stride);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                if (sb + u < s1) {
                    if (first) {
                        v = x[u];
                        first = false;
                    } else {
                        v.x += x[u].x;
                        v.y += x[u].y;
                        v.z += x[u].z;
                        v.w += x[u].w;
                    }
                }
            }
        }
        if (G > 1) part[g * n4 + o] = v;
        else skinny_store4(p, t0, 4 * o, v);
    }
    if (G > 1) {
        __syncthreads();
        if (tid < n4) {
            float4 v = part[tid];
            for (int g = 1; g < G; ++g) {
                if (g * per >= p.splits) break;  // an empty range (none summed)
                const float4 x = part[g * n4 + tid];
                v.x += x.x;
                v.y += x.y;
                v.z += x.z;
                v.w += x.w;
            }
            skinny_store4(p, t0, 4 * tid, v);
        }
    }
}

}  // namespace slope
