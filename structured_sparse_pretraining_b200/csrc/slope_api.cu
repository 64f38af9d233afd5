// slope_api.cu -- the C ABI of libslope.so (declared in include/slope.h):
// argument checks on the host, TMA tensor-map encoding, kernel launches.
// All kernels of the library live in this one translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/slope.h"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "gemm_wide.cuh"
#include "prune.cuh"
#include "skinny.cuh"

namespace {

thread_local char g_err[512] = "";
thread_local int64_t g_launches = 0;

int fail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(SLOPE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define CHECK_PTR(p)                                                              \
    do {                                                                          \
        if ((p) == nullptr) return fail(SLOPE_ERR_ARG, "%s is NULL", #p);         \
        if (!aligned16(p)) return fail(SLOPE_ERR_ALIGN, "%s is not 16-byte aligned", #p); \
    } while (0)

int check_features(int64_t v, const char *name) {
    if (v <= 0) return fail(SLOPE_ERR_ARG, "%s = %lld must be positive", name, (long long)v);
    if (v % 64 != 0) return fail(SLOPE_ERR_SHAPE, "%s = %lld must be a multiple of 64", name, (long long)v);
    if (v > (int64_t(1) << 30)) return fail(SLOPE_ERR_SHAPE, "%s = %lld too large", name, (long long)v);
    return SLOPE_OK;
}

int check_tokens(int64_t T) {
    if (T <= 0) return fail(SLOPE_ERR_ARG, "T = %lld must be positive", (long long)T);
    if (T > (int64_t(1) << 30)) return fail(SLOPE_ERR_SHAPE, "T = %lld too large", (long long)T);
    return SLOPE_OK;
}

int check_rank(int64_t r) {
    if (r < 0) return fail(SLOPE_ERR_ARG, "r = %lld must be >= 0", (long long)r);
    if (r % 8 != 0 || r > 256)
        return fail(SLOPE_ERR_SHAPE, "r = %lld must be 0 or a multiple of 8 up to 256 (zero-pad the adapter)",
                    (long long)r);
    return SLOPE_OK;
}

// ------------------------------------------------------------------ device info
struct DevInfo {
    int sms = 0;
    int major = 0, minor = 0;
};

int device_info(DevInfo &d) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    static thread_local int cached_dev = -1;
    static thread_local DevInfo cached;
    if (dev != cached_dev) {
        cudaDeviceProp prop;
        e = cudaGetDeviceProperties(&prop, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
        cached.sms = prop.multiProcessorCount;
        cached.major = prop.major;
        cached.minor = prop.minor;
        cached_dev = dev;
    }
    d = cached;
    if (d.major != 10 || d.minor != 0)
        return fail(SLOPE_ERR_UNSUPPORTED, "device is sm_%d%d; this library is built for sm_100a", d.major, d.minor);
    return SLOPE_OK;
}

// ------------------------------------------------------------------ tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn lookup_encode_fn() {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        return reinterpret_cast<EncodeTiledFn>(p);
    return nullptr;
}

EncodeTiledFn encode_fn() {
    static const EncodeTiledFn fn = lookup_encode_fn();  // initialised once, thread-safe
    return fn;
}

// 2-D 16-bit tensor [rows x cols] (cols contiguous, row pitch `ld` elements),
// box [box_rows x box_cols], out-of-bounds reads as zero (stores are clipped).
// Operand tiles use the 128-byte swizzle; code tiles and output blocks none.
// 2-D tensor map over a row-major [rows x cols] tensor with leading dimension
// `ld` (elements); `swizzle` is the shared-memory swizzle span in bytes
// (0, 32, 64 or 128), which must cover the box's inner extent.
int make_map(CUtensorMap &m, const void *base, int64_t rows, int64_t cols, int64_t ld, int box_cols, int box_rows,
             int swizzle = 128, bool bf16 = true) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(SLOPE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(&m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 2,
                    const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                    : swizzle == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                    : swizzle == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                    : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(SLOPE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for [%lld x %lld] box [%d x %d]", (int)r,
                    (long long)rows, (long long)cols, box_rows, box_cols);
    return SLOPE_OK;
}

// Blocks of `kern` resident per SM (cached per slot and device; 1 if the
// query fails), for sizing grid-stride launches to one wave.
template <typename Kern>
int resident_blocks(Kern kern, int threads, int smem_bytes, int slot) {
    static std::atomic<int> cache[8][64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && slot < 8) {
        const int c = cache[slot][dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem_bytes) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = 1;
    }
    if (dev < 64 && slot < 8) cache[slot][dev].store(n, std::memory_order_relaxed);
    return n;
}

// ------------------------------------------------------------------ launches
// Every launch may overlap the tail of the previous kernel in the stream
// (programmatic stream serialisation); each kernel waits for its predecessor
// with griddepcontrol.wait before it touches global memory.
template <typename Kern, typename... Args>
int launch_pdl(Kern kern, dim3 grid, dim3 block, int smem_bytes, cudaStream_t st, const char *what, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem_bytes;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
    if (e != cudaSuccess) return cuda_fail(e, what);
    ++g_launches;
    return SLOPE_OK;
}

template <bool A_MN, bool B_MN, int EPI, int BM, int BN>
int launch_gemm(const CUtensorMap &a, const CUtensorMap &b, const slope::GemmParams &p, int sms, cudaStream_t st) {
    using C = slope::GemmCfg<BM, BN>;
    auto kern = slope::gemm_kernel<A_MN, B_MN, EPI, BM, BN>;
    // the shared-memory opt-in is per device: remember it per device ordinal
    static std::atomic<uint64_t> attr_set_mask{0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !(attr_set_mask.load() & (1ull << dev))) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemm)");
        if (dev < 64) attr_set_mask.fetch_or(1ull << dev);
    }
    if (p.num_work <= 0) return SLOPE_OK;
    const int grid = p.num_work < sms ? p.num_work : sms;
    return launch_pdl(kern, dim3(grid), dim3(192), C::SMEM_BYTES, st, "gemm launch", a, b, p);
}

// Cluster launch of a paired (cta_group::2) kernel: clusters of 2 CTAs, as
// many clusters as can be resident at once (one CTA per SM), each looping over
// the work list.  `slot` tells apart the cached per-kernel set-up.
// Cluster launch with clusters of `csize` CTAs (one CTA per SM), as many
// clusters as can be resident at once, each looping over the work list.
template <typename Kern, typename... Args>
int launch_clusters(Kern kern, int slot, int csize, int threads, int smem_bytes, int num_work, int sms,
                    cudaStream_t st, Args... args) {
    static std::atomic<uint64_t> attr_set_mask[48];
    static std::atomic<int> max_clusters[48][64];
    int dev = 0;
    cudaGetDevice(&dev);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;  // the occupancy query takes the cluster shape only
    const bool cached = dev < 64 && (attr_set_mask[slot].load() & (1ull << dev));
    int pairs = cached ? max_clusters[slot][dev].load() : sms / csize;
    if (!cached) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(cluster kernel)");
        int n = 0;
        cfg.gridDim = dim3(csize * (sms / csize), 1, 1);
        e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
        if (e != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = sms / csize;
        }
        pairs = n;
        if (dev < 64) {
            max_clusters[slot][dev].store(n);
            attr_set_mask[slot].fetch_or(1ull << dev);
        }
    }
    if (num_work <= 0) return SLOPE_OK;
    if (pairs > num_work) pairs = num_work;
    if (pairs < 1) pairs = 1;
    cfg.gridDim = dim3(csize * pairs, 1, 1);
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
    if (e != cudaSuccess) return cuda_fail(e, "cluster kernel launch");
    ++g_launches;
    return SLOPE_OK;
}

template <typename Kern, typename... Args>
int launch_pairs(Kern kern, int slot, int threads, int smem_bytes, int num_work, int sms, cudaStream_t st,
                 Args... args) {
    return launch_clusters(kern, slot, 2, threads, smem_bytes, num_work, sms, st, args...);
}

template <bool A2_MN, int BN, bool SPLIT>
int launch_pair(const CUtensorMap &a, const CUtensorMap &b, const CUtensorMap &a2, const CUtensorMap &b2,
                const CUtensorMap &em, const slope::GemmParams &p, int sms, cudaStream_t st) {
    using C = slope::PairCfg<BN>;
    constexpr int bn_index = BN == 224 ? 0 : BN == 192 ? 1 : BN == 240 ? 2 : BN == 176 ? 3 : BN == 128 ? 4
                             : BN == 64 ? 5 : BN == 32 ? 6 : 7;
    const int slot = (A2_MN ? 0 : 1) + 2 * bn_index + 8 + (SPLIT ? 16 : 0);
    return launch_clusters(slope::sp_pair_kernel<A2_MN, BN, SPLIT>, slot, 2, 352, C::SMEM_BYTES, p.num_work, sms, st,
                           a, b, a2, b2, em, p);
}

// Per-device workspaces of the products split over their reduction
// dimension (the masked weight gradient over tokens, the sparse products over
// K at few tokens): fp32 partials and per-(tile, CTA, warp) counters.
//
// Lifetime: a workspace only grows, and a buffer it outgrows is never freed
// (it stays allocated until the process exits), because a CUDA graph captured
// earlier may still hold its address and replay into it.  Growth is allowed
// during stream capture: the allocation is not a stream operation, so the
// thread's capture mode is relaxed around cudaMalloc, and the new buffer is
// zeroed on the library's own non-capturing stream and waited for before the
// call returns, so it is ready both for the graph being captured and for
// eager calls.  Counters start at zero and every launch leaves them at zero.
// One mutex guards these tables and the other lazily filled host caches.
struct SplitWorkspace {
    float *ws = nullptr;
    int *count = nullptr;
    size_t ws_elems = 0, count_elems = 0;
};
SplitWorkspace g_dw_ws[64];  // masked weight gradient
SplitWorkspace g_sp_ws[64];  // sparse products
SplitWorkspace g_tp_ws[64];  // skinny token products (XL, G) at few tokens: CUDA-core partials
SplitWorkspace g_tpacc_ws[64];  // token products split over K on tensor cores: fp32 accumulators
SplitWorkspace g_tok_ws[64];    // fused rank products of the sparse products: per-unit flags (counters)
SplitWorkspace g_dwad_ws[64];   // adapter gradients fused into the masked gradient: split partials, counters
SplitWorkspace g_tokp_ws[64];   // fused rank products split into pieces: fp32 partials, per-(unit, CTA, warp) counters
std::mutex g_mu;                // guards the workspace tables and the per-device caches
cudaStream_t g_side[64] = {};   // per device: a private stream for zeroing new workspaces

// Zero `bytes` at `p` and wait for it, outside any stream capture in progress.
int zero_now(void *p, size_t bytes, int dev) {
    if (!g_side[dev]) {
        cudaError_t e = cudaStreamCreateWithFlags(&g_side[dev], cudaStreamNonBlocking);
        if (e != cudaSuccess) return cuda_fail(e, "cudaStreamCreate(workspace zeroing)");
    }
    cudaError_t e = cudaMemsetAsync(p, 0, bytes, g_side[dev]);
    if (e == cudaSuccess) e = cudaStreamSynchronize(g_side[dev]);
    if (e != cudaSuccess) return cuda_fail(e, "zero a new workspace");
    return SLOPE_OK;
}

// A new zeroed device buffer of `bytes`, callable while another stream of this
// thread is being captured (relaxed capture mode for the duration).
int alloc_zeroed(void **p, size_t bytes, int dev, const char *what) {
    cudaStreamCaptureMode mode = cudaStreamCaptureModeRelaxed;
    cudaThreadExchangeStreamCaptureMode(&mode);
    cudaError_t e = cudaMalloc(p, bytes);
    int rc = SLOPE_OK;
    if (e != cudaSuccess) {
        *p = nullptr;
        rc = fail(SLOPE_ERR_CUDA, "cudaMalloc(%s, %zu bytes): %s", what, bytes, cudaGetErrorString(e));
    } else {
        rc = zero_now(*p, bytes, dev);
    }
    cudaThreadExchangeStreamCaptureMode(&mode);  // restore the caller's mode
    return rc;
}

// Every fp32 area is zeroed when allocated (the tensor-core K split keeps an
// accumulator that must start at zero; every launch leaves it at zero).
int split_workspace(SplitWorkspace *table, size_t ws_elems, size_t count_elems, float *&ws, int *&count) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64) return fail(SLOPE_ERR_UNSUPPORTED, "device ordinal %d >= 64", dev);
    std::lock_guard<std::mutex> lock(g_mu);
    SplitWorkspace &w = table[dev];
    if (w.ws_elems < ws_elems) {
        void *p = nullptr;
        if (int rc = alloc_zeroed(&p, ws_elems * sizeof(float), dev, "split workspace")) return rc;
        w.ws = static_cast<float *>(p);  // the outgrown buffer stays allocated (see above)
        w.ws_elems = ws_elems;
    }
    if (w.count_elems < count_elems) {
        void *p = nullptr;
        if (int rc = alloc_zeroed(&p, count_elems * sizeof(int), dev, "split counters")) return rc;
        w.count = static_cast<int *>(p);
        w.count_elems = count_elems;
    }
    ws = w.ws;
    count = w.count;
    return SLOPE_OK;
}

// After a failed launch a split may not have arrived: clear the counters (and
// the tensor-core split accumulator).  Called after the stream was synchronised.
void reset_split_counters() {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64) return;
    std::lock_guard<std::mutex> lock(g_mu);
    const SplitWorkspace *tabs[7] = {&g_dw_ws[dev], &g_sp_ws[dev], &g_tp_ws[dev], &g_tpacc_ws[dev], &g_tok_ws[dev],
                                     &g_dwad_ws[dev], &g_tokp_ws[dev]};
    for (const SplitWorkspace *w : tabs)
        if (w->count) zero_now(w->count, w->count_elems * sizeof(int), dev);
    if (g_tpacc_ws[dev].ws) zero_now(g_tpacc_ws[dev].ws, g_tpacc_ws[dev].ws_elems * sizeof(float), dev);
}

// Token-tile width BN and K split of the SM-pair sparse product.  Measured
// on B200: a pair tile costs about the same time for every BN in {176 .. 224}
// (the operand ring, not the MMA, sets the pace), so the launch time follows
// the number of waves of pair tiles.  A 240-wide tile leaves TMEM room for
// only 8 code slots (12 otherwise) and costs ~3% more per wave.  Narrower
// tiles, for few tokens (inference), stream less: a k-tile moves 18 KB of
// weights and codes plus BN x 128 B of tokens, so their per-tile cost is
// taken in proportion to those bytes.  With a narrow tile the layer may have
// fewer tiles than SM pairs (weight streaming at a handful of tokens): the
// K range is then split over up to 8 work units per tile, each at least 4
// k-tiles, whose fp32 partials the last arriver sums (a small extra cost per
// split).  Pick the least waves x cost; among equal costs the least total
// tile area (fewer idle token columns in edge tiles).
struct SparseTile {
    int bn, splits;
    bool wide;  // sp_wide_kernel: 512-row pair tiles of two 256-row blocks (bn = 224, no split)
};

// Relative cost of a k-tile of a 512 x 224 pair tile of sp_wide_kernel against
// one of a 256 x 224 pair tile, and its exposed epilogue in k-tile units
// (measured on B200: 1119 against 790 cycles per k-tile with L2-resident
// operands, 1392 against 943 streaming from DRAM; the epilogue of a tile is
// about 4k cycles, half of it hidden by releasing the blocks one at a time).
constexpr double WIDE_KTILE_COST = 1.45;
constexpr double WIDE_EPILOGUE_KTILES = 2.0;

// The best 256-row pair tile (token width and K split) and its cost in units
// of one full-K 256 x 224 pair tile per SM pair.
SparseTile pick_pair_tile(int64_t M, int64_t T, int64_t K, int sms, double &cost_out) {
    const int bns[8] = {240, 224, 192, 176, 128, 64, 32, 16};
    const int64_t kt = (K + 127) / 128;
    double best_cost = 1e300;
    int64_t best_area = INT64_MAX;
    SparseTile best{224, 1, false};
    const int64_t pairs = sms / 2 > 0 ? sms / 2 : 1;
    for (int bn : bns) {
        const int64_t tiles = (M + 255) / 256 * ((T + bn - 1) / bn);
        const double per_tile = bn == 240 ? 1.03 : bn >= 176 ? 1.0 : (18432.0 + 128.0 * bn) / (18432.0 + 128.0 * 176);
        const int max_splits = bn >= 176 ? 1 : 8;
        for (int s = 1; s <= max_splits; ++s) {
            const int64_t kps = (kt + s - 1) / s;
            if (s > 1 && (kps < 4 || (kt + kps - 1) / kps != s)) continue;  // every split non-empty
            const int64_t waves = (tiles * s + pairs - 1) / pairs;
            const double cost = (double)waves * per_tile * (double)kps / (double)kt + 0.02 * (s - 1);
            const int64_t area = tiles * bn;
            if (cost < best_cost - 1e-9 || (cost < best_cost + 1e-9 && area < best_area)) {
                best_cost = cost;
                best_area = area;
                best = SparseTile{bn, s, false};
            }
        }
    }
    cost_out = best_cost;
    return best;
}

// Cost of the two-block 512 x 224 tiles (no K split) in the same units.
double wide_tile_cost(int64_t M, int64_t T, int64_t K, int sms) {
    const int64_t kt = (K + 127) / 128;
    const int64_t pairs = sms / 2 > 0 ? sms / 2 : 1;
    const int64_t tiles = (M + 511) / 512 * ((T + 223) / 224);
    const int64_t waves = (tiles + pairs - 1) / pairs;
    return (double)waves * (WIDE_KTILE_COST + WIDE_EPILOGUE_KTILES / (double)kt);
}

SparseTile pick_sparse_tile(int64_t M, int64_t T, int64_t K, int sms) {
    double pair_cost = 0.0;
    const SparseTile best = pick_pair_tile(M, T, K, sms, pair_cost);
    // the two-block tile: long reductions with codes by TMA (K a multiple of 128)
    if (K % 128 == 0 && (K + 127) / 128 >= 8 && wide_tile_cost(M, T, K, sms) < pair_cost - 1e-9)
        return SparseTile{224, 1, true};
    return best;
}

// A separate rank-product launch (and the second launch's start-up) costs
// about as much as this many k-tiles of one 256 x 224 pair tile (~14 us on
// B200): the planner's costs plus this charge, set against the fused launch,
// picked the faster form (or one within 0.5 us of it) on 161 of 196 measured
// shapes (every layer of the four transformer workloads at 16 to 8192
// tokens, both products), and one within 15% or 5 us on all but four.
constexpr double SEPARATE_LAUNCH_KTILES = 30.0;

// m-tiles per group of the wide kernel's grouped tile order: the pairs active
// at one time then share about sqrt(pairs x t / w) weight tiles and as many
// token tiles (t, w: bytes of a k-slice of a token tile and of a weight
// tile, 224 x 2 against 512 x 1.125), which keeps each slice in L2 while the
// pairs that need it read it.
int wide_raster_group(int64_t m_tiles, int sms) {
    const double pairs = sms / 2 > 0 ? sms / 2 : 1;
    int g = (int)(std::sqrt(pairs * (224.0 * 2.0) / (512.0 * 1.125)) + 0.5);
    if (g < 1) g = 1;
    if (g > m_tiles) g = (int)m_tiles;
    return g;
}

slope::GemmParams base_params(int64_t M, int64_t N, int BM, int BN) {
    slope::GemmParams p{};
    p.M = (int)M;
    p.N = (int)N;
    p.num_m_tiles = (int)((M + BM - 1) / BM);
    p.num_n_tiles = (int)((N + BN - 1) / BN);
    p.num_splits = 1;
    return p;
}

// No split: the whole K per tile.
void set_full_k(slope::GemmParams &p, int k_tiles) {
    p.k_tiles_total = k_tiles;
    p.k_tiles_per_split = k_tiles;
    p.num_splits = 1;
    p.num_work = p.num_m_tiles * p.num_n_tiles;
}

// Split K so that the work list fills at most one wave (one unit per SM);
// every split is non-empty.
void set_splits(slope::GemmParams &p, int k_tiles, int sms) {
    const int tiles = p.num_m_tiles * p.num_n_tiles;
    int splits = sms / tiles;
    if (splits > k_tiles) splits = k_tiles;
    if (splits < 1) splits = 1;
    const int per = (k_tiles + splits - 1) / splits;
    p.k_tiles_total = k_tiles;
    p.k_tiles_per_split = per;
    p.num_splits = (k_tiles + per - 1) / per;
    p.num_work = tiles * p.num_splits;
}

// Width of the adapter-rank dimension of a skinny product's tile.
int rank_tile(int64_t r) { return r <= 16 ? 16 : r <= 32 ? 32 : r <= 64 ? 64 : (r <= 128 ? 128 : 256); }

// Box of an MN-major B operand holding `bn` columns of rank: 64-column
// panels with a 128-byte swizzle, or one 16 / 32-column box with a 32 / 64-byte
// swizzle (the layout the skinny product's descriptors expect).
int make_mn_rank_map(CUtensorMap &m, const uint16_t *base, int64_t rows, int64_t r, int bn) {
    if (bn < 64) return make_map(m, base, rows, r, r, bn, 64, 2 * bn);
    return make_map(m, base, rows, r, r, 64, 64);
}

}  // namespace

namespace {
// Token products with at most this many tokens run on CUDA cores (skinny.cuh);
// measured on B200 (in = 9216 and 36864, r = 96), the tensor-core path with a
// K split is faster from 64 tokens on.
constexpr int64_t SKINNY_MAX_TOKENS = 32;
constexpr int SKINNY_SMEM_MAX = 200 * 1024;  // shared memory of a skinny CTA, at most

// out [T x r] = A [T x K] . B on CUDA cores, B = [K x r] (B_MN) or [r x K].
template <bool B_MN>
static int skinny_product(const uint16_t *A, const uint16_t *B, int64_t T, int64_t K, int64_t r, uint16_t *out,
                          const DevInfo &d, cudaStream_t st, float *zero0, int64_t zero_n0, float *zero1,
                          int64_t zero_n1) {
    slope::SkinnyParams p{};
    p.A = A;
    p.B = B;
    p.T = (int)T;
    p.K = (int)K;
    p.r = (int)r;
    // K chunk: K / 64 rounded up to a multiple of 64, so that one round of
    // at most 64 CTAs per token block covers K (each CTA stages one chunk:
    // a second round costs a whole extra load latency), as long as the
    // chunk fits SKINNY_SMEM_MAX of shared memory (A 16 x kc, B kc x r,
    // 32 KB of k-group partials); the final in-order sum then reads at most
    // 64 slots.
    int kc = (int)(((K + 63) / 64 + 63) / 64) * 64;
    while (kc > 64 && slope::SKINNY_TOK * kc * 2 + kc * (int)r * 2 + 32 * 1024 > SKINNY_SMEM_MAX) kc -= 64;
    if (kc < 64) kc = 64;
    if (kc > K) kc = (int)K;
    p.kc = kc;
    p.chunks = (int)((K + kc - 1) / kc);
    // blocks of 4 tokens up to 32 tokens (more CTAs, and each block's final
    // sum covers fewer outputs: measured 2x faster than blocks of 16 at 16
    // tokens), of 16 beyond
    p.tok = T <= 32 ? 4 : slope::SKINNY_TOK;
    const int tbs = (int)((T + p.tok - 1) / p.tok);
    int splits = p.chunks < 64 ? p.chunks : 64;
    const int cap = 2 * d.sms / tbs;  // at most two CTAs per SM in all
    if (splits > cap) splits = cap > 0 ? cap : 1;
    p.splits = splits;
    p.out = out;
    p.zero0 = zero0;
    p.zero_n0 = zero_n0;
    p.zero1 = zero1;
    p.zero_n1 = zero_n1;
    const size_t n_out = (size_t)slope::SKINNY_TOK * r;
    if (int rc = split_workspace(g_tp_ws, (size_t)tbs * splits * n_out, (size_t)tbs, p.ws, p.count)) return rc;
    p.ext_A = T * K;
    p.ext_B = K * r;
    p.ext_out = T * r;
    p.ext_ws = (int64_t)tbs * splits * n_out;
    p.ext_count = tbs;
    const int smem = slope::SKINNY_TOK * kc * 2 + kc * (int)r * 2 + 32 * 1024;
    auto kern = slope::skinny_kernel<B_MN>;
    static std::atomic<uint64_t> attr_set_mask{0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !(attr_set_mask.load() & (1ull << dev))) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SKINNY_SMEM_MAX);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(skinny)");
        if (dev < 64) attr_set_mask.fetch_or(1ull << dev);
    }
    return launch_pdl(kern, dim3((unsigned)splits, (unsigned)tbs), dim3(slope::SKINNY_THREADS), smem, st,
                      "skinny token product launch", p);
}

// Skinny product over tokens: out[T x r] (bf16) = A[T x K] (K-major) . B,
// B = L [K x r] read MN-major (B_MN) or R [r x K] read K-major.
template <bool B_MN>
static int token_product(const uint16_t *A, const uint16_t *B, int64_t T, int64_t K, int64_t r, uint16_t *out,
                         const DevInfo &d, cudaStream_t st, float *zero0 = nullptr, int64_t zero_n0 = 0,
                         float *zero1 = nullptr, int64_t zero_n1 = 0) {
    if (T <= SKINNY_MAX_TOKENS)
        return skinny_product<B_MN>(A, B, T, K, r, out, d, st, zero0, zero_n0, zero1, zero_n1);
    // 64-token tiles while 128-token tiles would leave SMs idle
    const bool small = (T + 127) / 128 < d.sms;
    const int bm = small ? 64 : 128;
    const int bn = rank_tile(r);
    CUtensorMap ta, tb;
    if (int rc = make_map(ta, A, T, K, K, 64, bm)) return rc;
    if (B_MN) {
        if (int rc = make_mn_rank_map(tb, B, K, r, bn)) return rc;
    } else {
        if (int rc = make_map(tb, B, r, K, K, 64, bn)) return rc;
    }
    slope::GemmParams p = base_params(T, r, bm, bn);
    const int kt = (int)((K + 63) / 64);
    set_full_k(p, kt);
    // Few tokens (inference): a handful of tiles would each stream all of K
    // on one SM.  Split K then, about 8 k-tiles per split and at most 16
    // splits, keeping one unit per SM; the splits add into an fp32
    // accumulator that the last arriver converts.
    const int tiles = p.num_m_tiles * p.num_n_tiles;
    if (tiles * 2 <= d.sms && kt >= 16) {
        int splits = kt / 8;
        if (splits > 16) splits = 16;
        if (splits > d.sms / tiles) splits = d.sms / tiles;
        const int per = (kt + splits - 1) / splits;
        p.k_tiles_per_split = per;
        p.num_splits = (kt + per - 1) / per;
        p.num_work = tiles * p.num_splits;
        if (p.num_splits > 1) {
            // an fp32 accumulator [T x r], zero between launches, and one counter per (tile, quarter)
            if (int rc = split_workspace(g_tpacc_ws, (size_t)T * r, (size_t)tiles * 4, p.ws, p.ws_count)) return rc;
            p.ext.ws = T * r;
            p.ext.ws_count = (int64_t)tiles * 4;
        }
    }
    p.out = out;
    p.ld_out = r;
    p.ext.out = T * r;
    p.zero0 = zero0;
    p.zero_n0 = zero_n0;
    p.zero1 = zero1;
    p.zero_n1 = zero_n1;
#define SLOPE_TOKEN_CASE(BM_, BN_)                                                                          \
    if (bm == BM_ && bn == BN_) return launch_gemm<false, B_MN, slope::EPI_BF16_ROW, BM_, BN_>(ta, tb, p, d.sms, st);
    SLOPE_TOKEN_CASE(64, 16)
    SLOPE_TOKEN_CASE(64, 32)
    SLOPE_TOKEN_CASE(128, 16)
    SLOPE_TOKEN_CASE(128, 32)
    SLOPE_TOKEN_CASE(64, 64)
    SLOPE_TOKEN_CASE(64, 128)
    SLOPE_TOKEN_CASE(64, 256)
    SLOPE_TOKEN_CASE(128, 64)
    SLOPE_TOKEN_CASE(128, 128)
    SLOPE_TOKEN_CASE(128, 256)
#undef SLOPE_TOKEN_CASE
    return fail(SLOPE_ERR_SHAPE, "no tile for r = %lld", (long long)r);
}

// Skinny reduction over tokens: out (fp32, cleared beforehand) += A^T[M x T] . B[T x r],
// A = [T x M] and B = [T x r] both read MN-major; split over T to fill the GPU.
// transposed_out: out is [r x M] (dR) instead of [M x r] (dL).
static int token_reduction(const uint16_t *A, const uint16_t *B, int64_t T, int64_t M, int64_t r, float *out,
                           bool transposed_out, const DevInfo &d, cudaStream_t st) {
    const int bn = rank_tile(r);
    const int bm = (M + 127) / 128 * ((r + bn - 1) / bn) >= d.sms / 2 ? 128 : 64;
    CUtensorMap ta, tb;
    if (int rc = make_map(ta, A, T, M, M, 64, 64)) return rc;
    if (int rc = make_mn_rank_map(tb, B, T, r, bn)) return rc;
    slope::GemmParams p = base_params(M, r, bm, bn);
    set_splits(p, (int)((T + 63) / 64), d.sms);
    p.out = out;
    p.ld_out = transposed_out ? M : r;
    p.ext.out = M * r;
#define SLOPE_RED_CASE(BM_, BN_)                                                                           \
    if (bm == BM_ && bn == BN_)                                                                             \
        return transposed_out                                                                               \
                   ? launch_gemm<true, true, slope::EPI_F32_ADD_T, BM_, BN_>(ta, tb, p, d.sms, st)          \
                   : launch_gemm<true, true, slope::EPI_F32_ADD_ROW, BM_, BN_>(ta, tb, p, d.sms, st);
    SLOPE_RED_CASE(64, 16)
    SLOPE_RED_CASE(64, 32)
    SLOPE_RED_CASE(128, 16)
    SLOPE_RED_CASE(128, 32)
    SLOPE_RED_CASE(64, 64)
    SLOPE_RED_CASE(64, 128)
    SLOPE_RED_CASE(64, 256)
    SLOPE_RED_CASE(128, 64)
    SLOPE_RED_CASE(128, 128)
    SLOPE_RED_CASE(128, 256)
#undef SLOPE_RED_CASE
    return fail(SLOPE_ERR_SHAPE, "no tile for r = %lld", (long long)r);
}

}  // namespace

namespace {
template <int BN>
int sparse_product_bn(const uint16_t *B, const uint16_t *vals, const uint16_t *meta, const uint16_t *B2,
                             const uint16_t *A2, bool a2_is_r, int64_t T, int64_t K, int64_t M, int64_t r,
                             uint16_t *out, int splits, const DevInfo &d, cudaStream_t st) {
    constexpr int BNH = slope::PairCfg<BN>::BNH;  // token rows per CTA
    CUtensorMap ta, tb, ta2, tb2;
    if (int rc = make_map(ta, vals, M, K / 2, K / 2, 64, 128)) return rc;
    if (int rc = make_map(tb, B, T, K, K, 64, BNH)) return rc;
    // Adapter operands.  r <= 32: one tile per output tile in a dedicated
    // buffer, r padded to rp = 16 or 32 columns (zero fill past r), 32- or
    // 64-byte swizzle; larger r: 64-wide k-tiles through the operand ring.
    const int rp = r <= 16 ? 16 : 32;
    const bool adp_buf = r > 0 && r <= 32;
    if (adp_buf) {
        if (a2_is_r) {
            if (int rc = make_map(ta2, A2, r, M, M, 64, rp)) return rc;  // R^T, MN-major: 64 features x rp
        } else {
            if (int rc = make_map(ta2, A2, M, r, r, rp, 128, 2 * rp)) return rc;  // L, K-major: 128 x rp
        }
        if (int rc = make_map(tb2, B2, T, r, r, rp, BNH, 2 * rp)) return rc;
    } else if (r > 0) {
        if (a2_is_r) {
            if (int rc = make_map(ta2, A2, r, M, M, 64, 64)) return rc;
        } else {
            if (int rc = make_map(ta2, A2, M, r, r, 64, 128)) return rc;
        }
        if (int rc = make_map(tb2, B2, T, r, r, 64, BNH)) return rc;
    } else {
        ta2 = ta;
        tb2 = tb;
    }
    // code tiles by TMA need 16-byte-aligned rows of codes: K a multiple of 128
    CUtensorMap te;
    const bool meta_tma = (K % 128) == 0;
    if (meta_tma) {
        if (int rc = make_map(te, meta, M, K / 16, K / 16, 8, 128, 0, false)) return rc;
    } else {
        te = ta;
    }
    slope::GemmParams p{};
    p.M = (int)M;
    p.N = (int)T;
    p.num_m_tiles = (int)((M + 255) / 256);  // SM-pair tiles of 256 rows
    p.num_n_tiles = (int)((T + BN - 1) / BN);
    p.k_tiles_total = (int)((K + 127) / 128);
    p.k_tiles_per_split = (p.k_tiles_total + splits - 1) / splits;
    p.num_splits = (p.k_tiles_total + p.k_tiles_per_split - 1) / p.k_tiles_per_split;  // all non-empty
    p.num_work = p.num_m_tiles * p.num_n_tiles * p.num_splits;
    p.k_logical = (int)K;
    if (p.num_splits > 1) {
        // partials: [tile][CTA][epilogue warp][split][BN tokens][32 features] fp32
        const size_t tiles = (size_t)p.num_m_tiles * p.num_n_tiles;
        if (int rc = split_workspace(g_sp_ws, tiles * 8 * p.num_splits * BN * 32, tiles * 8, p.ws, p.ws_count)) return rc;
        p.ext.ws = (int64_t)tiles * 8 * p.num_splits * BN * 32;
        p.ext.ws_count = (int64_t)tiles * 8;
    }
    p.meta_tma = meta_tma ? 1 : 0;
    p.r = (int)r;
    p.adp_buf = adp_buf ? rp : 0;
    p.adp_k_tiles = adp_buf ? 0 : (int)((r + 63) / 64);
    p.meta_a = meta;
    p.out = out;
    p.ld_out = M;
    p.ext.out = T * M;
    p.ext.meta_a = M * (K / 16);
    if (p.num_splits > 1) {
        // split launches exist for the narrow tiles only (the planner splits no other)
        if constexpr (BN < 176) {
            if (a2_is_r) return launch_pair<true, BN, true>(ta, tb, ta2, tb2, te, p, d.sms, st);
            return launch_pair<false, BN, true>(ta, tb, ta2, tb2, te, p, d.sms, st);
        } else {
            return fail(SLOPE_ERR_SHAPE, "no split launch for %d-wide token tiles", BN);
        }
    }
    if (a2_is_r) return launch_pair<true, BN, false>(ta, tb, ta2, tb2, te, p, d.sms, st);
    return launch_pair<false, BN, false>(ta, tb, ta2, tb2, te, p, d.sms, st);
}

// The same product on 512-row pair tiles (sp_wide_kernel); K % 128 == 0.
// With `factor` non-NULL the adapter's rank product is fused into the launch:
// B2 (XL for the forward, G for the input gradient) is not an input but is
// computed first as B . factor and written to B2, where factor is L [K x r]
// (a2_is_r: the forward) or R [r x K] (the input gradient); r <= 128.
int sparse_product_wide(const uint16_t *B, const uint16_t *vals, const uint16_t *meta, const uint16_t *B2,
                        const uint16_t *A2, bool a2_is_r, int64_t T, int64_t K, int64_t M, int64_t r, uint16_t *out,
                        const DevInfo &d, cudaStream_t st, const uint16_t *factor = nullptr) {
    using C = slope::WideCfg;
    CUtensorMap ta, tb, ta2, tb2, te, tta, ttb;
    if (int rc = make_map(ta, vals, M, K / 2, K / 2, 64, 128)) return rc;
    if (int rc = make_map(tb, B, T, K, K, 64, C::BNH)) return rc;
    if (int rc = make_map(te, meta, M, K / 16, K / 16, 8, 128, 0, false)) return rc;
    if (r > 0) {
        if (a2_is_r) {
            if (int rc = make_map(ta2, A2, r, M, M, 64, 64)) return rc;    // R^T, MN-major: 64 features x 64 rank
        } else {
            if (int rc = make_map(ta2, A2, M, r, r, 64, 128)) return rc;   // L, K-major: 128 rows x 64 rank
        }
        if (int rc = make_map(tb2, B2, T, r, r, 64, C::BNH)) return rc;    // XL or G, K-major
    } else {
        ta2 = ta;
        tb2 = tb;
    }
    slope::GemmParams p{};
    p.M = (int)M;
    p.N = (int)T;
    p.num_m_tiles = (int)((M + C::TILE_M - 1) / C::TILE_M);
    p.num_n_tiles = (int)((T + C::BN - 1) / C::BN);
    p.num_splits = 1;
    p.num_work = p.num_m_tiles * p.num_n_tiles;
    p.k_tiles_total = (int)(K / 128);
    p.k_tiles_per_split = p.k_tiles_total;
    p.k_logical = (int)K;
    p.meta_tma = 1;
    p.r = (int)r;
    p.adp_k_tiles = r > 0 ? (int)((r + 63) / 64) : 0;
    p.meta_a = meta;
    p.out = out;
    p.ld_out = M;
    p.ext.out = T * M;
    p.ext.meta_a = M * (K / 16);
    p.raster_g = wide_raster_group(p.num_m_tiles, d.sms);
    p.tok_split = 1;
    tta = ta;
    ttb = tb;
    if (factor) {
        p.tok_units = (int)((T + 255) / 256);
        p.tok_k_tiles = (int)(K / 64);
        p.tok_r = (int)r;
        p.tok_out = const_cast<uint16_t *>(B2);
        if (int rc = make_map(tta, B, T, K, K, 64, 128)) return rc;  // token rows as the MMA's A (128 per CTA)
        if (a2_is_r) {
            // XL = X . L: L [K x r] read MN-major, c columns per CTA (2c >= r), swizzle of 2c bytes
            const int c = r <= 32 ? 16 : r <= 64 ? 32 : 64;
            p.tok_b_mn = 1;
            p.tok_bc = c;
            p.tok_n = 2 * c;
            if (int rc = make_map(ttb, factor, K, r, r, c, 64, 2 * c)) return rc;
        } else {
            // G = dY . R^T: R [r x K] read K-major, n/2 rows per CTA (rows past r read as zero)
            p.tok_b_mn = 0;
            p.tok_n = (int)((r + 15) / 16 * 16);
            p.tok_bc = p.tok_n / 2;
            if (int rc = make_map(ttb, factor, r, K, K, 64, p.tok_bc)) return rc;
        }
        // k-slices per stage: as many as the stage holds (16 KB of token rows + the factor's slice each)
        p.tok_slice_bytes = (C::A_BYTES + 128 * p.tok_bc + 1023) / 1024 * 1024;
        p.tok_nsl = C::STAGE_BYTES / p.tok_slice_bytes;
        float *unused = nullptr;
        if (int rc = split_workspace(g_tok_ws, 1, (size_t)p.tok_units + 1, unused, p.tok_flags)) return rc;
        p.ext.tok_out = T * r;
        p.ext.tok_flags = p.tok_units + 1;
        // fewer units than SM pairs: split each over up to 4 ranges of the
        // reduction so that the units spread over the pairs (a unit streams
        // as many token bytes as a tile's B operand, so on a launch of about
        // one tile per pair a whole unit would add to the makespan)
        const int pairs = d.sms / 2 > 0 ? d.sms / 2 : 1;
        int split = 1;
        if (p.tok_units < pairs) {
            split = pairs / p.tok_units;
            if (split > 4) split = 4;
            if (split > p.tok_k_tiles) split = p.tok_k_tiles;
            // every piece non-empty: (split - 1) full ranges must leave some k-slices for the last
            while (split > 1 && (split - 1) * ((p.tok_k_tiles + split - 1) / split) >= p.tok_k_tiles) --split;
        }
        p.tok_split = split;
        p.tok_items = p.tok_units * split;
        if (split > 1) {
            if (int rc = split_workspace(g_tokp_ws, (size_t)p.tok_items * 256 * r, (size_t)p.tok_units * 8, p.tok_ws,
                                         p.tok_cnt))
                return rc;
            p.ext.tok_ws = (int64_t)p.tok_items * 256 * r;
            p.ext.tok_cnt = (int64_t)p.tok_units * 8;
        }
        p.num_work += p.tok_items;
    }
    if (a2_is_r)
        return launch_clusters(slope::sp_wide_kernel<true>, 40, 2, 352, C::SMEM_BYTES, p.num_work, d.sms, st, ta, tb, ta2,
                               tb2, te, tta, ttb, p);
    return launch_clusters(slope::sp_wide_kernel<false>, 41, 2, 352, C::SMEM_BYTES, p.num_work, d.sms, st, ta, tb, ta2, tb2,
                           te, tta, ttb, p);
}

// Whether the forward / input gradient of these sizes runs with the rank
// product fused (sp_wide_kernel; r up to 128): when the two-block tiles,
// which the fused kernel uses and which have no split of the sum over K, cost
// no more than the planner's best pair tiles plus the separate rank-product
// launch.  With a few tokens, or few output rows against a long reduction,
// the fused tiles leave SM pairs idle (up to 2.2x slower at 16 tokens on a
// 36864 -> 9216 layer); from about half a wave on, the saved launch wins
// (up to 1.4x faster at 128 to 2048 tokens on a 1024 x 1024 layer).
bool fusable(int64_t M, int64_t T, int64_t K, int64_t r, int sms) {
    if (!(r > 0 && r <= 128 && K % 128 == 0 && K >= 512)) return false;
    double pair_cost = 0.0;
    pick_pair_tile(M, T, K, sms, pair_cost);
    const double kt = (double)((K + 127) / 128);
    return wide_tile_cost(M, T, K, sms) <= pair_cost + SEPARATE_LAUNCH_KTILES / kt;
}

// Sparse product with the fused adapter phase on SM pairs.  A = compressed
// [M x K] (vals [M x K/2], meta), B = dense [T x K]; adapter: A2 = R^T (from
// R [r x M], MN-major) when a2_is_r, else A2 = L [M x r] (K-major); B2 = [T x r].
int sparse_product(const uint16_t *B, const uint16_t *vals, const uint16_t *meta, const uint16_t *B2,
                          const uint16_t *A2, bool a2_is_r, int64_t T, int64_t K, int64_t M, int64_t r,
                          uint16_t *out, cudaStream_t st) {
    DevInfo d;
    if (int rc = device_info(d)) return rc;
    const SparseTile t = pick_sparse_tile(M, T, K, d.sms);
    if (t.wide) return sparse_product_wide(B, vals, meta, B2, A2, a2_is_r, T, K, M, r, out, d, st);
    const int sp = t.splits;
    switch (t.bn) {
        case 240: return sparse_product_bn<240>(B, vals, meta, B2, A2, a2_is_r, T, K, M, r, out, sp, d, st);
        case 224: return sparse_product_bn<224>(B, vals, meta, B2, A2, a2_is_r, T, K, M, r, out, sp, d, st);
        case 192: return sparse_product_bn<192>(B, vals, meta, B2, A2, a2_is_r, T, K, M, r, out, sp, d, st);
        case 176: return sparse_product_bn<176>(B, vals, meta, B2, A2, a2_is_r, T, K, M, r, out, sp, d, st);
        case 128: return sparse_product_bn<128>(B, vals, meta, B2, A2, a2_is_r, T, K, M, r, out, sp, d, st);
        case 64: return sparse_product_bn<64>(B, vals, meta, B2, A2, a2_is_r, T, K, M, r, out, sp, d, st);
        case 32: return sparse_product_bn<32>(B, vals, meta, B2, A2, a2_is_r, T, K, M, r, out, sp, d, st);
        case 16: return sparse_product_bn<16>(B, vals, meta, B2, A2, a2_is_r, T, K, M, r, out, sp, d, st);
        default: break;
    }
    return fail(SLOPE_ERR_SHAPE, "no sparse tile");
}

}  // namespace

// Self-test of the failure path: one thread waits on an mbarrier that no one
// arrives on, with the same bounded try_wait loop the kernels use but a
// limit of `limit_cycles`.  When the limit runs out it records a timeout in
// the device error word and returns: no trap, no fault, the context stays
// usable.
__global__ void timeout_selftest_kernel(long long limit_cycles) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    slope::mbar_init(&bar, 1);
    slope::fence_barrier_init();
    const uint32_t a = slope::smem_addr(&bar);
    const long long t0 = clock64();
    while (!slope::mbar_try_wait(a, 0)) {
        if (clock64() - t0 > limit_cycles) {
            atomicOr(&slope::g_status, slope::ST_TIMEOUT);
            return;
        }
    }
}

// Scratch of slope_bwd_dw_masked_noalloc: the fp32 partials and counters of a
// token-split launch live in this library's own device memory, so that call
// allocates nothing.  The sizes are the limits stated in slope.h.
static __device__ __align__(256) float g_noalloc_ws[SLOPE_NOALLOC_SCRATCH_FLOATS];
static __device__ __align__(256) int g_noalloc_count[SLOPE_NOALLOC_SCRATCH_COUNTERS];

namespace {
// Device addresses of the no-allocation scratch, looked up once per device.
struct NoAllocScratch {
    float *ws = nullptr;
    int *count = nullptr;
};
NoAllocScratch g_noalloc[64];

int noalloc_scratch(float *&ws, int *&count) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64) return fail(SLOPE_ERR_UNSUPPORTED, "device ordinal %d >= 64", dev);
    std::lock_guard<std::mutex> lock(g_mu);
    NoAllocScratch &s = g_noalloc[dev];
    if (!s.ws) {
        void *a = nullptr, *c = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&a, g_noalloc_ws);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-allocation scratch)");
        e = cudaGetSymbolAddress(&c, g_noalloc_count);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-allocation counters)");
        s.ws = static_cast<float *>(a);
        s.count = static_cast<int *>(c);
    }
    ws = s.ws;
    count = s.count;
    return SLOPE_OK;
}
}  // namespace

namespace {
// Tile width and token split of the masked weight gradient, from sweeps and
// traces on B200.  A k-tile (64 tokens) of a pair tile takes about the same
// time, ~0.29 us, at BN = 128 and at BN = 256: the 256-wide MMA runs at the
// tensor pipe's rate (4 x 128 cycles), the 128-wide one at about half.  So
// tiles are 256 wide wherever `in` allows, and the tokens are split to fill
// the SM pairs: the split count minimises waves x k-tiles per split plus the
// fp32 partials' round trip through L2 (splits x out x in/2 floats, written
// and re-read, at ~10 TB/s).
struct DwPlan {
    int bn, splits;
};
DwPlan pick_dw_plan(int64_t out, int64_t in, int64_t T, int sms) {
    const int64_t pairs = sms / 2 > 0 ? sms / 2 : 1;
    const int64_t kt = (T + 63) / 64;
    DwPlan best{in % 256 == 0 ? 256 : 128, 1};
    const int64_t tiles = (out + 255) / 256 * ((in + best.bn - 1) / best.bn);
    double best_us = 1e300;
    for (int sp = 1; sp <= 8; ++sp) {
        if (sp > 1 && kt / sp < 8) break;
        const int64_t waves = (tiles * sp + pairs - 1) / pairs;
        double us = (double)waves * (double)((kt + sp - 1) / sp) * 0.29;
        if (sp > 1) us += (double)sp * (double)out * (double)in * 4.0 / 10.0e6;
        if (us < best_us) {
            best_us = us;
            best.splits = sp;
        }
    }
    return best;
}

// m-tiles per group of the masked gradient's grouped tile order (unsplit
// launches).  Measured with ncu on the 9216 -> 27648 layer over 8192 tokens:
// DRAM reads 16.3 GB with the m-tile fastest over all of out (every wave
// streams the dY columns of 74 different m-tiles again), 8.7 GB with groups of
// 8 and 7.9 GB with groups of 16; the tensor pipe is ~94% busy either way, so
// the time follows the clock under the power cap (3.45 -> 2.95 ms).
int dw_raster_group(int64_t m_tiles) { return (int)(m_tiles < 16 ? m_tiles : 16); }

// The masked gradient with the adapter gradients fused (dR^T and dL units
// after the dW tiles, all split over tokens the same way): the split count
// that minimises the launch's makespan under its static round-robin order
// (an adapter unit counted as 0.6 of a dW tile: its MMAs are narrow and its
// B operand small) plus the partials' round trip through L2.
DwPlan pick_dw_plan_fused(int64_t out, int64_t in, int64_t T, int64_t r, int sms) {
    const int64_t pairs = sms / 2 > 0 ? sms / 2 : 1;
    const int64_t kt = (T + 63) / 64;
    DwPlan best{in % 256 == 0 ? 256 : 128, 1};
    const int64_t tiles = (out + 255) / 256 * ((in + best.bn - 1) / best.bn);
    const int64_t extra = (out + 255) / 256 + (in + 255) / 256;
    double best_us = 1e300;
    for (int sp = 1; sp <= 8; ++sp) {
        if (sp > 1 && kt / sp < 8) break;
        const int64_t n = (tiles + extra) * sp;
        if (n > (int64_t)1 << 20) break;
        // round-robin makespan in dW-tile units: unit w goes to pair w % pairs
        double worst = 0.0;
        const int64_t np = pairs < n ? pairs : n;
        for (int64_t pr = 0; pr < np; ++pr) {
            double c = 0.0;
            for (int64_t w = pr; w < n; w += pairs) c += w < tiles * sp ? 1.0 : 0.6;
            if (c > worst) worst = c;
        }
        double us = worst * (double)((kt + sp - 1) / sp) * 0.29;
        if (sp > 1) us += (double)sp * ((double)out * (double)in * 4.0 + (double)(out + in) * r * 8.0) / 10.0e6;
        if (us < best_us) {
            best_us = us;
            best.splits = sp;
        }
    }
    return best;
}

// The second pruning, optionally with the AdamW step on the kept values
// fused into its expand phase (ADAM), or with the row pruning of dense W
// fused ahead of it (DENSE: W^R is written out and pruned again in one pass).
template <bool ADAM, bool DENSE = false>
static int double_prune_launch(const uint16_t *vals, const uint16_t *meta, int64_t out, int64_t in,
                               uint16_t *vals_t, uint16_t *meta_t, const slope::DpAdam &ad, cudaStream_t st,
                               const slope::DpRowPrune &rp = slope::DpRowPrune{}) {
    DevInfo d;
    if (int rc = device_info(d)) return rc;
    // 128-row tiles when out allows (twice the bytes per pass), else 64-row tiles
    const int rows_t = out % 128 == 0 ? 128 : 64;
    const int64_t tiles = (out / rows_t) * (in / slope::DP_TILE);
    const int slot = 1 + (ADAM ? 2 : 0) + (DENSE ? 4 : 0) + (rows_t == 128 ? 0 : 1);  // 0 is prune24's
    const int64_t cap =
        (int64_t)d.sms * (rows_t == 128 ? resident_blocks(slope::double_prune_kernel<128, ADAM, DENSE>, 256, 0, slot)
                                        : resident_blocks(slope::double_prune_kernel<64, ADAM, DENSE>, 256, 0, slot));
    const int64_t blocks = tiles < cap ? tiles : cap;
    if (rows_t == 128)
        return launch_pdl(slope::double_prune_kernel<128, ADAM, DENSE>, dim3((unsigned)blocks), dim3(256), 0, st,
                          "double_prune launch", vals, meta, (int)out, (int)in, vals_t, meta_t, ad, rp);
    return launch_pdl(slope::double_prune_kernel<64, ADAM, DENSE>, dim3((unsigned)blocks), dim3(256), 0, st,
                      "double_prune launch", vals, meta, (int)out, (int)in, vals_t, meta_t, ad, rp);
}

}  // namespace

extern "C" {

const char *slope_last_error(void) { return g_err; }

int slope_sparse_plan(int64_t M, int64_t T, int64_t K, int sms, int *bn, int *splits) {
    if (!bn || !splits) return fail(SLOPE_ERR_ARG, "slope_sparse_plan: NULL output");
    if (M <= 0 || T <= 0 || K <= 0 || sms <= 0) return fail(SLOPE_ERR_ARG, "slope_sparse_plan: non-positive size");
    const SparseTile t = pick_sparse_tile(M, T, K, sms);
    const int64_t kt = (K + 127) / 128;
    const int64_t kps = (kt + t.splits - 1) / t.splits;
    *bn = t.bn;
    *splits = (int)((kt + kps - 1) / kps);
    return SLOPE_OK;
}

int slope_fused_launches(int64_t M, int64_t T, int64_t K, int64_t r, int sms, int *launches) {
    if (!launches) return fail(SLOPE_ERR_ARG, "slope_fused_launches: NULL output");
    if (M <= 0 || T <= 0 || K <= 0 || r < 0 || sms <= 0) return fail(SLOPE_ERR_ARG, "slope_fused_launches: bad size");
    *launches = r == 0 ? 1 : fusable(M, T, K, r, sms) ? 1 : 2;
    return SLOPE_OK;
}

int slope_sparse_tile_rows(int64_t M, int64_t T, int64_t K, int sms, int *rows) {
    if (!rows) return fail(SLOPE_ERR_ARG, "slope_sparse_tile_rows: NULL output");
    if (M <= 0 || T <= 0 || K <= 0 || sms <= 0) return fail(SLOPE_ERR_ARG, "slope_sparse_tile_rows: non-positive size");
    *rows = pick_sparse_tile(M, T, K, sms).wide ? 512 : 256;
    return SLOPE_OK;
}

int64_t slope_launch_count(int reset) {
    int64_t v = g_launches;
    if (reset) g_launches = 0;
    return v;
}

int slope_device_check(void) {
    DevInfo d;
    return device_info(d);
}

int slope_selftest_wait_timeout(void *stream) {
    DevInfo d;
    if (int rc = device_info(d)) return rc;
    // ~10 ms at the B200's clocks
    timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(20000000LL);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "timeout self-test launch");
    ++g_launches;
    return SLOPE_OK;
}

int slope_debug_bounds(void) {
#ifdef SLOPE_DEBUG_BOUNDS
    return 1;
#else
    return 0;
#endif
}

int slope_status_sync(void *stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int word = 0;
    e = cudaMemcpyFromSymbol(&word, slope::g_status, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "read device error word");
    if (word != 0) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(slope::g_status, &zero, sizeof(int));
        if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
    }
    if (word & slope::ST_TIMEOUT) {
        reset_split_counters();  // a split launch may have stopped half-way
        return fail(SLOPE_ERR_TIMEOUT, "a kernel's bounded wait timed out");
    }
    if (word & slope::ST_BOUNDS) {
        reset_split_counters();  // a skipped access may have left a split half-way
        return fail(SLOPE_ERR_BOUNDS, "a kernel's global-memory index fell outside its buffer (access skipped)");
    }
    if (word & slope::ST_NONFINITE) return fail(SLOPE_ERR_NONFINITE, "prune24 input holds NaN or Inf");
    g_err[0] = 0;
    return SLOPE_OK;
}

int slope_prune24(const uint16_t *W, int64_t rows, int64_t K, uint16_t *vals, uint16_t *meta, void *stream) {
    CHECK_PTR(W);
    CHECK_PTR(vals);
    CHECK_PTR(meta);
    if (rows <= 0) return fail(SLOPE_ERR_ARG, "rows = %lld must be positive", (long long)rows);
    if (int rc = check_features(K, "K")) return rc;
    DevInfo d;
    if (int rc = device_info(d)) return rc;
    const int64_t chunks = rows * (K / 16);
    int64_t blocks = (chunks + 256 * slope::PR_UNROLL - 1) / (256 * slope::PR_UNROLL);
    // grid-stride kernel: no more blocks than can be resident at once
    const int64_t cap = (int64_t)d.sms * resident_blocks(slope::prune24_kernel, 256, 0, 0);
    if (blocks > cap) blocks = cap;
    return launch_pdl(slope::prune24_kernel, dim3((unsigned)blocks), dim3(256), 0, static_cast<cudaStream_t>(stream),
                      "prune24 launch", W, vals, meta, chunks);
}

int slope_prune_nm(const uint16_t *W, int64_t rows, int64_t K, int N, int M, uint16_t *vals, uint8_t *pos,
                   void *stream) {
    CHECK_PTR(W);
    CHECK_PTR(vals);
    CHECK_PTR(pos);
    if (rows <= 0 || K <= 0) return fail(SLOPE_ERR_ARG, "rows and K must be positive");
    if (M != 4 && M != 8 && M != 16) return fail(SLOPE_ERR_SHAPE, "M = %d must be 4, 8 or 16", M);
    if (N < 1 || N >= M) return fail(SLOPE_ERR_SHAPE, "need 1 <= N < M, got N = %d, M = %d", N, M);
    if (K % M != 0) return fail(SLOPE_ERR_SHAPE, "K = %lld must be a multiple of M = %d", (long long)K, M);
    DevInfo d;
    if (int rc = device_info(d)) return rc;
    const int64_t groups = rows * (K / M);
    int64_t blocks = (groups + slope::NM_GROUPS - 1) / slope::NM_GROUPS;
    const int64_t cap = (int64_t)d.sms * 8;  // grid-stride beyond eight blocks per SM
    if (blocks > cap) blocks = cap;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (M == 4)
        return launch_pdl(slope::prune_nm_kernel<4>, dim3((unsigned)blocks), dim3(slope::NM_GROUPS), 0, st, "prune_nm launch", W,
                          vals, pos, groups, N);
    if (M == 8)
        return launch_pdl(slope::prune_nm_kernel<8>, dim3((unsigned)blocks), dim3(slope::NM_GROUPS), 0, st, "prune_nm launch", W,
                          vals, pos, groups, N);
    return launch_pdl(slope::prune_nm_kernel<16>, dim3((unsigned)blocks), dim3(slope::NM_GROUPS), 0, st, "prune_nm launch", W,
                      vals, pos, groups, N);
}

int slope_double_prune(const uint16_t *vals, const uint16_t *meta, int64_t out, int64_t in, uint16_t *vals_t,
                       uint16_t *meta_t, void *stream) {
    CHECK_PTR(vals);
    CHECK_PTR(meta);
    CHECK_PTR(vals_t);
    CHECK_PTR(meta_t);
    if (int rc = check_features(out, "out")) return rc;
    if (int rc = check_features(in, "in")) return rc;
    return double_prune_launch<false>(vals, meta, out, in, vals_t, meta_t, slope::DpAdam{},
                                      static_cast<cudaStream_t>(stream));
}

int slope_prune24_double(const uint16_t *W, int64_t out, int64_t in, uint16_t *vals, uint16_t *meta,
                         uint16_t *vals_t, uint16_t *meta_t, void *stream) {
    CHECK_PTR(W);
    CHECK_PTR(vals);
    CHECK_PTR(meta);
    CHECK_PTR(vals_t);
    CHECK_PTR(meta_t);
    if (int rc = check_features(out, "out")) return rc;
    if (int rc = check_features(in, "in")) return rc;
    slope::DpRowPrune rp{W, vals, meta};
    return double_prune_launch<false, true>(nullptr, nullptr, out, in, vals_t, meta_t, slope::DpAdam{},
                                            static_cast<cudaStream_t>(stream), rp);
}

int slope_adamw_double_prune(uint16_t *vals, const uint16_t *meta, const uint16_t *dW_vals, float *m, float *v,
                             int64_t out, int64_t in, float lr, float beta1, float beta2, float eps,
                             float weight_decay, int64_t step, uint16_t *vals_t, uint16_t *meta_t, void *stream) {
    CHECK_PTR(vals);
    CHECK_PTR(meta);
    CHECK_PTR(dW_vals);
    CHECK_PTR(m);
    CHECK_PTR(v);
    CHECK_PTR(vals_t);
    CHECK_PTR(meta_t);
    if (int rc = check_features(out, "out")) return rc;
    if (int rc = check_features(in, "in")) return rc;
    if (step < 1) return fail(SLOPE_ERR_ARG, "adamw step must be >= 1, got %lld", (long long)step);
    if (!(beta1 >= 0.0f && beta1 < 1.0f) || !(beta2 >= 0.0f && beta2 < 1.0f) || !(eps > 0.0f) || !(lr >= 0.0f))
        return fail(SLOPE_ERR_ARG, "adamw: need 0 <= beta1, beta2 < 1, eps > 0, lr >= 0");
    slope::DpAdam ad{};
    ad.vals = vals;
    ad.grad = dW_vals;
    ad.m = m;
    ad.v = v;
    ad.lr = lr;
    ad.b1 = beta1;
    ad.b2 = beta2;
    ad.eps = eps;
    ad.wd = weight_decay;
    // bias corrections in binary64, rounded once to binary32
    ad.step_size = (float)((double)lr / (1.0 - std::pow((double)beta1, (double)step)));
    ad.inv_sqrt_bc2 = (float)(1.0 / std::sqrt(1.0 - std::pow((double)beta2, (double)step)));
    ad.n_vals = out * (in / 2);
    return double_prune_launch<true>(vals, meta, out, in, vals_t, meta_t, ad, static_cast<cudaStream_t>(stream));
}

// Sparse product with the fused adapter phase.  A = compressed [M x K]
// (vals [M x K/2], meta), B = dense [T x K]; adapter: A2 = R^T (from R
// [r x M], MN-major) when a2_is_r, else A2 = L [M x r] (K-major); B2 = [T x r].
int slope_fwd(const uint16_t *X, const uint16_t *vals, const uint16_t *meta, const uint16_t *XL, const uint16_t *R,
              int64_t T, int64_t in, int64_t out, int64_t r, uint16_t *Y, void *stream) {
    CHECK_PTR(X);
    CHECK_PTR(vals);
    CHECK_PTR(meta);
    CHECK_PTR(Y);
    if (int rc = check_tokens(T)) return rc;
    if (int rc = check_features(in, "in")) return rc;
    if (int rc = check_features(out, "out")) return rc;
    if (int rc = check_rank(r)) return rc;
    if (r > 0) {
        CHECK_PTR(XL);
        CHECK_PTR(R);
    }
    return sparse_product(X, vals, meta, XL, R, true, T, in, out, r, Y, static_cast<cudaStream_t>(stream));
}

int slope_bwd_dx(const uint16_t *dY, const uint16_t *vals_t, const uint16_t *meta_t, const uint16_t *G,
                 const uint16_t *L, int64_t T, int64_t in, int64_t out, int64_t r, uint16_t *dX, void *stream) {
    CHECK_PTR(dY);
    CHECK_PTR(vals_t);
    CHECK_PTR(meta_t);
    CHECK_PTR(dX);
    if (int rc = check_tokens(T)) return rc;
    if (int rc = check_features(in, "in")) return rc;
    if (int rc = check_features(out, "out")) return rc;
    if (int rc = check_rank(r)) return rc;
    if (r > 0) {
        CHECK_PTR(G);
        CHECK_PTR(L);
    }
    return sparse_product(dY, vals_t, meta_t, G, L, false, T, out, in, r, dX, static_cast<cudaStream_t>(stream));
}

int slope_fwd_fused(const uint16_t *X, const uint16_t *vals, const uint16_t *meta, const uint16_t *L, const uint16_t *R,
                    int64_t T, int64_t in, int64_t out, int64_t r, uint16_t *XL, uint16_t *Y, void *stream) {
    CHECK_PTR(X);
    CHECK_PTR(vals);
    CHECK_PTR(meta);
    CHECK_PTR(Y);
    if (int rc = check_tokens(T)) return rc;
    if (int rc = check_features(in, "in")) return rc;
    if (int rc = check_features(out, "out")) return rc;
    if (int rc = check_rank(r)) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (r == 0) return sparse_product(X, vals, meta, nullptr, nullptr, true, T, in, out, 0, Y, st);
    CHECK_PTR(L);
    CHECK_PTR(R);
    CHECK_PTR(XL);
    DevInfo d;
    if (int rc = device_info(d)) return rc;
    if (fusable(out, T, in, r, d.sms)) return sparse_product_wide(X, vals, meta, XL, R, true, T, in, out, r, Y, d, st, L);
    // not fusable (few-token tiles, rank above 128): the two launches
    if (int rc = token_product<true>(X, L, T, in, r, XL, d, st)) return rc;
    return sparse_product(X, vals, meta, XL, R, true, T, in, out, r, Y, st);
}

int slope_bwd_dx_fused(const uint16_t *dY, const uint16_t *vals_t, const uint16_t *meta_t, const uint16_t *R,
                       const uint16_t *L, int64_t T, int64_t in, int64_t out, int64_t r, uint16_t *G, uint16_t *dX,
                       void *stream) {
    CHECK_PTR(dY);
    CHECK_PTR(vals_t);
    CHECK_PTR(meta_t);
    CHECK_PTR(dX);
    if (int rc = check_tokens(T)) return rc;
    if (int rc = check_features(in, "in")) return rc;
    if (int rc = check_features(out, "out")) return rc;
    if (int rc = check_rank(r)) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (r == 0) return sparse_product(dY, vals_t, meta_t, nullptr, nullptr, false, T, out, in, 0, dX, st);
    CHECK_PTR(R);
    CHECK_PTR(L);
    CHECK_PTR(G);
    DevInfo d;
    if (int rc = device_info(d)) return rc;
    if (fusable(in, T, out, r, d.sms)) return sparse_product_wide(dY, vals_t, meta_t, G, L, false, T, out, in, r, dX, d, st, R);
    if (int rc = token_product<false>(dY, R, T, out, r, G, d, st)) return rc;
    return sparse_product(dY, vals_t, meta_t, G, L, false, T, out, in, r, dX, st);
}

int slope_bwd_dw_masked(const uint16_t *dY, const uint16_t *X, const uint16_t *meta, int64_t T, int64_t in,
                        int64_t out, uint16_t *dW_vals, void *stream) {
    CHECK_PTR(dY);
    CHECK_PTR(X);
    CHECK_PTR(meta);
    CHECK_PTR(dW_vals);
    if (int rc = check_tokens(T)) return rc;
    if (int rc = check_features(in, "in")) return rc;
    if (int rc = check_features(out, "out")) return rc;
    DevInfo d;
    if (int rc = device_info(d)) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    CUtensorMap ta, tb;
    if (int rc = make_map(ta, dY, T, out, out, 64, 64)) return rc;  // A = dY^T, MN-major
    if (int rc = make_map(tb, X, T, in, in, 64, 64)) return rc;     // B = X, MN-major
    const DwPlan plan = pick_dw_plan(out, in, T, d.sms);
    const int BN = plan.bn;
    slope::GemmParams p{};
    p.M = (int)out;
    p.N = (int)in;
    p.num_m_tiles = (int)((out + 255) / 256);
    p.num_n_tiles = (int)((in + BN - 1) / BN);
    p.num_splits = plan.splits;
    p.num_work = p.num_m_tiles * p.num_n_tiles * plan.splits;
    p.k_tiles_total = (int)((T + 63) / 64);
    p.k_tiles_per_split = (p.k_tiles_total + plan.splits - 1) / plan.splits;
    p.meta_mask = meta;
    p.out = dW_vals;
    p.ld_out = in / 2;
    p.raster_g = dw_raster_group(p.num_m_tiles);
    p.ext.out = out * (in / 2);
    p.ext.meta_mask = out * (in / 16);
    if (plan.splits > 1) {
        const int64_t tiles = (int64_t)p.num_m_tiles * p.num_n_tiles;
        if (int rc = split_workspace(g_dw_ws, (size_t)plan.splits * out * (in / 2), (size_t)tiles * 8, p.ws, p.ws_count)) return rc;
        p.ext.ws = (int64_t)plan.splits * out * (in / 2);
        p.ext.ws_count = tiles * 8;
    }
    const bool wide = BN == 256;
    if (wide)
        return launch_pairs(slope::dw_pair_kernel<256>, 2, 192, slope::DwPairCfg<256>::SMEM_BYTES, p.num_work, d.sms,
                            st, ta, tb, ta, tb, p);
    return launch_pairs(slope::dw_pair_kernel<128>, 3, 192, slope::DwPairCfg<128>::SMEM_BYTES, p.num_work, d.sms, st,
                        ta, tb, ta, tb, p);
}

int slope_bwd_dw_fused(const uint16_t *dY, const uint16_t *X, const uint16_t *meta, const uint16_t *XL,
                       const uint16_t *G, int64_t T, int64_t in, int64_t out, int64_t r, uint16_t *dW_vals, float *dL,
                       float *dR, void *stream) {
    CHECK_PTR(dY);
    CHECK_PTR(X);
    CHECK_PTR(meta);
    CHECK_PTR(dW_vals);
    if (int rc = check_tokens(T)) return rc;
    if (int rc = check_features(in, "in")) return rc;
    if (int rc = check_features(out, "out")) return rc;
    if (int rc = check_rank(r)) return rc;
    if (r == 0) return slope_bwd_dw_masked(dY, X, meta, T, in, out, dW_vals, stream);
    CHECK_PTR(XL);
    CHECK_PTR(G);
    CHECK_PTR(dL);
    CHECK_PTR(dR);
    DevInfo d;
    if (int rc = device_info(d)) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (r > 128) {  // ranks above 128: the masked gradient, then the two tensor-core reductions
        if (int rc = slope_bwd_dw_masked(dY, X, meta, T, in, out, dW_vals, stream)) return rc;
        if (cudaError_t e = cudaMemsetAsync(dR, 0, (size_t)r * out * sizeof(float), st)) return cuda_fail(e, "clear dR");
        if (cudaError_t e = cudaMemsetAsync(dL, 0, (size_t)in * r * sizeof(float), st)) return cuda_fail(e, "clear dL");
        if (int rc = token_reduction(dY, XL, T, out, r, dR, true, d, st)) return rc;
        return token_reduction(X, G, T, in, r, dL, false, d, st);
    }
    CUtensorMap ta, tb, txl, tg;
    if (int rc = make_map(ta, dY, T, out, out, 64, 64)) return rc;  // A = dY^T, MN-major
    if (int rc = make_map(tb, X, T, in, in, 64, 64)) return rc;     // B = X, MN-major (the A of the dL units)
    // XL and G as MN-major B operands: c rank columns per CTA (2c >= r), swizzle of 2c bytes
    const int c = r <= 32 ? 16 : r <= 64 ? 32 : 64;
    if (int rc = make_map(txl, XL, T, r, r, c, 64, 2 * c)) return rc;
    if (int rc = make_map(tg, G, T, r, r, c, 64, 2 * c)) return rc;
    const DwPlan plan = pick_dw_plan_fused(out, in, T, r, d.sms);
    const int BN = plan.bn;
    slope::GemmParams p{};
    p.M = (int)out;
    p.N = (int)in;
    p.num_m_tiles = (int)((out + 255) / 256);
    p.num_n_tiles = (int)((in + BN - 1) / BN);
    p.num_splits = plan.splits;
    p.k_tiles_total = (int)((T + 63) / 64);
    p.k_tiles_per_split = (p.k_tiles_total + plan.splits - 1) / plan.splits;
    p.meta_mask = meta;
    p.out = dW_vals;
    p.ld_out = in / 2;
    p.raster_g = dw_raster_group(p.num_m_tiles);
    p.ext.out = out * (in / 2);
    p.ext.meta_mask = out * (in / 16);
    p.ad_units_r = p.num_m_tiles * plan.splits;
    p.ad_units_l = (int)((in + 255) / 256) * plan.splits;
    p.ad_c = c;
    p.ad_n = 2 * c;
    p.ad_r = (int)r;
    p.ad_in = (int)in;
    p.dR = dR;
    p.dL = dL;
    p.ext.dR = r * out;
    p.ext.dL = in * r;
    p.num_work = p.num_m_tiles * p.num_n_tiles * plan.splits + p.ad_units_r + p.ad_units_l;
    if (plan.splits > 1) {
        const int64_t tiles = (int64_t)p.num_m_tiles * p.num_n_tiles;
        if (int rc = split_workspace(g_dw_ws, (size_t)plan.splits * out * (in / 2), (size_t)tiles * 8, p.ws, p.ws_count))
            return rc;
        const int64_t blocks = p.num_m_tiles + (in + 255) / 256;
        if (int rc = split_workspace(g_dwad_ws, (size_t)plan.splits * (out + in) * r, (size_t)blocks * 8, p.ws2,
                                     p.ws2_count))
            return rc;
        p.ext.ws = (int64_t)plan.splits * out * (in / 2);
        p.ext.ws_count = tiles * 8;
        p.ext.ws2 = (int64_t)plan.splits * (out + in) * r;
        p.ext.ws2_count = blocks * 8;
    }
    if (BN == 256)
        return launch_pairs(slope::dw_pair_kernel<256>, 2, 192, slope::DwPairCfg<256>::SMEM_BYTES, p.num_work, d.sms,
                            st, ta, tb, txl, tg, p);
    return launch_pairs(slope::dw_pair_kernel<128>, 3, 192, slope::DwPairCfg<128>::SMEM_BYTES, p.num_work, d.sms, st,
                        ta, tb, txl, tg, p);
}

int slope_bwd_dw_masked_noalloc(const uint16_t *dY, const uint16_t *X, const uint16_t *meta, int64_t T, int64_t in,
                                int64_t out, uint16_t *dW_vals, void *stream) {
    CHECK_PTR(dY);
    CHECK_PTR(X);
    CHECK_PTR(meta);
    CHECK_PTR(dW_vals);
    if (int rc = check_tokens(T)) return rc;
    if (int rc = check_features(in, "in")) return rc;
    if (int rc = check_features(out, "out")) return rc;
    DevInfo d;
    if (int rc = device_info(d)) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    CUtensorMap ta, tb;
    if (int rc = make_map(ta, dY, T, out, out, 64, 64)) return rc;  // A = dY^T, MN-major
    if (int rc = make_map(tb, X, T, in, in, 64, 64)) return rc;     // B = X, MN-major
    const DwPlan plan = pick_dw_plan(out, in, T, d.sms);
    const int BN = plan.bn;
    slope::GemmParams p{};
    p.M = (int)out;
    p.N = (int)in;
    p.num_m_tiles = (int)((out + 255) / 256);
    p.num_n_tiles = (int)((in + BN - 1) / BN);
    p.num_splits = plan.splits;
    p.num_work = p.num_m_tiles * p.num_n_tiles * plan.splits;
    p.k_tiles_total = (int)((T + 63) / 64);
    p.k_tiles_per_split = (p.k_tiles_total + plan.splits - 1) / plan.splits;
    p.meta_mask = meta;
    p.out = dW_vals;
    p.ld_out = in / 2;
    p.raster_g = dw_raster_group(p.num_m_tiles);
    p.ext.out = out * (in / 2);
    p.ext.meta_mask = out * (in / 16);
    if (plan.splits > 1) {
        const int64_t tiles = (int64_t)p.num_m_tiles * p.num_n_tiles;
        const int64_t floats = (int64_t)plan.splits * out * (in / 2);
        if (floats > SLOPE_NOALLOC_SCRATCH_FLOATS || tiles * 8 > SLOPE_NOALLOC_SCRATCH_COUNTERS)
            return fail(SLOPE_ERR_SHAPE,
                        "masked dW of [%lld x %lld] over %lld tokens is split %d ways and needs %lld floats of "
                        "scratch; the no-allocation entry point holds %lld (use slope_bwd_dw_masked)",
                        (long long)out, (long long)in, (long long)T, plan.splits, (long long)floats,
                        (long long)SLOPE_NOALLOC_SCRATCH_FLOATS);
        if (int rc = noalloc_scratch(p.ws, p.ws_count)) return rc;
        p.ext.ws = floats;
        p.ext.ws_count = tiles * 8;
        // the counters this launch uses start at zero
        cudaError_t e = cudaMemsetAsync(p.ws_count, 0, (size_t)tiles * 8 * sizeof(int), st);
        if (e != cudaSuccess) return cuda_fail(e, "clear the no-allocation counters");
    }
    if (BN == 256)
        return launch_pairs(slope::dw_pair_kernel<256>, 2, 192, slope::DwPairCfg<256>::SMEM_BYTES, p.num_work, d.sms,
                            st, ta, tb, ta, tb, p);
    return launch_pairs(slope::dw_pair_kernel<128>, 3, 192, slope::DwPairCfg<128>::SMEM_BYTES, p.num_work, d.sms, st,
                        ta, tb, ta, tb, p);
}

int slope_adapter_fwd(const uint16_t *X, const uint16_t *L, int64_t T, int64_t in, int64_t r, uint16_t *XL,
                      void *stream) {
    CHECK_PTR(X);
    CHECK_PTR(L);
    CHECK_PTR(XL);
    if (int rc = check_tokens(T)) return rc;
    if (int rc = check_features(in, "in")) return rc;
    if (int rc = check_rank(r)) return rc;
    if (r == 0) return fail(SLOPE_ERR_ARG, "adapter_fwd needs r > 0");
    DevInfo d;
    if (int rc = device_info(d)) return rc;
    // XL = X . L: A = X [T x in] K-major, B = L [in x r] MN-major
    return token_product<true>(X, L, T, in, r, XL, d, static_cast<cudaStream_t>(stream));
}

int slope_adapter_bwd(const uint16_t *X, const uint16_t *dY, const uint16_t *XL, const uint16_t *R, int64_t T,
                      int64_t in, int64_t out, int64_t r, float *dL, float *dR, uint16_t *G, void *stream) {
    CHECK_PTR(X);
    CHECK_PTR(dY);
    CHECK_PTR(XL);
    CHECK_PTR(R);
    CHECK_PTR(dL);
    CHECK_PTR(dR);
    CHECK_PTR(G);
    if (int rc = check_tokens(T)) return rc;
    if (int rc = check_features(in, "in")) return rc;
    if (int rc = check_features(out, "out")) return rc;
    if (int rc = check_rank(r)) return rc;
    if (r == 0) return fail(SLOPE_ERR_ARG, "adapter_bwd needs r > 0");
    DevInfo d;
    if (int rc = device_info(d)) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // G = dY . R^T: A = dY [T x out] K-major, B = R [r x out] K-major.  The
    // same launch clears dR and dL, which the two reductions below add into.
    if (int rc = token_product<false>(dY, R, T, out, r, G, d, st, dR, r * out, dL, in * r)) return rc;
    // dR^T = dY^T . XL  (dR stored [r x out])
    if (int rc = token_reduction(dY, XL, T, out, r, dR, true, d, st)) return rc;
    // dL = X^T . G
    return token_reduction(X, G, T, in, r, dL, false, d, st);
}

}  // extern "C"
