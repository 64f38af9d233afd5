// slope_api.cu -- the C ABI of libslope.so (declared in include/slope.h):
// argument checks on the host, TMA tensor-map encoding, kernel launches.
// All kernels of the library live in this one translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "../../include/slope.h"
#include "gemm.cuh"
#include "prune.cuh"

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

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D bf16 tensor [rows x cols] (cols contiguous, row pitch `ld` elements),
// box [box_rows x box_cols], 128-byte swizzle, out-of-bounds reads as zero.
int make_map(CUtensorMap &m, const void *base, int64_t rows, int64_t cols, int64_t ld, int box_cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(SLOPE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(SLOPE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for [%lld x %lld] box [%d x %d]", (int)r,
                    (long long)rows, (long long)cols, box_rows, box_cols);
    return SLOPE_OK;
}

// ------------------------------------------------------------------ launches
template <bool SPARSE, bool A_MN, bool B_MN, bool A2_MN, int EPI, int BN>
int launch_gemm(const CUtensorMap &a, const CUtensorMap &b, const CUtensorMap &a2, const CUtensorMap &b2,
                const slope::GemmParams &p, int sms, cudaStream_t st) {
    using C = slope::GemmCfg<SPARSE, BN>;
    auto kern = slope::gemm_kernel<SPARSE, A_MN, B_MN, A2_MN, EPI, BN>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemm)");
        attr_set = true;
    }
    if (p.num_work <= 0) return SLOPE_OK;
    const int grid = p.num_work < sms ? p.num_work : sms;
    kern<<<grid, C::NUM_WARPS * 32, C::SMEM_BYTES, st>>>(a, b, a2, b2, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
    ++g_launches;
    return SLOPE_OK;
}

slope::GemmParams base_params(int64_t M, int64_t N, int BN) {
    slope::GemmParams p{};
    p.M = (int)M;
    p.N = (int)N;
    p.num_m_tiles = (int)((M + 127) / 128);
    p.num_n_tiles = (int)((N + BN - 1) / BN);
    p.num_splits = 1;
    return p;
}

// Split K so that the work list roughly fills the GPU; every split non-empty.
void set_splits(slope::GemmParams &p, int k_tiles, int sms) {
    const int tiles = p.num_m_tiles * p.num_n_tiles;
    int splits = (sms + tiles - 1) / tiles;
    if (splits > k_tiles) splits = k_tiles;
    if (splits < 1) splits = 1;
    const int per = (k_tiles + splits - 1) / splits;
    p.k_tiles_total = k_tiles;
    p.k_tiles_per_split = per;
    p.num_splits = (k_tiles + per - 1) / per;
    p.num_work = tiles * p.num_splits;
}

int zero_f32(float *p, int64_t n, cudaStream_t st);

}  // namespace

// zero-fill helper kernel for the split-K outputs
__global__ void zero_f32_kernel(float *p, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        p[i] = 0.0f;
}

namespace {
int zero_f32(float *p, int64_t n, cudaStream_t st) {
    int blocks = (int)((n + 255) / 256);
    if (blocks > 4096) blocks = 4096;
    zero_f32_kernel<<<blocks, 256, 0, st>>>(p, n);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "zero launch");
    ++g_launches;
    return SLOPE_OK;
}
}  // namespace

extern "C" {

const char *slope_last_error(void) { return g_err; }

int64_t slope_launch_count(int reset) {
    int64_t v = g_launches;
    if (reset) g_launches = 0;
    return v;
}

int slope_device_check(void) {
    DevInfo d;
    return device_info(d);
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
    if (word & slope::ST_TIMEOUT) return fail(SLOPE_ERR_TIMEOUT, "a kernel's bounded wait timed out");
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
    int64_t blocks = (chunks + 255) / 256;
    const int64_t cap = (int64_t)d.sms * 8;
    if (blocks > cap) blocks = cap;
    slope::prune24_kernel<<<(int)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(W, vals, meta, chunks);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "prune24 launch");
    ++g_launches;
    return SLOPE_OK;
}

int slope_double_prune(const uint16_t *vals, const uint16_t *meta, int64_t out, int64_t in, uint16_t *vals_t,
                       uint16_t *meta_t, void *stream) {
    CHECK_PTR(vals);
    CHECK_PTR(meta);
    CHECK_PTR(vals_t);
    CHECK_PTR(meta_t);
    if (int rc = check_features(out, "out")) return rc;
    if (int rc = check_features(in, "in")) return rc;
    DevInfo d;
    if (int rc = device_info(d)) return rc;
    const int64_t tiles = (out / slope::DP_TILE) * (in / slope::DP_TILE);
    int64_t blocks = tiles < (int64_t)d.sms * 8 ? tiles : (int64_t)d.sms * 8;
    slope::double_prune_kernel<<<(int)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(vals, meta, (int)out,
                                                                                           (int)in, vals_t, meta_t);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "double_prune launch");
    ++g_launches;
    return SLOPE_OK;
}

// Sparse product with the fused adapter phase.  A = compressed [M x K]
// (vals [M x K/2], meta), B = dense [T x K]; adapter: A2 = R^T (from R
// [r x M], MN-major) when a2_is_r, else A2 = L [M x r] (K-major); B2 = [T x r].
static int sparse_product(const uint16_t *B, const uint16_t *vals, const uint16_t *meta, const uint16_t *B2,
                          const uint16_t *A2, bool a2_is_r, int64_t T, int64_t K, int64_t M, int64_t r,
                          uint16_t *out, cudaStream_t st) {
    DevInfo d;
    if (int rc = device_info(d)) return rc;
    constexpr int BN = 128;
    CUtensorMap ta, tb, ta2, tb2;
    if (int rc = make_map(ta, vals, M, K / 2, K / 2, 64, 128)) return rc;
    if (int rc = make_map(tb, B, T, K, K, 64, BN)) return rc;
    if (r > 0) {
        if (a2_is_r) {
            if (int rc = make_map(ta2, A2, r, M, M, 64, 64)) return rc;
        } else {
            if (int rc = make_map(ta2, A2, M, r, r, 64, 128)) return rc;
        }
        if (int rc = make_map(tb2, B2, T, r, r, 64, BN)) return rc;
    } else {
        ta2 = ta;
        tb2 = tb;
    }
    slope::GemmParams p = base_params(M, T, BN);
    p.k_tiles_total = (int)((K + 127) / 128);
    p.k_tiles_per_split = p.k_tiles_total;
    p.num_work = p.num_m_tiles * p.num_n_tiles;
    p.k_logical = (int)K;
    p.r = (int)r;
    p.adp_k_tiles = (int)((r + 63) / 64);
    p.meta_a = meta;
    p.out = out;
    p.ld_out = M;
    if (a2_is_r)
        return launch_gemm<true, false, false, true, slope::EPI_BF16_T, BN>(ta, tb, ta2, tb2, p, d.sms, st);
    return launch_gemm<true, false, false, false, slope::EPI_BF16_T, BN>(ta, tb, ta2, tb2, p, d.sms, st);
}

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
    constexpr int BN = 128;
    CUtensorMap ta, tb;
    if (int rc = make_map(ta, dY, T, out, out, 64, 64)) return rc;  // A = dY^T, MN-major
    if (int rc = make_map(tb, X, T, in, in, 64, 64)) return rc;     // B = X, MN-major
    slope::GemmParams p = base_params(out, in, BN);
    p.k_tiles_total = (int)((T + 63) / 64);
    p.k_tiles_per_split = p.k_tiles_total;
    p.num_work = p.num_m_tiles * p.num_n_tiles;
    p.meta_mask = meta;
    p.out = dW_vals;
    p.ld_out = in / 2;
    return launch_gemm<false, true, true, false, slope::EPI_DW_COMPRESS, BN>(ta, tb, ta, tb, p, d.sms,
                                                                              static_cast<cudaStream_t>(stream));
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
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    CUtensorMap ta, tb;
    if (int rc = make_map(ta, X, T, in, in, 64, 128)) return rc;  // A = X, K-major
    if (int rc = make_map(tb, L, in, r, r, 64, 64)) return rc;    // B = L^T from L [in x r], MN-major
    const int kt = (int)((in + 63) / 64);
    if (r <= 64) {
        slope::GemmParams p = base_params(T, r, 64);
        p.k_tiles_total = kt;
        p.k_tiles_per_split = kt;
        p.num_work = p.num_m_tiles * p.num_n_tiles;
        p.out = XL;
        p.ld_out = r;
        return launch_gemm<false, false, true, false, slope::EPI_BF16_ROW, 64>(ta, tb, ta, tb, p, d.sms, st);
    }
    slope::GemmParams p = base_params(T, r, 128);
    p.k_tiles_total = kt;
    p.k_tiles_per_split = kt;
    p.num_work = p.num_m_tiles * p.num_n_tiles;
    p.out = XL;
    p.ld_out = r;
    return launch_gemm<false, false, true, false, slope::EPI_BF16_ROW, 128>(ta, tb, ta, tb, p, d.sms, st);
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
    const bool wide = r > 64;
    // 1) G = dY . R^T : M = T, N = r, K = out; A = dY (K-major), B = R [r x out] (K-major)
    {
        CUtensorMap ta, tb;
        if (int rc = make_map(ta, dY, T, out, out, 64, 128)) return rc;
        const int bn = wide ? 128 : 64;
        if (int rc = make_map(tb, R, r, out, out, 64, bn)) return rc;
        slope::GemmParams p = base_params(T, r, bn);
        const int kt = (int)((out + 63) / 64);
        p.k_tiles_total = kt;
        p.k_tiles_per_split = kt;
        p.num_work = p.num_m_tiles * p.num_n_tiles;
        p.out = G;
        p.ld_out = r;
        int rc = wide ? launch_gemm<false, false, false, false, slope::EPI_BF16_ROW, 128>(ta, tb, ta, tb, p, d.sms, st)
                      : launch_gemm<false, false, false, false, slope::EPI_BF16_ROW, 64>(ta, tb, ta, tb, p, d.sms, st);
        if (rc) return rc;
    }
    if (int rc = zero_f32(dR, r * out, st)) return rc;
    if (int rc = zero_f32(dL, in * r, st)) return rc;
    const int ktT = (int)((T + 63) / 64);
    // 2) dR^T = dY^T . XL : M = out, N = r, K = T; A = dY^T (MN-major), B = XL (MN-major)
    {
        CUtensorMap ta, tb;
        if (int rc = make_map(ta, dY, T, out, out, 64, 64)) return rc;
        if (int rc = make_map(tb, XL, T, r, r, 64, 64)) return rc;
        const int bn = wide ? 128 : 64;
        slope::GemmParams p = base_params(out, r, bn);
        set_splits(p, ktT, d.sms);
        p.out = dR;
        p.ld_out = out;
        int rc = wide ? launch_gemm<false, true, true, false, slope::EPI_F32_ADD_T, 128>(ta, tb, ta, tb, p, d.sms, st)
                      : launch_gemm<false, true, true, false, slope::EPI_F32_ADD_T, 64>(ta, tb, ta, tb, p, d.sms, st);
        if (rc) return rc;
    }
    // 3) dL = X^T . G : M = in, N = r, K = T; A = X^T (MN-major), B = G (MN-major)
    {
        CUtensorMap ta, tb;
        if (int rc = make_map(ta, X, T, in, in, 64, 64)) return rc;
        if (int rc = make_map(tb, G, T, r, r, 64, 64)) return rc;
        const int bn = wide ? 128 : 64;
        slope::GemmParams p = base_params(in, r, bn);
        set_splits(p, ktT, d.sms);
        p.out = dL;
        p.ld_out = r;
        int rc = wide ? launch_gemm<false, true, true, false, slope::EPI_F32_ADD_ROW, 128>(ta, tb, ta, tb, p, d.sms, st)
                      : launch_gemm<false, true, true, false, slope::EPI_F32_ADD_ROW, 64>(ta, tb, ta, tb, p, d.sms, st);
        if (rc) return rc;
    }
    return SLOPE_OK;
}

}  // extern "C"
