/*
 * slope.h -- C ABI of libslope.so: the SLoPe 2:4 double-pruned sparse linear
 * layer with a lazy low-rank adapter, as sm_100a (B200) CUDA kernels.
 *
 * Sources for what each call computes (the method has no printed code here;
 * these are the passages the definitions follow):
 *   [S2A] SLoPe technical summary (gist.science), §2.A "Double-Pruned Backward
 *         Pass": the forward pass uses the row-wise pruned W^R, the backward
 *         pass the double-pruned W^{R,C}, obtained by transposing the already
 *         N:M-sparse matrix and imposing N:M sparsity again.
 *   [S1]  same page, §1 "Structured Sparsity (N:M)": N:M constrains groups of
 *         M consecutive elements (2:4 keeps two of every four).
 *   [S2B] same page, §2.B "Lazy Low-Rank Adapters": W_dense = W_sparse + L R.
 *   [S2C] same page, §2.C "Optimized CUDA Kernels": the sparse product and the
 *         low-rank adapter are fused into one kernel.
 *   [RM]  SLoPe OpenReview rebuttal (paperhub.cn), "Memory Footprint Reduction
 *         During Pretraining and Inference": non-zeros plus index bits per
 *         four weights; the transposed copy is stored for the backward pass;
 *         the gradient holds only the non-zeros (2 x 16 bits per four).
 *   [RI]  same page, "SLoPe inference computation": adapters are not merged;
 *         inference runs the sparse product alongside the low-rank product.
 *   [RF]  same page, "SLoPe downstream finetuning": the mask is kept and only
 *         non-zero weights are updated.
 *
 * Conventions for every call:
 *   - bf16 tensors are passed as uint16_t pointers to their bit patterns;
 *     every matrix is dense row-major with no padding between rows.
 *   - All tensor pointers are DEVICE pointers to memory the caller allocated
 *     and owns; each must be 16-byte aligned.  The library keeps no state
 *     between calls except a per-device error word (see slope_status_sync),
 *     a per-thread error string and the per-device fp32 workspaces of the
 *     products it splits over their reduction dimension (slope_fwd and
 *     slope_bwd_dx at few tokens, slope_bwd_dw_masked on layers with few
 *     tiles, slope_adapter_fwd / slope_adapter_bwd at few tokens).
 *     Workspaces (a reading of the boundary's "allocates nothing persistent":
 *     these are the library's own scratch, not outputs):
 *       * allocated on first need and grown when a larger shape needs more;
 *         an outgrown buffer is kept allocated until the process exits, so a
 *         CUDA graph captured earlier stays valid and replays into memory
 *         that still belongs to it;
 *       * growth may happen while the caller's stream is being captured:
 *         the allocation and its zeroing run outside the capture (relaxed
 *         capture mode, a private stream waited for before the call
 *         returns), so no warm-up call is needed before capture;
 *       * one workspace serves every call of its kind on a device, so such
 *         calls must not overlap in time (calls on one stream never do; on
 *         several streams, or from several host threads without ordering,
 *         they race).  The host-side tables are guarded by a mutex.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *     only enqueues work on it and returns at once; argument errors are
 *     detected on the host before anything is enqueued.
 *   - Return value: SLOPE_OK or one of the SLOPE_ERR_* codes below; the
 *     matching message is in slope_last_error().  Nothing throws.
 *   - Shapes: in_features and out_features must be positive multiples of 64;
 *     tokens T >= 1 (any value); adapter rank r = 0 (no adapter: L, R, XL, G
 *     may then be NULL) or a multiple of 8 up to 256.  A rank that is not a
 *     multiple of 8 is stored zero-padded (extra zero columns of L and zero
 *     rows of R), which leaves every output unchanged.
 *   - Compressed 2:4 format ("vals/meta"): a matrix S [rows x K] whose every
 *     group of four consecutive elements of a row holds at most two non-zeros
 *     is stored as vals [rows x K/2] (the two kept values of each group, in
 *     ascending position) and meta [rows x K/16] uint16 (group g of a row is
 *     the 4-bit code i0 | i1 << 2 of its kept positions, i0 < i1, stored in
 *     bits 4*(g%4)..4*(g%4)+3 of word g/4).  Legal codes: 0x4 0x8 0xC 0x9 0xD 0xE.
 */
#ifndef SLOPE_H
#define SLOPE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
    SLOPE_OK = 0,
    SLOPE_ERR_ARG = 1,         /* NULL pointer where one is required, negative size */
    SLOPE_ERR_SHAPE = 2,       /* size rule above violated                           */
    SLOPE_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned                   */
    SLOPE_ERR_NONFINITE = 4,   /* prune24 saw NaN or Inf (reported by slope_status_sync) */
    SLOPE_ERR_TIMEOUT = 5,     /* a kernel's bounded wait ran out (slope_status_sync) */
    SLOPE_ERR_CUDA = 6,        /* a CUDA runtime or driver call failed               */
    SLOPE_ERR_UNSUPPORTED = 7, /* the current device is not sm_100                   */
    SLOPE_ERR_BOUNDS = 8       /* debug build only: a kernel's global-memory index fell
                                  outside its buffer; the access was skipped (slope_status_sync) */
};

/*
 * Row-wise 2:4 magnitude pruning [S1][S2A], done once when the static mask is
 * set: W [rows x K] (dense bf16) -> vals [rows x K/2], meta [rows x K/16].
 * In each group the two largest |w| are kept; ties go to the lower position
 * and +0/-0 count as equal; kept values are copied bit for bit.  NaN/Inf in W
 * sets SLOPE_ERR_NONFINITE in the device error word (outputs are then
 * unspecified).  K must be a multiple of 64, rows >= 1.
 */
int slope_prune24(const uint16_t *W, int64_t rows, int64_t K, uint16_t *vals, uint16_t *meta,
                  void *stream);

/*
 * General N:M magnitude pruning along rows [S1] (only 2:4 has tensor-core
 * support; this is the stored form for any other pattern): for every group
 * of M consecutive elements of a row of W [rows x K] bf16, keep the N of
 * largest magnitude (ties to the lower position, +0 == -0) and write them in
 * ascending position to vals [rows x K*N/M] bf16, and their positions
 * (0 .. M-1) to pos [rows x K*N/M] uint8.  M in {4, 8, 16}, 1 <= N < M,
 * K a multiple of M (else SLOPE_ERR_SHAPE); NaN/Inf in W sets
 * SLOPE_ERR_NONFINITE as slope_prune24 does.  W, vals and pos are 16-byte
 * aligned like every tensor here (SLOPE_ERR_ALIGN otherwise).  With N = 2,
 * M = 4 the kept values equal slope_prune24's and the positions are its
 * codes' fields.
 */
int slope_prune_nm(const uint16_t *W, int64_t rows, int64_t K, int N, int M, uint16_t *vals, uint8_t *pos,
                   void *stream);

/*
 * Double pruning [S2A][RM]: from W^R (compressed, [out x in]) build the
 * backward-pass copy W^{R,C}, stored TRANSPOSED and compressed:
 * vals_t [in x out/2], meta_t [in x out/16].  Row i of the result is column i
 * of W^R pruned 2:4 along out with the prune24 rule (pruned positions of W^R
 * count as +0; a group with fewer than two non-zeros keeps its lowest-index
 * zeros).  Run after every update of vals, because the column mask follows
 * the values.
 */
int slope_double_prune(const uint16_t *vals, const uint16_t *meta, int64_t out, int64_t in,
                       uint16_t *vals_t, uint16_t *meta_t, void *stream);

/*
 * Both prunings in one pass [S1][S2A][RM]: from dense W [out x in] bf16,
 * the row-wise 2:4 pruning of slope_prune24 (vals [out x in/2],
 * meta [out x in/16]) and, from that W^R, the transposed second pruning of
 * slope_double_prune (vals_t [in x out/2], meta_t [in x out/16]); every
 * output bit for bit equal to slope_prune24 followed by slope_double_prune.
 * One launch that reads W once and never reads W^R back (4.25 bytes moved per
 * weight instead of 5.375).  out and in multiples of 64; NaN/Inf in W sets
 * SLOPE_ERR_NONFINITE as slope_prune24 does.
 */
int slope_prune24_double(const uint16_t *W, int64_t out, int64_t in, uint16_t *vals, uint16_t *meta,
                         uint16_t *vals_t, uint16_t *meta_t, void *stream);

/*
 * Compressed AdamW step fused with the second pruning [RM][RF], one pass:
 * the kept values of W^R (vals, updated in place) take one AdamW step from
 * the compressed gradient dW_vals (slope_bwd_dw_masked's output, same slots)
 * with fp32 states m, v [out x in/2] (updated in place; zero before the first
 * step), the mask staying as it is; then the updated W^R is transposed and
 * pruned 2:4 again into vals_t/meta_t exactly as slope_double_prune does.
 * The rebuttal fixes the optimizer (AdamW, "Choice of Optimizer") and its
 * state budget (two 32-bit states per non-zero); the step is the
 * decoupled-decay form, each operation one correctly rounded binary32
 * operation in this order, w rounded once to bf16 (nearest even):
 *     w <- w * (1 - lr * weight_decay)
 *     m <- beta1 * m + (1 - beta1) * g,  v <- beta2 * v + (1 - beta2) * (g * g)
 *     w <- w - step_size * (m / (sqrt(v) * inv_sqrt_bc2 + eps))
 * with step_size = lr / (1 - beta1^step) and inv_sqrt_bc2 =
 * 1 / sqrt(1 - beta2^step) evaluated in binary64 and rounded to binary32.
 * step >= 1 (the step number, 1 for the first), 0 <= beta1, beta2 < 1,
 * eps > 0, lr >= 0; else SLOPE_ERR_ARG.  m and v must be 16-byte aligned.
 * Same shape rules as slope_double_prune.  No counterpart in the pages'
 * kernels: they name the optimizer and its memory, not a kernel.
 */
int slope_adamw_double_prune(uint16_t *vals, const uint16_t *meta, const uint16_t *dW_vals, float *m, float *v,
                             int64_t out, int64_t in, float lr, float beta1, float beta2, float eps,
                             float weight_decay, int64_t step, uint16_t *vals_t, uint16_t *meta_t, void *stream);

/*
 * Adapter down-projection [S2B]: XL = X . L, X [T x in], L [in x r] -> XL
 * [T x r] bf16 (fp32 accumulation, rounded to nearest even).  r >= 8.
 * Up to 32 tokens the product runs on CUDA cores split over K, its partials
 * summed in a fixed order.  With few token tiles above that, the tensor-core
 * product splits K and adds the partials into an fp32 accumulator with
 * atomics, so the last bit of an output can vary between runs.  Both use
 * the per-device workspaces described above.
 */
int slope_adapter_fwd(const uint16_t *X, const uint16_t *L, int64_t T, int64_t in, int64_t r,
                      uint16_t *XL, void *stream);

/*
 * Sparse forward [S2A][S2B][S2C][RI]: Y = X . (W^R)^T + XL . R.
 * X [T x in]; vals/meta = W^R [out x in] compressed; XL [T x r]; R [r x out];
 * Y [T x out] bf16.  One kernel: 2:4 sparse tensor-core products over in, then
 * the rank-r term accumulated into the same fp32 tile, rounded once.
 * At few tokens (a layer with fewer output tiles than SM pairs, see
 * slope_sparse_plan) the sum over in is split into up to 8 ranges whose fp32
 * partials, summed in range order, go through a per-device workspace (about
 * splits x out x BN floats; see the conventions above).
 */
int slope_fwd(const uint16_t *X, const uint16_t *vals, const uint16_t *meta, const uint16_t *XL,
              const uint16_t *R, int64_t T, int64_t in, int64_t out, int64_t r, uint16_t *Y,
              void *stream);

/*
 * Forward with the adapter's down-projection in the same launch [S2B][S2C]
 * ([S2C]: the sparse product and the low-rank adapter in one kernel, the
 * down-projection concatenated with the sparse weights): XL = X . L is
 * computed first by the launch's own tensor-core units (256 tokens each,
 * written to XL [T x r] bf16, which the backward needs) and then
 * Y = X . (W^R)^T + XL . R as in slope_fwd; XL is rounded once to bf16
 * before its product with R, exactly as slope_adapter_fwd + slope_fwd.
 * Arguments as slope_adapter_fwd and slope_fwd (L [in x r], R [r x out]).
 * One launch when in is a multiple of 128, at least 512, 0 < r <= 128, and
 * the launch planner's cost model favours it (slope_fused_launches says which:
 * the fused launch's 512 x 224 tiles have no split of the sum over in, so
 * with a few tokens, or few output rows against a long reduction, they
 * leave SM pairs idle); otherwise the same two launches as
 * slope_adapter_fwd + slope_fwd.  Only the one-launch form is
 * bit-reproducible run to run (its sums run in a fixed order); the two-launch
 * form inherits slope_adapter_fwd's.  r = 0: plain slope_fwd (L, R, XL may
 * be NULL).  Uses a per-device flag workspace like the split workspaces
 * above.
 */
int slope_fwd_fused(const uint16_t *X, const uint16_t *vals, const uint16_t *meta, const uint16_t *L,
                    const uint16_t *R, int64_t T, int64_t in, int64_t out, int64_t r, uint16_t *XL, uint16_t *Y,
                    void *stream);

/*
 * Input gradient with the adapter's G = dY . R^T in the same launch
 * (chain rule on [S2B]; [S2C]): G [T x r] bf16 is computed first by the
 * launch's own units and written (slope_bwd_dw_fused needs it), then
 * dX = dY . W^{R,C} + G . L^T as in slope_bwd_dx.  Conditions and fallback
 * as slope_fwd_fused, with out in place of in and in in place of out.
 */
int slope_bwd_dx_fused(const uint16_t *dY, const uint16_t *vals_t, const uint16_t *meta_t, const uint16_t *R,
                       const uint16_t *L, int64_t T, int64_t in, int64_t out, int64_t r, uint16_t *G, uint16_t *dX,
                       void *stream);

/*
 * Adapter backward (chain rule on [S2B]): G = dY . R^T [T x r] (bf16),
 * dR = XL^T . dY [r x out] (fp32), dL = X^T . G [in x r] (fp32).
 * dL uses G as this call stores it (bf16).  dL and dR are overwritten.
 * G is computed like XL in slope_adapter_fwd; dR and dL are split over
 * tokens and summed with fp32 atomics (their last bits can vary between runs).
 */
int slope_adapter_bwd(const uint16_t *X, const uint16_t *dY, const uint16_t *XL, const uint16_t *R,
                      int64_t T, int64_t in, int64_t out, int64_t r, float *dL, float *dR,
                      uint16_t *G, void *stream);

/*
 * Sparse input gradient [S2A][S2B]: dX = dY . W^{R,C} + G . L^T.
 * dY [T x out]; vals_t/meta_t = (W^{R,C})^T [in x out] compressed (from
 * slope_double_prune); G [T x r]; L [in x r]; dX [T x in] bf16.  The same
 * kernel as slope_fwd (with M = in, K = out), split the same way at few
 * tokens.
 */
int slope_bwd_dx(const uint16_t *dY, const uint16_t *vals_t, const uint16_t *meta_t,
                 const uint16_t *G, const uint16_t *L, int64_t T, int64_t in, int64_t out,
                 int64_t r, uint16_t *dX, void *stream);

/*
 * Masked weight gradient [RM][RF]: dW = (dY^T . X) at the static mask's
 * positions only, written compressed in W^R's slot order:
 * dW_vals [out x in/2] bf16, dW_vals[o][2g+s] = sum_t dY[t][o] X[t][4g+i_s]
 * where (i_0, i_1) are the kept positions of group g of row o in `meta`.
 * Layers with few 256 x 256 tiles are split over tokens: the fp32 partials go
 * to a per-device workspace (about splits x out x in/2 floats; see the
 * conventions above), summed in split order by the last split to arrive.
 */
int slope_bwd_dw_masked(const uint16_t *dY, const uint16_t *X, const uint16_t *meta, int64_t T,
                        int64_t in, int64_t out, uint16_t *dW_vals, void *stream);

/*
 * Masked weight gradient with the adapter gradients in the same launch
 * ([RM][RF] for dW; chain rule on [S2B] for dR and dL; [S2C] for the fusion):
 * dW_vals as slope_bwd_dw_masked, dR = XL^T . dY [r x out] and
 * dL = X^T . G [in x r] (fp32, overwritten), from XL and G as
 * slope_fwd_fused / slope_bwd_dx_fused wrote them.  The dR and dL units run
 * after the dW tiles over the same operand loads of dY and X, split over
 * tokens like them; split partials are summed in split order, so every
 * output is the same bit for bit from run to run (unlike slope_adapter_bwd's
 * atomics).  0 < r <= 128 (larger ranks: slope_bwd_dw_masked plus the
 * separate reductions; r = 0: slope_bwd_dw_masked, XL, G, dL, dR may be
 * NULL).  Uses per-device workspaces like slope_bwd_dw_masked.
 */
int slope_bwd_dw_fused(const uint16_t *dY, const uint16_t *X, const uint16_t *meta, const uint16_t *XL,
                       const uint16_t *G, int64_t T, int64_t in, int64_t out, int64_t r, uint16_t *dW_vals, float *dL,
                       float *dR, void *stream);

/*
 * slope_bwd_dw_masked for callers that cannot allocate device memory (a
 * fixed memory budget, an allocator that must not be entered).  The pages
 * have no counterpart: it is the same masked weight gradient, same kernel,
 * same plan and bit-identical results, but the token-split scratch comes from
 * a fixed array in this library's own device memory instead of an allocated
 * workspace.  This call allocates nothing, on the device or the host.
 *
 * Limit: a layer whose plan splits over tokens needs splits x out x in/2
 * floats of scratch and 8 counters per 256-row x BN tile; beyond
 * SLOPE_NOALLOC_SCRATCH_FLOATS / SLOPE_NOALLOC_SCRATCH_COUNTERS the call
 * returns SLOPE_ERR_SHAPE and launches nothing (slope_bwd_dw_masked handles
 * any size).  Layers that are not split need no scratch and have no limit.
 *
 * The scratch is one per device and shared by all calls: two calls of this
 * entry point on the same device that can overlap (on different streams, or
 * on different host threads without ordering) race on it and give wrong
 * results.  Serialise them, for instance on one stream.
 */
#define SLOPE_NOALLOC_SCRATCH_FLOATS (1 << 22)   /* 16 MiB of fp32 partials */
#define SLOPE_NOALLOC_SCRATCH_COUNTERS 4096
int slope_bwd_dw_masked_noalloc(const uint16_t *dY, const uint16_t *X, const uint16_t *meta, int64_t T,
                                int64_t in, int64_t out, uint16_t *dW_vals, void *stream);

/*
 * Wait for `stream`, then read and clear the current device's error word:
 * returns SLOPE_OK, SLOPE_ERR_NONFINITE, SLOPE_ERR_TIMEOUT, SLOPE_ERR_BOUNDS
 * (debug build) or SLOPE_ERR_CUDA.
 */
int slope_status_sync(void *stream);

/*
 * 1 in the debug build of this library (compiled with -DSLOPE_DEBUG_BOUNDS),
 * else 0 (no counterpart in the pages).  In the debug build every plain
 * global-memory load and store of the kernels checks its index range against
 * the extent of its buffer that the host derived from the call's sizes (TMA
 * tiles are bounded by their tensor maps and need no check); an access
 * outside it is skipped and recorded, and the next slope_status_sync returns
 * SLOPE_ERR_BOUNDS.  Nothing traps.  The checks cost time: the debug build is
 * for tests, not for measurement.
 */
int slope_debug_bounds(void);

/* SLOPE_OK when the current device is sm_100 (B200), else SLOPE_ERR_UNSUPPORTED. */
int slope_device_check(void);

/*
 * Self-test of the failure path (no counterpart in the pages).  It launches
 * one thread that waits on a barrier no one signals, with the same bounded
 * wait the kernels use but a limit of about 10 ms, after which it records a
 * timeout and returns.  A following slope_status_sync returns
 * SLOPE_ERR_TIMEOUT and clears it; the device stays usable.  Nothing faults,
 * traps or hangs.
 */
int slope_selftest_wait_timeout(void *stream);

/*
 * Launch plan of the sparse products (host only, no device call; no
 * counterpart in the pages): for an M x K sparse operand (M = out, K = in for
 * slope_fwd; M = in, K = out for slope_bwd_dx) times T tokens on a device
 * with `sms` SMs, the token-tile width BN (16 .. 240) and the number of
 * ranges the sum over K is split into (1 = no split) that those calls use.
 * Returns SLOPE_ERR_ARG for NULL outputs or non-positive sizes.
 */
int slope_sparse_plan(int64_t M, int64_t T, int64_t K, int sms, int *bn, int *splits);

/*
 * Launches of slope_fwd_fused (M = out, K = in) or slope_bwd_dx_fused
 * (M = in, K = out) for these sizes and rank on a device with `sms` SMs
 * (host only, no device call; no counterpart in the pages): 1 when the rank
 * product runs inside the sparse product's launch (or r = 0), 2 when it
 * takes a launch of its own.  The choice sets the planner's best 256-row
 * pair tiles (slope_sparse_plan) plus the cost of the extra launch against
 * the fused launch's 512-row tiles.  Returns SLOPE_ERR_ARG for a NULL
 * output or bad sizes.
 */
int slope_fused_launches(int64_t M, int64_t T, int64_t K, int64_t r, int sms, int *launches);

/*
 * Height of the sparse products' output tile (host only, no device call; no
 * counterpart in the pages) for the same arguments as slope_sparse_plan:
 * 256 (one 256-row block per SM pair, the kernel slope_sparse_plan
 * describes) or 512 (two 256-row blocks per SM pair sharing the token
 * operand, taken for long reductions: K a multiple of 128, at least 1024,
 * and enough tiles that the unhidden epilogue is cheap; the token tile is
 * then 224 wide and the sum over K is not split).  Returns SLOPE_ERR_ARG for
 * a NULL output or non-positive sizes.
 */
int slope_sparse_tile_rows(int64_t M, int64_t T, int64_t K, int sms, int *rows);

/* Message of the last failing call on this host thread ("" if none). */
const char *slope_last_error(void);

/* Number of kernels this library launched on this host thread since the last
 * reset (reset = nonzero argument); used to count launches in benchmarks. */
int64_t slope_launch_count(int reset);

#ifdef __cplusplus
}
#endif

#endif /* SLOPE_H */
