/*
 * SLoPe layer oracle -- plain, slow, scalar C.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests, __graft_entry__.smoke() and the CPU-baseline
 * leg of bench.py use it.  It shares no code, header, table or constant with
 * the CUDA library; the two meet only through the seeded input generators.
 *
 * What it computes (the 2:4 double-pruned sparse linear layer with a lazy
 * low-rank adapter):
 *   - prune24:        row-wise 2:4 magnitude pruning of W [out x in] along in
 *                     (SLoPe technical summary (gist.science), §1 "Structured
 *                     Sparsity (N:M)" and §2.A "Mechanism / Forward Pass").
 *   - double_prune:   transpose the already 2:4-sparse W^R and prune it to 2:4
 *                     again along the new rows, giving W^{R,C}
 *                     (same page, §2.A "Approach" and "Backward Pass").
 *   - adapter_fwd:    XL = X . L                (same page, §2.B: W = W_sparse + L R)
 *   - fwd:            Y = X . (W^R)^T + XL . R  (§2.A forward pass + §2.B; the
 *                     adapter is kept unmerged, SLoPe OpenReview rebuttal
 *                     (paperhub.cn), "SLoPe inference computation")
 *   - adapter_bwd:    G = dY . R^T, dR = XL^T . dY, dL = X^T . G  (chain rule on §2.B)
 *   - bwd_dx:         dX = dY . W^{R,C} + G . L^T                 (§2.A backward pass)
 *   - bwd_dw_masked:  dW = (dY^T . X) restricted to the static mask M
 *                     (rebuttal, "Memory Footprint Reduction ...": gradient
 *                     stored as 2*16 bits per four weights; rebuttal,
 *                     "SLoPe downstream finetuning": only non-zeros updated).
 *   - prune_nm:       row-wise N:M magnitude pruning for general N < M
 *                     (same page, §1: N:M keeps N of every M consecutive
 *                     elements; only 2:4 has tensor-core support, so this
 *                     form stores each kept value's position in a byte).
 *   - adamw_compressed: one AdamW step on the kept values only, with fp32
 *                     states for the non-zeros (rebuttal, "Memory Footprint
 *                     Reduction ...": optimizer states 2 * 2 * 32 bits per
 *                     four weights; "Choice of Optimizer": AdamW), the mask
 *                     left as it is (rebuttal, "SLoPe downstream finetuning").
 *   - mem_ratio:      the per-four-element memory arithmetic of the rebuttal
 *                     section "Memory Footprint Reduction During Pretraining
 *                     and Inference" (printed results 54% and 68%).
 *
 * Storage format (fixed by this project, not by the pages): for every group
 * of four consecutive elements of a row, the two kept values are stored in
 * ascending index order, and a 4-bit code i0 | i1 << 2 (i0 < i1) records
 * their positions.  Codes of groups 4w..4w+3 of a row share the 16-bit word
 * w, group 4w+q in bits 4q..4q+3.
 *
 * Readings where the pages are silent:
 *   - the pruning criterion is magnitude; ties go to the lower index; +0 and
 *     -0 have equal magnitude; values are copied bit for bit;
 *   - the second pruning uses the same rule on the columns of W^R, where
 *     pruned positions hold +0; a group with fewer than two non-zeros keeps
 *     its lowest-index zeros, so every group still has a legal code;
 *   - NaN or Inf in W is a precondition violation (status ORACLE_NONFINITE);
 *   - floating point: inputs are bf16 (decoded exactly), every sum is taken
 *     in fp64 in ascending index order, nothing is rounded on the way;
 *   - AdamW is the decoupled-decay form (decay the weight by 1 - lr * wd,
 *     then the bias-corrected Adam step), in binary32 in the fixed order
 *     written out below, the weight rounded once to bf16 (nearest even):
 *     the updated weights decide the second pruning's integer choices, so
 *     both sides take them in the same precision.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_SHAPE 1
#define ORACLE_NONFINITE 2

/* bf16 bit pattern -> its exact value (bf16 is the top half of a binary32). */
static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int bf16_is_nonfinite(uint16_t bits) { return (bits & 0x7F80u) == 0x7F80u; }

/* Magnitude of a finite bf16 as an integer: clearing the sign bit leaves a
 * pattern whose unsigned order is the order of |value| (IEEE-754 layout). */
static unsigned bf16_magnitude(uint16_t bits) { return bits & 0x7FFFu; }

/*
 * Top-2-of-4 selection.  Element k survives iff fewer than two elements beat
 * it, where m beats k when |v_m| > |v_k|, or |v_m| == |v_k| and m < k.
 * Exactly two survive; they are returned in ascending index order.
 */
static void keep_two_of_four(const uint16_t v[4], int *i0, int *i1)
{
    int kept[4], n = 0;
    for (int k = 0; k < 4; ++k) {
        int beaten_by = 0;
        for (int m = 0; m < 4; ++m) {
            if (bf16_magnitude(v[m]) > bf16_magnitude(v[k]) ||
                (bf16_magnitude(v[m]) == bf16_magnitude(v[k]) && m < k))
                beaten_by++;
        }
        if (beaten_by < 2) kept[n++] = k;
    }
    *i0 = kept[0];
    *i1 = kept[1];
}

static unsigned code_of(const uint16_t *meta, int64_t words_per_row, int64_t row, int64_t group)
{
    uint16_t w = meta[row * words_per_row + group / 4];
    return (w >> (4 * (group % 4))) & 0xFu;
}

/* Set the 4-bit code of one group; the word must start at zero. */
static void put_code(uint16_t *meta, int64_t words_per_row, int64_t row, int64_t group, unsigned code)
{
    meta[row * words_per_row + group / 4] |= (uint16_t)(code << (4 * (group % 4)));
}

int oracle_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* prune24: W [rows x K] -> vals [rows x K/2], meta [rows x K/16]. */
int oracle_prune24(const uint16_t *W, int64_t rows, int64_t K, uint16_t *vals, uint16_t *meta)
{
    if (rows < 0 || K < 0 || K % 16 != 0) return ORACLE_BAD_SHAPE;
    int status = ORACLE_OK;
    int64_t wpr = K / 16;
    memset(meta, 0, (size_t)(rows * wpr) * sizeof(uint16_t));
    for (int64_t o = 0; o < rows; ++o) {
        for (int64_t g = 0; g < K / 4; ++g) {
            const uint16_t *grp = W + o * K + 4 * g;
            for (int k = 0; k < 4; ++k)
                if (bf16_is_nonfinite(grp[k])) status = ORACLE_NONFINITE;
            int i0, i1;
            keep_two_of_four(grp, &i0, &i1);
            vals[o * (K / 2) + 2 * g] = grp[i0];
            vals[o * (K / 2) + 2 * g + 1] = grp[i1];
            put_code(meta, wpr, o, g, (unsigned)(i0 | (i1 << 2)));
        }
    }
    return status;
}

/* W^R[o][i] as a bf16 pattern, reconstructed from the compressed row o
 * (pruned positions read as +0). */
static uint16_t wr_at(const uint16_t *vals, const uint16_t *meta, int64_t K, int64_t o, int64_t i)
{
    unsigned c = code_of(meta, K / 16, o, i / 4);
    int i0 = (int)(c & 3u), i1 = (int)(c >> 2);
    int q = (int)(i % 4);
    if (q == i0) return vals[o * (K / 2) + 2 * (i / 4)];
    if (q == i1) return vals[o * (K / 2) + 2 * (i / 4) + 1];
    return 0;
}

/* Expand a compressed [rows x K] matrix to its dense bf16 patterns. */
int oracle_decompress(const uint16_t *vals, const uint16_t *meta, int64_t rows, int64_t K, uint16_t *dense)
{
    if (rows < 0 || K < 0 || K % 16 != 0) return ORACLE_BAD_SHAPE;
    for (int64_t o = 0; o < rows; ++o)
        for (int64_t i = 0; i < K; ++i) dense[o * K + i] = wr_at(vals, meta, K, o, i);
    return ORACLE_OK;
}

/*
 * double_prune: the compressed W^R [out x in] -> compressed (W^{R,C})^T
 * [in x out]: row i of the result is column i of W^R pruned 2:4 along out.
 */
int oracle_double_prune(const uint16_t *vals, const uint16_t *meta, int64_t out, int64_t in,
                        uint16_t *vals_t, uint16_t *meta_t)
{
    if (out < 0 || in < 0 || out % 16 != 0 || in % 16 != 0) return ORACLE_BAD_SHAPE;
    int64_t wpr_t = out / 16;
    memset(meta_t, 0, (size_t)(in * wpr_t) * sizeof(uint16_t));
    for (int64_t i = 0; i < in; ++i) {
        for (int64_t h = 0; h < out / 4; ++h) {
            uint16_t col[4];
            for (int j = 0; j < 4; ++j) col[j] = wr_at(vals, meta, in, 4 * h + j, i);
            int i0, i1;
            keep_two_of_four(col, &i0, &i1);
            vals_t[i * (out / 2) + 2 * h] = col[i0];
            vals_t[i * (out / 2) + 2 * h + 1] = col[i1];
            put_code(meta_t, wpr_t, i, h, (unsigned)(i0 | (i1 << 2)));
        }
    }
    return ORACLE_OK;
}

/*
 * prune_nm: W [rows x K] -> vals [rows x K*N/M] (the N kept values of every
 * group of M consecutive elements, in ascending position) and pos [same
 * shape] (each kept value's position within its group, 0 .. M-1).  Element
 * k of a group is kept iff fewer than N elements beat it (the rule of
 * keep_two_of_four with N for 2).  1 <= N < M, M in {4, 8, 16}, K % M == 0.
 */
int oracle_prune_nm(const uint16_t *W, int64_t rows, int64_t K, int N, int M, uint16_t *vals, uint8_t *pos)
{
    if (rows < 0 || K < 0 || N < 1 || N >= M || (M != 4 && M != 8 && M != 16) || K % M != 0)
        return ORACLE_BAD_SHAPE;
    int status = ORACLE_OK;
    const int64_t kept_per_row = K / M * N;
    for (int64_t o = 0; o < rows; ++o) {
        for (int64_t g = 0; g < K / M; ++g) {
            const uint16_t *grp = W + o * K + (int64_t)M * g;
            int64_t out = o * kept_per_row + (int64_t)N * g;
            for (int k = 0; k < M; ++k) {
                if (bf16_is_nonfinite(grp[k])) status = ORACLE_NONFINITE;
                int beaten_by = 0;
                for (int m = 0; m < M; ++m) {
                    if (bf16_magnitude(grp[m]) > bf16_magnitude(grp[k]) ||
                        (bf16_magnitude(grp[m]) == bf16_magnitude(grp[k]) && m < k))
                        beaten_by++;
                }
                if (beaten_by < N) {
                    vals[out] = grp[k];
                    pos[out] = (uint8_t)k;
                    ++out;
                }
            }
        }
    }
    return status;
}

/* Row selection helper: rows == NULL means "all n rows, in order". */
static int64_t pick(const int64_t *rows, int64_t idx) { return rows ? rows[idx] : idx; }

/* adapter_fwd: XL[t][j] = sum_i X[t][i] L[i][j], for the selected tokens. */
void oracle_adapter_fwd(const uint16_t *X, const uint16_t *L, int64_t T, int64_t in, int64_t r,
                        const int64_t *rows, int64_t n_rows, double *XL)
{
    (void)T;
#pragma omp parallel for schedule(dynamic)
    for (int64_t a = 0; a < n_rows; ++a) {
        int64_t t = pick(rows, a);
        for (int64_t j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t i = 0; i < in; ++i) acc += bf16_value(X[t * in + i]) * bf16_value(L[i * r + j]);
            XL[a * r + j] = acc;
        }
    }
}

/*
 * Sparse product with a compressed operand: out[t][o] = sum over the kept
 * positions k of row o of S: A[t][k] * S[o][k], plus sum_j P[t][j] Q[j][o].
 * Used for fwd (A = X, S = W^R, P = XL, Q = R) and, with S = (W^{R,C})^T,
 * for bwd_dx (A = dY, P = G, Q = L^T given as L [in x r], see below).
 */
static double sparse_row_dot(const uint16_t *a_row, const uint16_t *vals, const uint16_t *meta,
                             int64_t K, int64_t o)
{
    double acc = 0.0;
    for (int64_t g = 0; g < K / 4; ++g) {
        unsigned c = code_of(meta, K / 16, o, g);
        int i0 = (int)(c & 3u), i1 = (int)(c >> 2);
        acc += bf16_value(a_row[4 * g + i0]) * bf16_value(vals[o * (K / 2) + 2 * g]);
        acc += bf16_value(a_row[4 * g + i1]) * bf16_value(vals[o * (K / 2) + 2 * g + 1]);
    }
    return acc;
}

/* fwd: Y[t][o] = sum_{i in M_o} X[t][i] W[o][i] + sum_j XL[t][j] R[j][o]. */
void oracle_fwd(const uint16_t *X, const uint16_t *vals, const uint16_t *meta, const double *XL,
                const uint16_t *R, int64_t T, int64_t in, int64_t out, int64_t r,
                const int64_t *rows, int64_t n_rows, double *Y)
{
    (void)T;
#pragma omp parallel for schedule(dynamic)
    for (int64_t a = 0; a < n_rows; ++a) {
        int64_t t = pick(rows, a);
        for (int64_t o = 0; o < out; ++o) {
            double acc = sparse_row_dot(X + t * in, vals, meta, in, o);
            for (int64_t j = 0; j < r; ++j) acc += XL[a * r + j] * bf16_value(R[j * out + o]);
            Y[a * out + o] = acc;
        }
    }
}

/* bwd_dx: dX[t][i] = sum_o dY[t][o] W^{R,C}[o][i] + sum_j G[t][j] L[i][j];
 * W^{R,C} is given as its transpose, compressed [in x out]. */
void oracle_bwd_dx(const uint16_t *dY, const uint16_t *vals_t, const uint16_t *meta_t, const double *G,
                   const uint16_t *L, int64_t T, int64_t in, int64_t out, int64_t r,
                   const int64_t *rows, int64_t n_rows, double *dX)
{
    (void)T;
#pragma omp parallel for schedule(dynamic)
    for (int64_t a = 0; a < n_rows; ++a) {
        int64_t t = pick(rows, a);
        for (int64_t i = 0; i < in; ++i) {
            double acc = sparse_row_dot(dY + t * out, vals_t, meta_t, out, i);
            for (int64_t j = 0; j < r; ++j) acc += G[a * r + j] * bf16_value(L[i * r + j]);
            dX[a * in + i] = acc;
        }
    }
}

/* adapter_bwd, part 1: G[t][j] = sum_o dY[t][o] R[j][o]. */
void oracle_adapter_g(const uint16_t *dY, const uint16_t *R, int64_t T, int64_t out, int64_t r,
                      const int64_t *rows, int64_t n_rows, double *G)
{
    (void)T;
#pragma omp parallel for schedule(dynamic)
    for (int64_t a = 0; a < n_rows; ++a) {
        int64_t t = pick(rows, a);
        for (int64_t j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t o = 0; o < out; ++o) acc += bf16_value(dY[t * out + o]) * bf16_value(R[j * out + o]);
            G[a * r + j] = acc;
        }
    }
}

/* adapter_bwd, part 2: dR[j][o] = sum_t XL[t][j] dY[t][o], for the selected
 * columns o (output dR_sel[a][j] = dR[j][cols[a]]).  XL is [T x r]. */
void oracle_adapter_dr(const double *XL, const uint16_t *dY, int64_t T, int64_t out, int64_t r,
                       const int64_t *cols, int64_t n_cols, double *dR_sel)
{
#pragma omp parallel for schedule(dynamic)
    for (int64_t a = 0; a < n_cols; ++a) {
        int64_t o = pick(cols, a);
        for (int64_t j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t t = 0; t < T; ++t) acc += XL[t * r + j] * bf16_value(dY[t * out + o]);
            dR_sel[a * r + j] = acc;
        }
    }
}

/* adapter_bwd, part 3: dL[i][j] = sum_t X[t][i] G[t][j], for the selected
 * rows i.  G is [T x r]. */
void oracle_adapter_dl(const uint16_t *X, const double *G, int64_t T, int64_t in, int64_t r,
                       const int64_t *rows, int64_t n_rows, double *dL_sel)
{
#pragma omp parallel for schedule(dynamic)
    for (int64_t a = 0; a < n_rows; ++a) {
        int64_t i = pick(rows, a);
        for (int64_t j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t t = 0; t < T; ++t) acc += bf16_value(X[t * in + i]) * G[t * r + j];
            dL_sel[a * r + j] = acc;
        }
    }
}

/*
 * bwd_dw_masked: for each selected out row o and each kept slot (group g,
 * position i_s), dW[o][2g+s] = sum_t dY[t][o] X[t][4g+i_s].  The sum runs
 * over t in ascending order for every output (the loop over t is outermost
 * only so that rows of X are read in order).
 */
void oracle_bwd_dw_masked(const uint16_t *dY, const uint16_t *X, const uint16_t *meta, int64_t T,
                          int64_t in, int64_t out, const int64_t *rows, int64_t n_rows, double *dW)
{
#pragma omp parallel for schedule(dynamic)
    for (int64_t a = 0; a < n_rows; ++a) {
        int64_t o = pick(rows, a);
        double *acc = dW + a * (in / 2);
        for (int64_t s = 0; s < in / 2; ++s) acc[s] = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            double d = bf16_value(dY[t * out + o]);
            const uint16_t *xr = X + t * in;
            for (int64_t g = 0; g < in / 4; ++g) {
                unsigned c = code_of(meta, in / 16, o, g);
                acc[2 * g] += d * bf16_value(xr[4 * g + (int)(c & 3u)]);
                acc[2 * g + 1] += d * bf16_value(xr[4 * g + (int)(c >> 2)]);
            }
        }
    }
}

/* binary32 value -> bf16 pattern, round to nearest, ties to even (finite values). */
static uint16_t bf16_round(float x)
{
    uint32_t b;
    memcpy(&b, &x, sizeof b);
    b += 0x7FFFu + ((b >> 16) & 1u);
    return (uint16_t)(b >> 16);
}

static float bf16_float(uint16_t bits)
{
    uint32_t b = (uint32_t)bits << 16;
    float x;
    memcpy(&x, &b, sizeof x);
    return x;
}

/*
 * adamw_compressed: one AdamW step (step number `step` >= 1) on n kept
 * values: vals (bf16 patterns) and their fp32 states m, v are updated in
 * place from the compressed gradient grad (bf16 patterns, same slots).
 * Each operation below is one binary32 operation (no fused multiply-add):
 *     w  <- w * (1 - lr * wd)
 *     m  <- b1 * m + (1 - b1) * g
 *     v  <- b2 * v + (1 - b2) * (g * g)
 *     w  <- w - step_size * (m / (sqrt(v) * inv_sqrt_bc2 + eps))
 * with step_size = lr / (1 - b1^step) and inv_sqrt_bc2 = 1 / sqrt(1 - b2^step)
 * evaluated in binary64 and rounded to binary32; w is then rounded to bf16.
 */
void oracle_adamw_compressed(uint16_t *vals, const uint16_t *grad, float *m, float *v, int64_t n, float lr,
                             float b1, float b2, float eps, float wd, int64_t step)
{
    const float step_size = (float)((double)lr / (1.0 - pow((double)b1, (double)step)));
    const float inv_sqrt_bc2 = (float)(1.0 / sqrt(1.0 - pow((double)b2, (double)step)));
    const float decay = 1.0f - lr * wd;
    const float omb1 = 1.0f - b1, omb2 = 1.0f - b2;
    for (int64_t k = 0; k < n; ++k) {
        const float g = bf16_float(grad[k]);
        float w = bf16_float(vals[k]) * decay;
        const float mk = b1 * m[k] + omb1 * g;
        const float gg = g * g;
        const float vk = b2 * v[k] + omb2 * gg;
        const float denom = sqrtf(vk) * inv_sqrt_bc2 + eps;
        const float q = mk / denom;
        w = w - step_size * q;
        m[k] = mk;
        v[k] = vk;
        vals[k] = bf16_round(w);
    }
}

/*
 * Memory per four consecutive weights, as a fraction of the dense layout
 * (rebuttal section "Memory Footprint Reduction During Pretraining and
 * Inference").  Inference: (N*b_val + b_idx) / (M*b_val).  Training adds the
 * transposed copy, a per-element binary mask of b_mask bits, the gradient of
 * the non-zeros and n_states optimizer states for the non-zeros, against a
 * dense weight, a dense gradient and n_states dense states.
 * Returns the two ratios through out[0] (inference) and out[1] (training).
 */
void oracle_mem_ratio(int n_keep, int m_group, int b_val, int b_idx, int b_mask, int b_grad,
                      int b_state, int n_states, double out[2])
{
    double sparse_w = (double)(n_keep * b_val + b_idx);
    double dense_w = (double)(m_group * b_val);
    out[0] = sparse_w / dense_w;
    double sparse_train = sparse_w                       /* weight             */
                          + sparse_w                     /* weight transpose   */
                          + (double)(m_group * b_mask)   /* binary mask        */
                          + (double)(n_keep * b_grad)    /* gradient           */
                          + (double)(n_states * n_keep * b_state); /* optimizer states */
    double dense_train = dense_w + (double)(m_group * b_grad) + (double)(n_states * m_group * b_state);
    out[1] = sparse_train / dense_train;
}
