/*
 * oracle.c -- plain fp64 CPU oracle for the batch-invariant reduction kernels.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library
 * libbi.so and its Python binding) may include, link, load or call this file.
 * Only the test-suite, the smoke check and the CPU-baseline leg of the
 * benchmark use it.  It shares no code, header, table or helper with the CUDA
 * path: it is written from the definitions of the operations, not from the
 * kernels.
 *
 * What it computes.  The pages on batch-invariant inference define the
 * property, not new arithmetic: a kernel is batch-invariant when the numbers it
 * returns for one row ("a given sequence") do not depend on how many rows share
 * the batch, which it obtains by always reducing in the same order
 *   - readhandoff.com "Agent run reproducibility pinning", section
 *     "What does temperature zero actually guarantee?" (matmul, RMSNorm,
 *     attention are "not batch-invariant"; the reduction tree changes with
 *     batch size);
 *   - wiki.aimuse.me "Thinking Machines", section on the batch-invariant
 *     kernel claim (same input, same accumulation order);
 *   - glasp.co "How to achieve deterministic LLMs with batch invariant
 *     inference", Key Insights (reduction order fixed across batches).
 * The operations themselves are the ordinary PyTorch ones the library replaces
 * (ross.abutalabs.com "thinking-machines-lab/batch_invariant_ops", sections
 * "What it is" and "When to avoid": mm, addmm, log_softmax, mean), plus RMSNorm
 * (readhandoff.com page, same section) and the SiLU-times-up glue of a
 * gated MLP.  So the oracle is each operation's plain mathematical definition
 * evaluated in IEEE binary64 with sequential loops in index order: any fixed
 * order a GPU kernel uses agrees with it up to rounding.
 *
 * Inputs.  bf16 tensors arrive as their raw 16-bit patterns; a bf16 value is by
 * definition the binary32 number whose upper 16 bits are that pattern and whose
 * lower 16 bits are zero, so the widening below is exact.  fp32 tensors arrive
 * as float.  All results are written as double.
 *
 * Threads.  `nthreads` only splits independent output elements (rows, or
 * (row, column) pairs of a matmul) across OpenMP threads; the arithmetic for
 * each output element is the same sequential loop whatever the thread count.
 *
 * Every function returns 0 on success and -1 on an invalid argument (negative
 * size, leading dimension smaller than the row length, null pointer with a
 * non-zero size).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 bit pattern -> exact double (definition of the bfloat16 format). */
static double bf16_to_double(uint16_t bits)
{
    uint32_t word = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &word, sizeof f);
    return (double)f;
}

static int threads_or_one(int nthreads) { return nthreads > 0 ? nthreads : 1; }

/*
 * Element (k, j) of the right-hand matrix B of C = A.B.
 *   layout 0: B is stored [K, N] row-major (torch.mm operand), leading dim ldb
 *   layout 1: B is stored [N, K] row-major (nn.Linear weight), leading dim ldb
 */
static double b_elem(const uint16_t *B, int64_t ldb, int layout, int64_t k, int64_t j)
{
    return layout == 0 ? bf16_to_double(B[k * ldb + j]) : bf16_to_double(B[j * ldb + k]);
}

static int check_matmul_args(const void *A, int64_t lda, const void *B, int64_t ldb, int layout,
                             const void *C, int64_t ldc, int64_t M, int64_t N, int64_t K)
{
    if (M < 0 || N < 0 || K < 0) return -1;
    if (layout != 0 && layout != 1) return -1;
    if (M > 0 && N > 0 && C == 0) return -1;
    if (M > 0 && K > 0 && (A == 0 || lda < K)) return -1;
    if (N > 0 && K > 0 && B == 0) return -1;
    if (N > 0 && K > 0 && ldb < (layout == 0 ? N : K)) return -1;
    if (M > 0 && ldc < N) return -1;
    return 0;
}

/*
 * mm: C[i][j] = sum_{k=0}^{K-1} A[i][k] * B[k][j], k ascending, in binary64.
 * A is [M, K] bf16 row-major (leading dim lda); C is [M, N] (leading dim ldc).
 * The product of two bf16 numbers is exact in binary64, so the only rounding
 * is in the running sum.  K = 0 gives C = 0.
 */
int oracle_matmul(const uint16_t *A, int64_t lda, const uint16_t *B, int64_t ldb, int b_layout,
                  double *C, int64_t ldc, int64_t M, int64_t N, int64_t K, int nthreads)
{
    if (check_matmul_args(A, lda, B, ldb, b_layout, C, ldc, M, N, K)) return -1;
    int64_t total = M * N;
#pragma omp parallel for num_threads(threads_or_one(nthreads)) schedule(static)
    for (int64_t e = 0; e < total; ++e) {
        int64_t i = e / N, j = e % N;
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k)
            acc += bf16_to_double(A[i * lda + k]) * b_elem(B, ldb, b_layout, k, j);
        C[i * ldc + j] = acc;
    }
    return 0;
}

/*
 * addmm with alpha = beta = 1: C = input + A.B (torch.addmm).
 * `input` is bf16; ld_input == 0 means a bias vector [N] broadcast over rows,
 * otherwise a full [M, N] matrix (e.g. a residual) with leading dim ld_input.
 * The matrix product is the sum of mm above; the input is added once, after.
 */
int oracle_addmm(const uint16_t *input, int64_t ld_input, const uint16_t *A, int64_t lda,
                 const uint16_t *B, int64_t ldb, int b_layout, double *C, int64_t ldc,
                 int64_t M, int64_t N, int64_t K, int nthreads)
{
    if (check_matmul_args(A, lda, B, ldb, b_layout, C, ldc, M, N, K)) return -1;
    if (M > 0 && N > 0 && input == 0) return -1;
    if (ld_input != 0 && ld_input < N) return -1;
    if (ld_input < 0) return -1;
    int64_t total = M * N;
#pragma omp parallel for num_threads(threads_or_one(nthreads)) schedule(static)
    for (int64_t e = 0; e < total; ++e) {
        int64_t i = e / N, j = e % N;
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k)
            acc += bf16_to_double(A[i * lda + k]) * b_elem(B, ldb, b_layout, k, j);
        double add = ld_input == 0 ? bf16_to_double(input[j]) : bf16_to_double(input[i * ld_input + j]);
        C[i * ldc + j] = acc + add;
    }
    return 0;
}

/*
 * RMSNorm over the last dimension H of x [M, H] (bf16) with weight w [H] (bf16):
 *   r    = 1 / sqrt( (sum_j x_j^2) / H + eps )
 *   y_j  = x_j * r * w_j
 * eps sits inside the square root; the weight multiplies the normalised value.
 */
int oracle_rmsnorm(const uint16_t *x, const uint16_t *w, double *y, int64_t M, int64_t H,
                   double eps, int nthreads)
{
    if (M < 0 || H <= 0) return (M == 0 && H >= 0) ? 0 : -1;
    if (M > 0 && (x == 0 || w == 0 || y == 0)) return -1;
#pragma omp parallel for num_threads(threads_or_one(nthreads)) schedule(static)
    for (int64_t i = 0; i < M; ++i) {
        const uint16_t *row = x + i * H;
        double ss = 0.0;
        for (int64_t j = 0; j < H; ++j) {
            double v = bf16_to_double(row[j]);
            ss += v * v;
        }
        double r = 1.0 / sqrt(ss / (double)H + eps);
        for (int64_t j = 0; j < H; ++j)
            y[i * H + j] = bf16_to_double(row[j]) * r * bf16_to_double(w[j]);
    }
    return 0;
}

/* mean over the last dimension of x [M, H] (fp32): y_i = (sum_j x_ij) / H. */
int oracle_mean_f32(const float *x, double *y, int64_t M, int64_t H, int nthreads)
{
    if (M < 0 || H <= 0) return (M == 0 && H >= 0) ? 0 : -1;
    if (M > 0 && (x == 0 || y == 0)) return -1;
#pragma omp parallel for num_threads(threads_or_one(nthreads)) schedule(static)
    for (int64_t i = 0; i < M; ++i) {
        double s = 0.0;
        for (int64_t j = 0; j < H; ++j) s += (double)x[i * H + j];
        y[i] = s / (double)H;
    }
    return 0;
}

/*
 * log_softmax over the last dimension V of one row held as doubles:
 *   m   = max_j x_j
 *   s   = sum_j exp(x_j - m)
 *   y_j = (x_j - m) - log(s)
 * Subtracting the maximum first is the usual overflow-safe form; it does not
 * change the mathematical value.
 */
static void log_softmax_row(const double *xr, double *yr, int64_t V)
{
    double m = -INFINITY;
    for (int64_t j = 0; j < V; ++j)
        if (xr[j] > m) m = xr[j];
    double s = 0.0;
    for (int64_t j = 0; j < V; ++j) s += exp(xr[j] - m);
    double ls = log(s);
    for (int64_t j = 0; j < V; ++j) yr[j] = (xr[j] - m) - ls;
}

/* log_softmax of x [M, V] given as fp32.  Each row is widened into its slot of y
 * and transformed there in place. */
int oracle_log_softmax_f32(const float *x, double *y, int64_t M, int64_t V, int nthreads)
{
    if (M < 0 || V <= 0) return (M == 0 && V >= 0) ? 0 : -1;
    if (M > 0 && (x == 0 || y == 0)) return -1;
#pragma omp parallel for num_threads(threads_or_one(nthreads)) schedule(static)
    for (int64_t i = 0; i < M; ++i) {
        double *yr = y + i * V;
        for (int64_t j = 0; j < V; ++j) yr[j] = (double)x[i * V + j];
        log_softmax_row(yr, yr, V);
    }
    return 0;
}

/* log_softmax of x [M, V] given as bf16 bit patterns (e.g. logits of an LM head). */
int oracle_log_softmax_bf16(const uint16_t *x, double *y, int64_t M, int64_t V, int nthreads)
{
    if (M < 0 || V <= 0) return (M == 0 && V >= 0) ? 0 : -1;
    if (M > 0 && (x == 0 || y == 0)) return -1;
#pragma omp parallel for num_threads(threads_or_one(nthreads)) schedule(static)
    for (int64_t i = 0; i < M; ++i) {
        double *yr = y + i * V;
        for (int64_t j = 0; j < V; ++j) yr[j] = bf16_to_double(x[i * V + j]);
        log_softmax_row(yr, yr, V);
    }
    return 0;
}

/*
 * Gated-MLP glue: gu is [M, 2F] bf16 with the gate in columns [0, F) and the
 * up projection in columns [F, 2F).  h_ij = silu(g_ij) * u_ij with
 * silu(g) = g / (1 + exp(-g)).
 */
int oracle_silu_mul(const uint16_t *gu, double *h, int64_t M, int64_t F, int nthreads)
{
    if (M < 0 || F <= 0) return (M == 0 && F >= 0) ? 0 : -1;
    if (M > 0 && (gu == 0 || h == 0)) return -1;
#pragma omp parallel for num_threads(threads_or_one(nthreads)) schedule(static)
    for (int64_t i = 0; i < M; ++i) {
        for (int64_t j = 0; j < F; ++j) {
            double g = bf16_to_double(gu[i * 2 * F + j]);
            double u = bf16_to_double(gu[i * 2 * F + F + j]);
            h[i * F + j] = g / (1.0 + exp(-g)) * u;
        }
    }
    return 0;
}

/*
 * The same gated-MLP glue on binary64 inputs: gu is [M, 2F] double (gate columns [0, F),
 * up columns [F, 2F)), as produced by oracle_matmul without an intermediate rounding.
 */
int oracle_silu_mul_f64(const double *gu, double *h, int64_t M, int64_t F, int nthreads)
{
    if (M < 0 || F <= 0) return (M == 0 && F >= 0) ? 0 : -1;
    if (M > 0 && (gu == 0 || h == 0)) return -1;
#pragma omp parallel for num_threads(threads_or_one(nthreads)) schedule(static)
    for (int64_t i = 0; i < M; ++i) {
        for (int64_t j = 0; j < F; ++j) {
            double g = gu[i * 2 * F + j];
            double u = gu[i * 2 * F + F + j];
            h[i * F + j] = g / (1.0 + exp(-g)) * u;
        }
    }
    return 0;
}

/*
 * Decode attention (one query token per sequence), grouped-query heads.
 *   q  [B, Hq, D]          bf16
 *   k  [B, Lmax, Hkv, D]   bf16 (key cache), v likewise (value cache)
 *   lens[b] in 1 .. Lmax   tokens of sequence b
 * Query head h reads kv head h / (Hq / Hkv).  For each (b, h):
 *   s_t = scale * sum_d q[d] * k[t][d]             t < lens[b]
 *   p_t = exp(s_t - max_t s_t)
 *   o_d = (sum_t p_t * v[t][d]) / (sum_t p_t)
 * (softmax attention; subtracting the maximum does not change the value).
 * o is [B, Hq, D] double.
 */
int oracle_decode_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v, const int32_t *lens,
                            double *o, int64_t B, int64_t Hq, int64_t Hkv, int64_t D, int64_t Lmax,
                            double scale, int nthreads)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Lmax <= 0 || Hq % Hkv) return B == 0 ? 0 : -1;
    if (B > 0 && (!q || !k || !v || !lens || !o)) return -1;
    for (int64_t b = 0; b < B; ++b)
        if (lens[b] < 1 || lens[b] > Lmax) return -1;
    const int64_t group = Hq / Hkv;
#pragma omp parallel for num_threads(threads_or_one(nthreads)) schedule(dynamic)
    for (int64_t bh = 0; bh < B * Hq; ++bh) {
        const int64_t b = bh / Hq, h = bh % Hq, g = h / group;
        const int64_t L = lens[b];
        const uint16_t *qv = q + (b * Hq + h) * D;
        double m = -INFINITY;
        for (int64_t t = 0; t < L; ++t) {
            const uint16_t *kt = k + ((b * Lmax + t) * Hkv + g) * D;
            double sdot = 0.0;
            for (int64_t d = 0; d < D; ++d) sdot += bf16_to_double(qv[d]) * bf16_to_double(kt[d]);
            const double st = scale * sdot;
            if (st > m) m = st;
        }
        double l = 0.0;
        double *ov = o + (b * Hq + h) * D;
        for (int64_t d = 0; d < D; ++d) ov[d] = 0.0;
        for (int64_t t = 0; t < L; ++t) {
            const uint16_t *kt = k + ((b * Lmax + t) * Hkv + g) * D;
            const uint16_t *vt = v + ((b * Lmax + t) * Hkv + g) * D;
            double sdot = 0.0;
            for (int64_t d = 0; d < D; ++d) sdot += bf16_to_double(qv[d]) * bf16_to_double(kt[d]);
            const double pt = exp(scale * sdot - m);
            l += pt;
            for (int64_t d = 0; d < D; ++d) ov[d] += pt * bf16_to_double(vt[d]);
        }
        for (int64_t d = 0; d < D; ++d) ov[d] /= l;
    }
    return 0;
}

/* Number of OpenMP threads the runtime would use by default (1 without OpenMP). */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
