/*
 * bi.h -- C ABI of libbi.so: batch-invariant reduction kernels for NVIDIA B200 (sm_100a).
 *
 * A kernel is batch-invariant when the bits it returns for one row of its input
 * do not depend on how many other rows share the call or where the row sits in
 * the batch.  The source pages state the property and its cause: inference
 * kernels such as matmul and RMSNorm reduce in an order shaped by the total
 * batch size, so a row's last bits change with the batch (readhandoff.com,
 * agent-run-reproducibility-pinning, "What does temperature zero actually
 * guarantee?"); the remedy is that the same input always takes the same
 * accumulation order (wiki.aimuse.me "Thinking Machines", batch-invariant
 * kernel section; glasp.co "How to achieve deterministic LLMs with batch
 * invariant inference", Key Insights), which rules out split-K and
 * shape-aware tiling (wiki.aimuse.me "Thinking Machines", section on the loss
 * of dynamic-batching optimisations).  The operations are those the public
 * library replaces -- mm, addmm, log_softmax, mean (ross.abutalabs.com
 * "thinking-machines-lab/batch_invariant_ops", "When to avoid") -- plus RMSNorm
 * and the SiLU-times-up glue of a gated MLP.
 *
 * How each entry point fixes its order (the same for every M):
 *   - bi_matmul / bi_addmm: tcgen05/TMEM tiles fed by TMA; the tile width is a
 *     function of the weight's shape alone (bi_gemm_config), never of M; every
 *     output element accumulates its K products in fp32, 16 at a time, in
 *     ascending K, in every configuration; no split-K, no stream-K.
 *   - bi_rmsnorm / bi_mean / bi_log_softmax: each row is reduced by one thread
 *     block (for long-row means, persistent blocks take rows in turn); the
 *     block size and each thread's element set depend only on the row length;
 *     partial results merge through a fixed warp-shuffle tree and a fixed
 *     cross-warp tree.
 *
 * Conventions shared by every entry point
 *   - Tensors are row-major.  Pointers marked "device" point to global memory
 *     of the current CUDA device; the caller allocates, owns and frees every
 *     buffer.  The library allocates no device memory in any call.
 *   - `stream` is a cudaStream_t passed as `void *` (so that this header needs no CUDA
 *     header; NULL = the legacy default stream).  Calls are
 *     asynchronous on that stream.  Argument errors are returned before anything
 *     is launched; a launch failure returns BI_ERR_CUDA.  The status is the result of this
 *     call's own launches: an error left by another library's earlier launch on the thread
 *     is neither reported nor cleared (apart from a context-wide fault, which fails every
 *     launch).  The GEMM, RMSNorm, mean,
 *     one-block log_softmax and decode-attention kernels are launched with programmatic
 *     stream serialization:
 *     they may start their on-chip set-up while the previous kernel on the stream drains,
 *     and read or write global memory only after that kernel has completed, so stream
 *     order holds as for any launch.
 *   - M = 0 (no rows) is a no-op that returns BI_OK.
 *   - Outputs must not overlap inputs.
 *   - bf16 is IEEE-style bfloat16 (1-8-7); every bf16 output is rounded once,
 *     to nearest-even, from an fp32 value.
 *   - The library keeps per-device state for the life of the process (the SM count, the
 *     status word's address, kernel attributes, the no-allocation array's address) and a
 *     cache of encoded TMA tensor maps keyed by (base address, extents, row stride, box).
 *     Calls across a cudaDeviceReset of a device the library has already used are not
 *     supported: the cached device addresses belong to the context that reset destroyed.
 *   - Every device-side wait is bounded; a wait that runs out records
 *     BI_ERR_TIMEOUT in a per-device status word, the kernel releases what it
 *     holds and returns.  Read it with bi_get_device_status.
 */
#ifndef BI_H
#define BI_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BI_OK = 0,
    BI_ERR_INVALID_ARG = 1,  /* null pointer, negative size, leading dim too small, bad enum */
    BI_ERR_UNSUPPORTED = 2,  /* a size the kernels do not handle (e.g. > 2^31-1 rows)        */
    BI_ERR_ALIGNMENT = 3,    /* base pointer or leading dimension breaks the 16-byte rule   */
    BI_ERR_CUDA = 4,         /* a CUDA runtime/driver call or a launch failed                */
    BI_ERR_TIMEOUT = 5       /* a bounded device-side wait ran out (reported via the status) */
} bi_status;

typedef enum { BI_BF16 = 0, BI_F32 = 1 } bi_dtype;

typedef enum {
    BI_B_KN = 0, /* B stored [K, N] row-major: the right operand of torch.mm           */
    BI_B_NK = 1  /* B stored [N, K] row-major: an nn.Linear weight (C = A . B^T)       */
} bi_b_layout;

/*
 * bi_matmul -- C = A . B  (torch.mm; for BI_B_NK, torch.nn.functional.linear without bias).
 * Passage: ross.abutalabs.com "thinking-machines-lab/batch_invariant_ops", "When to
 * avoid" (mm is covered) and "Use cases" (matrix multiplication gives the same output
 * for different batch sizes).
 *
 *   A  device, bf16, [M, K], leading dimension lda >= K (elements)
 *   B  device, bf16, [K, N] with ldb >= N (BI_B_KN) or [N, K] with ldb >= K (BI_B_NK)
 *   C  device, [M, N], leading dimension ldc >= N, element type c_dtype (BI_BF16 or BI_F32)
 *   C[i][j] = round_{c_dtype}( sum_{k ascending} A[i][k] * B(k, j) ), products and sums in fp32.
 *   K = 0 writes zeros.
 * Alignment: A, B, C base addresses 16-byte aligned; lda, ldb multiples of 8 elements;
 *   ldc a multiple of 8 (bf16) or 4 (f32) elements.  Otherwise BI_ERR_ALIGNMENT.
 * Limits: M, N, K <= 2^31 - 1; otherwise BI_ERR_UNSUPPORTED.
 */
bi_status bi_matmul(const void *A, int64_t lda, const void *B, int64_t ldb, bi_b_layout b_layout,
                    void *C, int64_t ldc, bi_dtype c_dtype, int64_t M, int64_t N, int64_t K,
                    void *stream);

/*
 * bi_addmm -- C = input + A . B  (torch.addmm with alpha = beta = 1).
 * Passage: ross.abutalabs.com "thinking-machines-lab/batch_invariant_ops", "When to
 * avoid" (addmm is covered).
 *
 *   input  device, bf16.  ld_input == 0: a bias vector [N] added to every row.
 *          ld_input >= N: a matrix [M, N] (e.g. a residual) with that leading dimension,
 *          which must be a multiple of 8; base 16-byte aligned.
 *   The input is widened to fp32 and added to the fp32 accumulator once, after the last
 *   product, before the single rounding to c_dtype.  All else as bi_matmul.
 */
bi_status bi_addmm(const void *input, int64_t ld_input, const void *A, int64_t lda, const void *B,
                   int64_t ldb, bi_b_layout b_layout, void *C, int64_t ldc, bi_dtype c_dtype,
                   int64_t M, int64_t N, int64_t K, void *stream);

/*
 * bi_matmul_silu_mul -- H = silu(A . Wg) * (A . Wu): the gate/up projection of a gated MLP
 * with the SiLU-times-up glue applied in the GEMM's epilogue, so the [M, 2F] gate/up
 * activations never reach memory.  Elementwise glue after the same batch-invariant
 * reduction as bi_matmul; not an operation the pages name (the MLP block of the workload).
 *
 *   A  device, bf16, [M, K], lda >= K.
 *   B  device, bf16, the gate and up weights stacked: BI_B_NK: [2F, K] with rows [0, F) the
 *      gate and rows [F, 2F) the up projection (ldb >= K); BI_B_KN: [K, 2F] with columns
 *      [0, F) gate and [F, 2F) up (ldb >= 2F).
 *   H  device, bf16, [M, F], ldh >= F.
 *   g and u are the fp32 accumulators of bi_matmul (same K order); h = (g / (1 + exp(-g))) * u
 *   in fp32, one rounding to bf16.  (bi_matmul followed by bi_silu_mul rounds g and u to bf16
 *   first, so the two paths agree to the bf16 tolerance, not bit for bit.)
 *   Alignment and limits as bi_matmul; 2F <= 2^31 - 1; with BI_B_KN, F must also be a multiple
 *   of 8 (the up half starts at column F), else BI_ERR_ALIGNMENT.  K = 0 writes zeros.
 */
bi_status bi_matmul_silu_mul(const void *A, int64_t lda, const void *B, int64_t ldb,
                             bi_b_layout b_layout, void *H, int64_t ldh, int64_t M, int64_t F,
                             int64_t K, void *stream);

/*
 * bi_rmsnorm -- y = x * r * w,  r = 1 / sqrt( sum_j x_j^2 / H + eps ), per row.
 * Passage: readhandoff.com agent-run-reproducibility-pinning, "What does temperature
 * zero actually guarantee?" and the FAQ (RMSNorm is one of the kernels whose result
 * depends on the batch by default).
 *
 *   x  device, bf16, [M, H] contiguous;  w device, bf16, [H];  y device, bf16, [M, H].
 *   fp32 arithmetic inside; one rounding of (x * r) * w to bf16.  eps >= 0.
 *   x, w, y 16-byte aligned when H is a multiple of 8 (the vector path), else any alignment.
 */
bi_status bi_rmsnorm(const void *x, const void *w, void *y, int64_t M, int64_t H, float eps,
                     void *stream);

/*
 * bi_mean -- y_i = ( sum_j x_ij ) / H, per row (torch.mean over the last dimension).
 * Passage: ross.abutalabs.com "thinking-machines-lab/batch_invariant_ops", "When to
 * avoid" (mean is covered); trustbutveri.fyi "Evidence & limits", Evidence (SGLang
 * integrated the mean kernel).
 *
 *   x  device, fp32, [M, H] contiguous;  y device, fp32, [M].
 *   fp32 sum in a fixed tree, then one IEEE division by H.
 *   x 16-byte aligned when H is a multiple of 4 (the vector path).
 */
bi_status bi_mean(const float *x, float *y, int64_t M, int64_t H, void *stream);

/*
 * bi_log_softmax -- y_j = (x_j - m) - log( sum_k exp(x_k - m) ),  m = max_k x_k, per row.
 * Passage: ross.abutalabs.com "thinking-machines-lab/batch_invariant_ops", "When to
 * avoid" (log_softmax is covered); trustbutveri.fyi "Evidence & limits", Evidence.
 *
 *   x  device, [M, V] contiguous, x_dtype BI_F32 or BI_BF16 (bf16 is widened exactly);
 *   y  device, fp32, [M, V].
 *   One thread block per row.  Per-thread running (max, sum) pairs merged through a fixed
 *   tree; the row is read twice (once for the statistics, once to write y; the last chunks of
 *   the first pass are still in shared memory for the second).
 *   x and y 16-byte aligned when V is a multiple of 8 (bf16) / 4 (f32), the vector path.
 */
bi_status bi_log_softmax(const void *x, bi_dtype x_dtype, float *y, int64_t M, int64_t V,
                         void *stream);

/*
 * bi_log_softmax_cluster -- the same y as bi_log_softmax, for long rows, computed by a cluster of
 * 4 CTAs per row (an opt-in variant: bi_log_softmax keeps one CTA per row).  Passage: as
 * bi_log_softmax.  The row is cut into 4 slices of S = 8 * ceil(V / 32) elements, a cut fixed by V
 * alone; each CTA bulk-copies its slice into shared memory, reduces it to a (max, sum of exp)
 * pair, and every CTA folds the 4 pairs in rank order (distributed shared memory) before
 * writing its slice of y from shared memory, so the row is read from memory once.  The result
 * is batch-invariant; it is a different fixed order from bi_log_softmax's, so the two agree to
 * the tolerance, not bit for bit.
 *
 *   x, x_dtype, y, M, V as bi_log_softmax; x and y 16-byte aligned.
 *   Rows it takes: V % 8 == 0 (bf16) or V % 4 == 0 (fp32), V * element size >= 64 KiB and
 *   S * element size <= 96 KiB, i.e. 32768 <= V <= 196608 for bf16 and 16384 <= V <= 98304 for
 *   fp32.  Any other V returns BI_ERR_UNSUPPORTED without launching.
 */
bi_status bi_log_softmax_cluster(const void *x, bi_dtype x_dtype, float *y, int64_t M, int64_t V,
                                 void *stream);

/*
 * bi_log_softmax_split -- the same y as bi_log_softmax, computed by many blocks per row, for
 * short batches (decode-time sampling) where one block per row leaves most SMs idle.
 * Passage: as bi_log_softmax.  The row is cut into chunks of 4096 elements, a cut fixed by V
 * alone; each chunk is reduced to a (max, sum of exp) partial, and every block of the row
 * merges the row's partials in one fixed tree before writing its chunk.  The result is
 * batch-invariant; it is a different fixed order from bi_log_softmax's, so the two agree to
 * the tolerance, not bit for bit.
 *
 *   x, x_dtype, y, M, V as bi_log_softmax; V must be a multiple of 8 (else
 *   BI_ERR_UNSUPPORTED), x and y 16-byte aligned; M <= 65535.
 *   scratch  device memory owned by the caller, 16-byte aligned, at least
 *            bi_log_softmax_split_scratch_bytes(M, V) bytes; overwritten by the call (two
 *            launches on `stream`), so calls that overlap on the GPU need separate scratch.
 *   Too small a scratch returns BI_ERR_INVALID_ARG.
 */
bi_status bi_log_softmax_split(const void *x, bi_dtype x_dtype, float *y, int64_t M, int64_t V,
                               void *scratch, size_t scratch_bytes, void *stream);

/* Bytes of scratch bi_log_softmax_split needs for M rows of V elements (0 if M or V <= 0). */
size_t bi_log_softmax_split_scratch_bytes(int64_t M, int64_t V);

/*
 * bi_log_softmax_split_noalloc -- bi_log_softmax_split for callers that cannot allocate
 * device memory at call time: ones working inside a device-memory budget reserved up front
 * by a pool they do not own, plugins whose host framework controls every allocation, or hot
 * paths that cannot afford the synchronisation a cudaMalloc implies.  The paper has no
 * counterpart; this is a library convenience.
 *
 * The per-(row, chunk) partials live in a fixed array inside libbi.so's device image (512 KiB,
 * 65536 partials) instead of caller scratch.  Every GPU that loads the library holds that
 * array until the process exits; no call allocates or frees anything.
 *
 *   x, x_dtype, y, M, V as bi_log_softmax_split (V a multiple of 8, 16-byte aligned x and y,
 *   M <= 65535).  Limit: M * ceil(V / 4096) <= 65536 (e.g. M <= 1724 rows at V = 151936);
 *   larger calls return BI_ERR_UNSUPPORTED without launching.
 *   The result is the same as bi_log_softmax_split's for the same input.
 *   The first call on a device looks up the array's device address (once per device, with
 *   that device current); make that first call before capturing any stream.
 *   All calls on a device share the one array, and it keeps the last call's partials (every
 *   call overwrites all the partials it reads, so nothing has to start at zero).  Calls that
 *   overlap on the GPU -- on different streams without ordering between them -- race on it.
 */
bi_status bi_log_softmax_split_noalloc(const void *x, bi_dtype x_dtype, float *y, int64_t M,
                                       int64_t V, void *stream);

/*
 * bi_silu_mul -- h_ij = silu(g_ij) * u_ij with g = gu[:, 0:F], u = gu[:, F:2F],
 * silu(g) = g / (1 + exp(-g)).  Elementwise glue of a gated MLP (no reduction, so
 * batch-invariant by construction); not an operation the pages name.
 *
 *   gu device, bf16, [M, 2F] contiguous;  h device, bf16, [M, F].
 *   fp32 inside, one rounding to bf16.  16-byte aligned when F is a multiple of 8.
 */
bi_status bi_silu_mul(const void *gu, void *h, int64_t M, int64_t F, void *stream);

/*
 * bi_decode_attention -- one decode step of softmax attention with grouped-query heads:
 * for each sequence b and query head h (reading kv head h / (Hq / Hkv)),
 *   s_t = scale * q[b,h,:] . k[b,t,g,:],  p = softmax over t < seq_lens[b],  out[b,h,:] = sum_t p_t v[b,t,g,:].
 * Passage: trustbutveri.fyi "Evidence & limits", Evidence and Limitations (SGLang wrote
 * batch-invariant attention kernels; an improved attention kernel took the deterministic
 * Qwen3-8B run from 55 s to 42 s); readhandoff.com agent-run-reproducibility-pinning,
 * "What does temperature zero actually guarantee?" (attention is not batch-invariant by
 * default).
 *
 * Batch invariance: each sequence's cache is cut into splits of 512 tokens, a cut fixed by
 * its own length (never by the batch size or the GPU's occupancy, unlike split-KV decoding
 * that sizes splits to fill the machine).  Per split, scores are fp32 dot products over D in
 * ascending order; the split is taken in four 128-token pieces in ascending order, each
 * raising a running maximum by a fixed tree and rescaling the sums of exp(s - max) and the
 * weighted value sums accumulated so far, which run over tokens in ascending order; the
 * splits are then folded in ascending order.  A sequence's output does not depend on the
 * other sequences in the batch.
 *
 *   q        device, bf16, [B, Hq, D];  out device, bf16, [B, Hq, D] (one rounding).
 *   k_cache, v_cache  device, bf16, [B, Lmax, Hkv, D]; only the first seq_lens[b] tokens of
 *            sequence b are read.
 *   seq_lens device, int32, [B], each in 1 .. Lmax.  A value outside is clamped and
 *            BI_ERR_INVALID_ARG is recorded in the device status word.
 *   D must be 64 or 128 and Hq / Hkv one of 1, 2, 4, 8 (else BI_ERR_UNSUPPORTED); B, Hq, Hkv <= 65535
 *   and B * Hkv * ceil(Lmax / 512) < 2^31 (else BI_ERR_UNSUPPORTED).
 *   scratch  caller-owned device memory, 16-byte aligned, at least
 *            bi_decode_attention_scratch_bytes(B, Hq, D, Lmax) bytes; overwritten (two
 *            launches on `stream`; one when Lmax <= 512, where every sequence is one split
 *            and the first launch writes out itself), so overlapping calls need separate
 *            scratch.
 *   q, caches 16-byte aligned; seq_lens 4-byte aligned.
 */
bi_status bi_decode_attention(const void *q, const void *k_cache, const void *v_cache,
                              const int32_t *seq_lens, void *out, int64_t B, int64_t Hq, int64_t Hkv,
                              int64_t D, int64_t Lmax, float scale, void *scratch, size_t scratch_bytes,
                              void *stream);

/* Bytes of scratch bi_decode_attention needs (0 if any size is <= 0). */
size_t bi_decode_attention_scratch_bytes(int64_t B, int64_t Hq, int64_t D, int64_t Lmax);

/*
 * bi_get_device_status -- synchronise `stream`, then read and clear the current
 * device's status word.  *out receives BI_OK or the first error a kernel recorded
 * since the last read (BI_ERR_TIMEOUT for a bounded wait that ran out).
 * Returns BI_ERR_CUDA if the synchronisation or the read fails.
 */
bi_status bi_get_device_status(void *stream, int32_t *out);

/*
 * bi_selftest_wait_timeout -- launch one block that waits on a shared-memory
 * barrier nothing will complete, through the same bounded wait the GEMM uses,
 * with the given limit (nanoseconds, 1000 .. 10^10).  The wait gives up, records
 * BI_ERR_TIMEOUT in the status word and the kernel returns normally; the device
 * context stays usable.  For testing the failure path without a GPU fault.
 */
bi_status bi_selftest_wait_timeout(int64_t limit_ns, void *stream);

/* Human-readable name of a status code (static storage; never NULL). */
const char *bi_status_string(bi_status status);

/*
 * bi_gemm_config -- report the tile configuration the GEMM entry points use for a
 * weight of `weight_rows` rows in [N, K] (BI_B_NK) storage: N for bi_matmul /
 * bi_addmm, 2F for bi_matmul_silu_mul.  It reports the output tile bm x bn, K per
 * pipeline stage bk, the number of stages, and the K step of one tensor-core
 * instruction.  bn is 128 up to 1024 rows. Above that it is 192 where 192-column
 * tiles fill the B200's CTA pairs in fewer cost-weighted waves than 256-column tiles
 * for a 1024-row batch (e.g. 6144 or 24576 rows), else 256. [K, N] (BI_B_KN)
 * weights run bn = 256 where this reports 192.  The configuration depends on the
 * weight alone -- every M of a given weight runs the same one -- and all
 * configurations take the same 16-wide K steps in ascending order, so an element's
 * bits do not depend on it.  weight_rows <= 0 reports bn = 256.  Any pointer may be NULL.
 */
void bi_gemm_config(int64_t weight_rows, int32_t *bm, int32_t *bn, int32_t *bk, int32_t *stages, int32_t *mma_k);

/*
 * bi_tensor_map_cache_stats -- how many TMA tensor-map look-ups of the GEMM entry points were
 * served from the library's cache (*hits) and how many had to be encoded (*misses) since the
 * library was loaded.  A GEMM call looks up two maps (weights and activations), keyed by
 * (base address, extents, row stride, box); a repeated call with the same buffers hits twice.
 * Either pointer may be NULL.
 */
void bi_tensor_map_cache_stats(int64_t *hits, int64_t *misses);

/* Library version as major*10000 + minor*100 + patch. */
int32_t bi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BI_H */
