// rowops.cuh -- one-block-per-row reductions (RMSNorm, mean, log_softmax) and the
// elementwise SiLU-times-up glue.
//
// Batch invariance: a row is reduced by one thread block whose size, and whose
// assignment of elements to threads, depend only on the row length.  Each thread
// folds its elements in a fixed sequence; the per-thread partials meet in a fixed
// xor-butterfly over the warp and then a fixed butterfly over the warp partials.
// Nothing in a row's arithmetic depends on M, on the block's index or on timing, and
// no atomics are used.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "maxsum.cuh"
#include "ptx.cuh"

namespace bi {

// --------------------------------------------------------------- fixed-order trees

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Sum over the block; every thread returns the same bits.  `red` holds >= 32 floats.
__device__ __forceinline__ float block_sum(float v, float *red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    v = warp_sum(v);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = lane < nwarps ? red[lane] : 0.0f;
    t = warp_sum(t);
    __syncthreads();  // `red` may be reused by the caller
    return t;
}

__device__ __forceinline__ MaxSum block_merge(MaxSum v, float *red_m, float *red_s)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    v = warp_merge(v);
    if (lane == 0) {
        red_m[warp] = v.m;
        red_s[warp] = v.s;
    }
    __syncthreads();
    MaxSum t = lane < nwarps ? MaxSum{red_m[lane], red_s[lane]} : MaxSum{kNegInf, 0.0f};
    t = warp_merge(t);
    __syncthreads();
    return t;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&p);
}

// --------------------------------------------------------------- block-size rules
// Functions of the row length only.

__host__ __device__ inline int round_up32(long long v) { return (int)((v + 31) / 32 * 32); }

__host__ __device__ inline int clamp_threads(long long v)
{
    int t = round_up32(v);
    return t < 32 ? 32 : (t > 1024 ? 1024 : t);
}

// RMSNorm, bf16 rows: aim for two 16-byte chunks per thread.
__host__ inline int rmsnorm_threads(long long H) { return clamp_threads((H / 8 + 1) / 2); }
// mean, fp32 rows: aim for four 16-byte chunks per thread.
__host__ inline int mean_threads(long long H) { return clamp_threads((H / 4 + 3) / 4); }
// log_softmax, scalar path (rows whose length breaks the 16-byte vector rule).
__host__ inline int log_softmax_threads(long long V) { return clamp_threads((V + 7) / 8); }

// --------------------------------------------------------------- RMSNorm

// Vector path: H % 8 == 0, row held in registers as CPT 16-byte chunks per thread.
// Chunk c of a row belongs to thread c % T, as its (c / T)-th chunk.
template <int CPT>
__global__ void __launch_bounds__(1024) rmsnorm_vec_kernel(const uint4 *__restrict__ x,
                                                          const uint4 *__restrict__ w,
                                                          uint4 *__restrict__ y, int64_t H,
                                                          float eps)
{
    __shared__ float red[32];
    griddep_wait();  // the previous kernel's output (x) is complete
    griddep_launch_dependents();
    const int64_t nch = H / 8;
    const int T = blockDim.x;
    const uint4 *xr = x + (int64_t)blockIdx.x * nch;
    uint4 *yr = y + (int64_t)blockIdx.x * nch;

    uint4 v[CPT];
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int64_t c = threadIdx.x + (int64_t)i * T;
        v[i] = c < nch ? __ldg(xr + c) : make_uint4(0, 0, 0, 0);
    }
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const uint32_t q[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float a = bf16lo(q[k]), b = bf16hi(q[k]);
            ss = fmaf(a, a, ss);
            ss = fmaf(b, b, ss);
        }
    }
    ss = block_sum(ss, red);
    const float r = rsqrtf(ss / (float)H + eps);
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int64_t c = threadIdx.x + (int64_t)i * T;
        if (c < nch) {
            const uint4 wv = __ldg(w + c);
            const uint32_t q[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
            const uint32_t g[4] = {wv.x, wv.y, wv.z, wv.w};
            uint32_t o[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                o[k] = pack_bf16x2(__fmul_rn(__fmul_rn(bf16lo(q[k]), r), bf16lo(g[k])),
                                   __fmul_rn(__fmul_rn(bf16hi(q[k]), r), bf16hi(g[k])));
            yr[c] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

// Scalar path for any H: element j belongs to thread j % T; the row is read twice.
__global__ void __launch_bounds__(1024) rmsnorm_scalar_kernel(const __nv_bfloat16 *__restrict__ x,
                                                             const __nv_bfloat16 *__restrict__ w,
                                                             __nv_bfloat16 *__restrict__ y,
                                                             int64_t H, float eps)
{
    __shared__ float red[32];
    const __nv_bfloat16 *xr = x + (int64_t)blockIdx.x * H;
    __nv_bfloat16 *yr = y + (int64_t)blockIdx.x * H;
    float ss = 0.0f;
    for (int64_t j = threadIdx.x; j < H; j += blockDim.x) {
        const float a = __bfloat162float(xr[j]);
        ss = fmaf(a, a, ss);
    }
    ss = block_sum(ss, red);
    const float r = rsqrtf(ss / (float)H + eps);
    for (int64_t j = threadIdx.x; j < H; j += blockDim.x)
        yr[j] = __float2bfloat16_rn(
            __fmul_rn(__fmul_rn(__bfloat162float(xr[j]), r), __bfloat162float(w[j])));
}

// --------------------------------------------------------------- mean

// Vector path: H % 4 == 0.  Chunk c (4 floats) belongs to thread c % T; each thread
// keeps four running sums (one per float4 lane), adds its chunks in ascending order with four
// float4 loads in flight, and folds the sums as (s0+s1)+(s2+s3).  x is read once, with an
// evict-first hint, so the reads do not push out of L2 the lines of x (e.g. the last rows a
// log_softmax just wrote) not yet read.  Rows of at least 8 T chunks run mean_rows_kernel below,
// whose per-row arithmetic is the same.
__global__ void __launch_bounds__(1024) mean_vec_kernel(const float4 *__restrict__ x,
                                                       float *__restrict__ y, int64_t H)
{
    __shared__ float red[32];
    griddep_wait();  // the previous kernel's output (x) is complete
    griddep_launch_dependents();
    const int64_t nch = H / 4;
    const float4 *xr = x + (int64_t)blockIdx.x * nch;
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
    int64_t c = threadIdx.x;
    const int T = blockDim.x;
    for (; c + 3 * (int64_t)T < nch; c += 4 * (int64_t)T) {
        float4 a = __ldcs(xr + c), b = __ldcs(xr + c + T), d = __ldcs(xr + c + 2 * T),
               e = __ldcs(xr + c + 3 * T);
        s0 += a.x; s1 += a.y; s2 += a.z; s3 += a.w;
        s0 += b.x; s1 += b.y; s2 += b.z; s3 += b.w;
        s0 += d.x; s1 += d.y; s2 += d.z; s3 += d.w;
        s0 += e.x; s1 += e.y; s2 += e.z; s3 += e.w;
    }
    for (; c < nch; c += T) {
        float4 a = __ldcs(xr + c);
        s0 += a.x; s1 += a.y; s2 += a.z; s3 += a.w;
    }
    float s = __fadd_rn(__fadd_rn(s0, s1), __fadd_rn(s2, s3));
    s = block_sum(s, red);
    if (threadIdx.x == 0) y[blockIdx.x] = s / (float)H;
}

// Long rows (H / 4 >= 8 T), persistent: block b takes rows b, b + G, b + 2G, ... (G blocks, as
// many as fit at once), so rows do not wait for block launches; eight float4 loads per thread are
// in flight, and each block issues the first eight of its next row before the current row's
// block reduction, so the reduction overlaps those reads.  Per row the arithmetic is
// mean_vec_kernel's: thread t adds its chunks t, t + T, ... in ascending order into four running
// sums, folds them as (s0+s1)+(s2+s3), and the block tree adds the threads' sums.  (B200, fp32
// rows of 151936, L2 flushed: 103.9 us at M = 1024 against 108.6 us with a block per row; the
// same bits.)
constexpr int kMeanRowsThreads = 1024;  // the thread count mean_threads(H) gives every long row
__global__ void __launch_bounds__(kMeanRowsThreads) mean_rows_kernel(const float4 *__restrict__ x, float *__restrict__ y,
                                                        int64_t H, int64_t M)
{
    __shared__ float red[32];
    griddep_wait();  // the previous kernel's output (x) is complete
    griddep_launch_dependents();
    const int nch = (int)(H / 4);  // H < 2^31
    constexpr int T = kMeanRowsThreads;
    int64_t row = blockIdx.x;
    if (row >= M) return;
    float4 g[8];
    const float4 *xr = x + row * nch;
#pragma unroll
    for (int k = 0; k < 8; ++k) g[k] = __ldcs(xr + threadIdx.x + k * T);
    for (;;) {
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
        int c = threadIdx.x;
        for (;;) {  // g holds groups c, c + T, ..., c + 7T
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                s0 += g[k].x; s1 += g[k].y; s2 += g[k].z; s3 += g[k].w;
            }
            c += 8 * T;
            if (c + 7 * T >= nch) break;
#pragma unroll
            for (int k = 0; k < 8; ++k) g[k] = __ldcs(xr + c + k * T);
        }
        for (; c + 3 * T < nch; c += 4 * T) {
            float4 a = __ldcs(xr + c), b = __ldcs(xr + c + T), d = __ldcs(xr + c + 2 * T), e = __ldcs(xr + c + 3 * T);
            s0 += a.x; s1 += a.y; s2 += a.z; s3 += a.w;
            s0 += b.x; s1 += b.y; s2 += b.z; s3 += b.w;
            s0 += d.x; s1 += d.y; s2 += d.z; s3 += d.w;
            s0 += e.x; s1 += e.y; s2 += e.z; s3 += e.w;
        }
        for (; c < nch; c += T) {
            float4 a = __ldcs(xr + c);
            s0 += a.x; s1 += a.y; s2 += a.z; s3 += a.w;
        }
        const int64_t next = row + gridDim.x;
        if (next < M) {
            xr = x + next * nch;
#pragma unroll
            for (int k = 0; k < 8; ++k) g[k] = __ldcs(xr + threadIdx.x + k * T);
        }
        float sum = __fadd_rn(__fadd_rn(s0, s1), __fadd_rn(s2, s3));
        sum = block_sum(sum, red);
        if (threadIdx.x == 0) y[row] = sum / (float)H;
        if (next >= M) break;
        row = next;
    }
}

__global__ void __launch_bounds__(1024) mean_scalar_kernel(const float *__restrict__ x,
                                                          float *__restrict__ y, int64_t H)
{
    __shared__ float red[32];
    const float *xr = x + (int64_t)blockIdx.x * H;
    float s = 0.f;
    for (int64_t j = threadIdx.x; j < H; j += blockDim.x) s += xr[j];
    s = block_sum(s, red);
    if (threadIdx.x == 0) y[blockIdx.x] = s / (float)H;
}

// --------------------------------------------------------------- log_softmax

// Scalar path for any V: element j belongs to thread j % T.
template <bool BF16>
__global__ void __launch_bounds__(1024, 1) log_softmax_scalar_kernel(const void *__restrict__ xv,
                                                                    float *__restrict__ y,
                                                                    int64_t V)
{
    __shared__ float red_m[32], red_s[32];
    const int64_t base = (int64_t)blockIdx.x * V;
    auto load = [&](int64_t j) -> float {
        if (BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(xv)[base + j]);
        return reinterpret_cast<const float *>(xv)[base + j];
    };
    MaxSum acc{kNegInf, 0.0f};
    for (int64_t j = threadIdx.x; j < V; j += blockDim.x) {
        float v[1] = {load(j)};
        lsm_accumulate(acc, v);
    }
    const MaxSum row = block_merge(acc, red_m, red_s);
    const float m = row.m, ls = __logf(row.s);
    for (int64_t j = threadIdx.x; j < V; j += blockDim.x) y[base + j] = (load(j) - m) - ls;
}

// --------------------------------------------------------------- log_softmax, streamed rows

// Vector path of log_softmax.  One block of kLsmThreads threads per row, two blocks per
// SM.  The row streams through a ring of kLsmStages shared-memory chunks of kLsmChunk
// bytes, each filled by one 1-D bulk copy that completes on its own mbarrier.  Pass 1
// builds the row's (max, sum of exp); pass 2 writes y = (x - max) - log(sum), starting
// with the last chunks of the row, which are still in the ring, and streaming the rest
// again in descending order, so the chunk read most recently (the likeliest to be still in
// L2) comes first.  Pass-1 copies of the chunks pass 2 reads again ask L2 to keep their lines;
// every other copy (the chunks that stay in the ring, and the second reads) asks it to drop
// them, and y is written with streaming stores, so that neither pushes the rows' inputs out of
// L2 before their second read.  (B200, M = 1024, V = 151936
// bf16 with L2 flushed: 180 us, against 186 us with ascending re-reads and default-policy y
// stores; the same bits.)
//
// Element order (fixed by V alone): the row is cut into chunks of kLsmChunk bytes and, in
// pass 1, each chunk into sub-blocks of kLsmFoldBytes; a sub-block into groups of 8 elements,
// thread t owning groups t and t + T (bf16; group t for fp32): per sub-block a thread takes the
// maximum of its elements, rescales its running pair once and adds their exp(x - max) in
// order, sub-block after sub-block.  Pass 2 writes 4-element groups,
// thread t owning t, t + T, ...  Consecutive threads read consecutive 16-byte shared-memory
// pieces and write consecutive 16-byte pieces of y.
//
// Copy schedule: copy j (j = 0, 1, ...) goes to stage j % S and completes phase j / S of
// that stage's barrier.  Copies 0 .. n-1 are the n chunks of pass 1; copies n .. n+R-1
// (R = max(0, n - S)) are chunks R-1, R-2, .., 0 again for pass 2.  Chunks R .. n-1 are still in
// their stages when pass 1 ends and are used by pass 2 without a copy.  A copy is issued
// once the previous occupant of its stage has been consumed for the last time.
constexpr int kLsmThreads = 512;
constexpr int kLsmChunk = 32768;      // bytes per bulk copy
constexpr int kLsmStages = 3;
constexpr int kLsmFoldBytes = 16384;  // pass 1 folds a chunk in sub-blocks of this many bytes

template <bool BF16>
__global__ void __launch_bounds__(kLsmThreads, 2)
    log_softmax_stream_kernel(const uint8_t *__restrict__ x, float *__restrict__ y, int64_t V,
                              int32_t *status, uint64_t wait_limit_ns)
{
    constexpr int kElem = BF16 ? 2 : 4;
    constexpr int kPerChunk = kLsmChunk / kElem;      // elements per chunk
    extern __shared__ __align__(128) uint8_t lsm_smem[];
    uint8_t(*ring)[kLsmChunk] = reinterpret_cast<uint8_t(*)[kLsmChunk]>(lsm_smem);
    __shared__ uint64_t full[kLsmStages];
    __shared__ float red_m[32], red_s[32];
    __shared__ int abort_flag_s;
    volatile int *abort_flag = &abort_flag_s;

    const int64_t row_bytes = V * kElem;
    const int n = (int)((row_bytes + kLsmChunk - 1) / kLsmChunk);
    const int R = n > kLsmStages ? n - kLsmStages : 0;  // chunks pass 2 must copy again
    const int copies = n + R;
    const uint8_t *xr = x + (int64_t)blockIdx.x * row_bytes;
    float *yr = y + (int64_t)blockIdx.x * V;
    const int tid = threadIdx.x;

    if (tid == 0) {
        for (int s = 0; s < kLsmStages; ++s) mbar_init(&full[s], 1);
        abort_flag_s = 0;
        fence_mbar_init();
    }
    griddep_wait();  // the previous kernel's output (x) is complete
    griddep_launch_dependents();
    __syncthreads();

    int issued = 0;  // meaningful in thread 0 only
    // Chunk held by copy j: pass 1 in ascending order, pass 2 (copies n .. n+R-1) over chunks
    // R-1 down to 0.
    auto chunk_of = [&](int j) -> int { return j < n ? j : R - 1 - (j - n); };
    auto issue = [&](int j) {
        const int c = chunk_of(j);
        const int64_t off = (int64_t)c * kLsmChunk;
        const uint32_t bytes = (uint32_t)(row_bytes - off < kLsmChunk ? row_bytes - off : kLsmChunk);
        uint64_t *bar = &full[j % kLsmStages];
        mbar_arrive_expect_tx(bar, bytes);
        // Only the chunks pass 2 reads again (0 .. R-1) ask L2 to keep their lines.
        bulk_load_hint(ring[j % kLsmStages], xr + off, bytes, bar,
                       j < R ? l2_policy_evict_last() : l2_policy_evict_first());
    };
    if (tid == 0)
        for (; issued < kLsmStages && issued < n; ++issued) issue(issued);

    // Wait for copy j (all threads agree on the outcome).
    auto landed = [&](int j) -> bool {
        const bool ok = wait_bounded(&full[j % kLsmStages], (uint32_t)(j / kLsmStages) & 1u,
                                     abort_flag, status, wait_limit_ns);
        return __syncthreads_and(ok ? 1 : 0) != 0;
    };
    // Fold the chunk held by copy j: thread t takes the 8-element groups t, t + T, ... of the
    // chunk (one 16-byte shared-memory read per group for bf16, two for fp32; elements past V
    // count as -inf), reduces them to their maximum, rescales its running pair once, then adds
    // exp(x - max) for its elements in order.
    MaxSum acc{kNegInf, 0.0f};
    float m = 0.0f, ls = 0.0f;
    // Pass 1 folds a chunk in sub-blocks of kLsmFoldBytes, each as described above.
    constexpr int kSubPer = kLsmFoldBytes / kElem;        // elements per sub-block
    constexpr int kFoldPer = kSubPer / kLsmThreads;        // per thread and sub-block: 16 bf16, 8 fp32
    // Elements of the row in the chunk of copy j (kPerChunk except in the row's last chunk).
    auto chunk_valid = [&](int j) -> int {
        const int64_t e0 = (int64_t)chunk_of(j) * kPerChunk;
        return V - e0 < kPerChunk ? (int)(V - e0) : kPerChunk;
    };
    auto fold = [&](int j) {
        const int chunk_elems = chunk_valid(j);
#pragma unroll 1
        for (int sb = 0; sb < kLsmChunk / kLsmFoldBytes; ++sb) {
            const int valid = chunk_elems - sb * kSubPer;  // elements of the row in this sub-block
            if (valid <= 0) break;
            const uint8_t *buf = ring[j % kLsmStages] + sb * kLsmFoldBytes;
            float v[kFoldPer];
#pragma unroll
            for (int i = 0; i < kFoldPer / 8; ++i) {
                const int g = tid + i * kLsmThreads;
                float *w = v + 8 * i;
                if (BF16) {
                    const uint4 u =
                        8 * g < valid ? *reinterpret_cast<const uint4 *>(buf + 16 * g) : make_uint4(0, 0, 0, 0);
                    w[0] = bf16lo(u.x); w[1] = bf16hi(u.x); w[2] = bf16lo(u.y); w[3] = bf16hi(u.y);
                    w[4] = bf16lo(u.z); w[5] = bf16hi(u.z); w[6] = bf16lo(u.w); w[7] = bf16hi(u.w);
                } else {
                    const float4 a = 8 * g < valid ? *reinterpret_cast<const float4 *>(buf + 32 * g)
                                                   : make_float4(0, 0, 0, 0);
                    const float4 b = 8 * g + 4 < valid ? *reinterpret_cast<const float4 *>(buf + 32 * g + 16)
                                                       : make_float4(0, 0, 0, 0);
                    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
                }
            }
            if (valid < kSubPer) {  // the row's last sub-block: elements past V count as -inf
#pragma unroll
                for (int i = 0; i < kFoldPer / 8; ++i)
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        if (8 * (tid + i * kLsmThreads) + k >= valid) v[8 * i + k] = kNegInf;
            }
            lsm_accumulate(acc, v);
        }
    };
    // Write y for the chunk held by copy j: thread t takes the 4-element groups t, t + T, ...
    // (one coalesced 16-byte store each).
    auto write_y = [&](int j) {
        const int valid = chunk_valid(j);
        const uint8_t *buf = ring[j % kLsmStages];
        float4 *yc = reinterpret_cast<float4 *>(yr + (int64_t)chunk_of(j) * kPerChunk);
        for (int g = tid; 4 * g < valid; g += kLsmThreads) {
            float v[4];
            if (BF16) {
                const uint2 u = *reinterpret_cast<const uint2 *>(buf + 8 * g);
                v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
            } else {
                const float4 f = *reinterpret_cast<const float4 *>(buf + 16 * g);
                v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
            }
            __stcs(yc + g, make_float4((v[0] - m) - ls, (v[1] - m) - ls, (v[2] - m) - ls, (v[3] - m) - ls));
        }
    };
    // After the last use of copy j's stage, start copy j + S if it exists.
    auto refill = [&](int j) {
        __syncthreads();  // every thread is done with this stage
        if (tid == 0 && j + kLsmStages < copies && issued == j + kLsmStages) {
            fence_proxy_async_smem();  // order the reads above before the copy that overwrites
            issue(issued++);
        }
    };

    bool ok = true;
    // Pass 1: copies 0 .. n-1.  Stages of the last S chunks are kept for pass 2.
    for (int j = 0; j < n && ok; ++j) {
        if (!(ok = landed(j))) break;
        fold(j);
        if (j + kLsmStages < n) refill(j);
        else __syncthreads();
    }
    if (ok) {
        const MaxSum row = block_merge(acc, red_m, red_s);
        m = row.m;
        ls = __logf(row.s);
        // Pass 2, resident chunks R .. n-1 (copies R .. n-1), then copies n .. n+R-1.
        for (int j = R; j < n; ++j) {
            write_y(j);
            refill(j);
        }
        for (int j = n; j < copies && ok; ++j) {
            if (!(ok = landed(j))) break;
            write_y(j);
            refill(j);
        }
    }
    if (!ok && tid == 0) {
        // A wait ran out: let every copy already issued land before the block's shared
        // memory goes away (at most one outstanding copy per stage).
        for (int j = issued > kLsmStages ? issued - kLsmStages : 0; j < issued; ++j) {
            const uint32_t a = smem_addr(&full[j % kLsmStages]);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(a, (uint32_t)(j / kLsmStages) & 1u) &&
                   global_timer_ns() - t0 < wait_limit_ns) {
            }
        }
    }
}

constexpr int kLsmSmem = kLsmStages * kLsmChunk;

// --------------------------------------------------------------- long rows: one cluster per row

// The cluster variant of log_softmax (bi_log_softmax_cluster, an opt-in entry point beside the
// one-block-per-row bi_log_softmax): rows of at least kClusterRowBytes bytes whose slices fit in
// shared memory are reduced by a cluster of kRowCluster CTAs.  CTA r owns the slice [r S, min(V, (r + 1) S)) of the row, with
// S = cluster_slice(V) a multiple of 8 elements fixed by V alone.  Each CTA reduces its slice
// in a fixed order; the CTAs' results meet through distributed shared memory and are folded in
// rank order 0, 1, ..., kRowCluster - 1.  A short batch spreads over kRowCluster times as many
// SMs as with one block per row, and each CTA keeps its slice in shared memory between the two
// passes: the row is read from global memory once.
#ifndef BI_ROW_CLUSTER
#define BI_ROW_CLUSTER 4           // the one cluster shape every call uses; other values exist for experiments only
#endif
#ifndef BI_ROW_CLUSTER_THREADS
#define BI_ROW_CLUSTER_THREADS 512
#endif
#ifndef BI_CLUSTER_ROW_BYTES
#define BI_CLUSTER_ROW_BYTES (64 * 1024)
#endif
constexpr int kRowCluster = BI_ROW_CLUSTER;
constexpr int kClThreads = BI_ROW_CLUSTER_THREADS;
constexpr int64_t kClusterRowBytes = BI_CLUSTER_ROW_BYTES;
constexpr int kClSliceBytesMax = 96 * 1024;  // log_softmax: largest slice held in shared memory
constexpr int kClPieces = 4;                 // bulk copies per slice, each on its own barrier

__host__ __device__ inline int64_t cluster_slice(int64_t V)
{
    return (V + 8 * kRowCluster - 1) / (8 * kRowCluster) * 8;
}

// log_softmax of one row per cluster; V % 8 == 0 (bf16) or V % 4 == 0 (fp32), x and y 16-byte
// aligned, cluster_slice(V) * element size <= kClSliceBytesMax.  Grid (kRowCluster, rows).
// Inside a slice, thread t folds the 4-element groups t, t + T, ... of each bulk piece in turn.
template <bool BF16>
__global__ void __launch_bounds__(kClThreads) log_softmax_cluster_kernel(
    const uint8_t *__restrict__ x, float *__restrict__ y, int64_t V, int32_t *status, uint64_t wait_limit_ns,
    int64_t row0)
{
    constexpr int kElem = BF16 ? 2 : 4;
    extern __shared__ __align__(128) uint8_t cl_smem[];
    __shared__ uint64_t full[kClPieces];
    __shared__ float red_m[32], red_s[32];
    __shared__ float2 cta_part;
    __shared__ int abort_flag_s;
    volatile int *abort_flag = &abort_flag_s;

    const int tid = threadIdx.x;
    const uint32_t rank = cluster_ctarank();
    const int64_t row = row0 + blockIdx.y;
    const int64_t S = cluster_slice(V);
    const int64_t e_begin = (int64_t)rank * S;
    const int64_t e_end = e_begin + S < V ? e_begin + S : V;
    const int64_t n = e_end > e_begin ? e_end - e_begin : 0;  // elements of this CTA's slice
    const uint32_t bytes = (uint32_t)(n * kElem);             // a multiple of 16
    const uint32_t piece = ((bytes + kClPieces - 1) / kClPieces + 15u) / 16u * 16u;
    const uint8_t *src = x + (row * V + e_begin) * kElem;

    if (tid == 0) {
        for (int p = 0; p < kClPieces; ++p) mbar_init(&full[p], 1);
        abort_flag_s = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        const uint64_t pol = l2_policy_evict_first();  // each byte of x is read once
        for (int p = 0; p < kClPieces; ++p) {
            const uint32_t off = (uint32_t)p * piece;
            const uint32_t b = off < bytes ? (bytes - off < piece ? bytes - off : piece) : 0u;
            if (b) {
                mbar_arrive_expect_tx(&full[p], b);
                bulk_load_hint(cl_smem + off, src + off, b, &full[p], pol);
            } else {
                mbar_arrive(&full[p]);  // an empty piece completes at once
            }
        }
    }

    auto load4 = [&](int64_t g, float (&v)[4]) {
        if (BF16) {
            const uint2 u = *reinterpret_cast<const uint2 *>(cl_smem + 8 * g);
            v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
        } else {
            const float4 f = *reinterpret_cast<const float4 *>(cl_smem + 16 * g);
            v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
        }
    };

    MaxSum acc{kNegInf, 0.0f};
    bool ok = true;
    for (int p = 0; p < kClPieces; ++p) {
        const bool got = wait_bounded(&full[p], 0, abort_flag, status, wait_limit_ns);
        ok = __syncthreads_and(got ? 1 : 0) != 0;
        if (!ok) break;
        const uint32_t off = (uint32_t)p * piece;
        const int64_t g0 = off / (4 * kElem);                                   // first group
        const int64_t g1 = (off + piece < bytes ? off + piece : bytes) / (4 * kElem);
        for (int64_t g = g0 + tid; g < g1; g += kClThreads) {
            float v[4];
            load4(g, v);
            lsm_accumulate(acc, v);
        }
    }
    const MaxSum cta = ok ? block_merge(acc, red_m, red_s) : MaxSum{kNegInf, 0.0f};
    if (tid == 0) cta_part = make_float2(cta.m, cta.s);
    cluster_sync_all();  // every CTA's (max, sum) is visible to the cluster
    MaxSum row_ms{kNegInf, 0.0f};
    for (uint32_t r = 0; r < (uint32_t)kRowCluster; ++r) {
        const float2 pr = ld_dsmem_f32x2(map_to_rank(smem_addr(&cta_part), r));
        row_ms = merge(row_ms, MaxSum{pr.x, pr.y});
    }
    if (ok) {
        const float m = row_ms.m, ls = __logf(row_ms.s);
        float *yr = y + row * V + e_begin;
        for (int64_t g = tid; 4 * g < n; g += kClThreads) {
            float v[4];
            load4(g, v);
            __stcs(reinterpret_cast<float4 *>(yr + 4 * g),
                   make_float4((v[0] - m) - ls, (v[1] - m) - ls, (v[2] - m) - ls, (v[3] - m) - ls));
        }
    } else if (tid == 0) {
        // A wait ran out: let the copies already issued land before shared memory goes away.
        for (int p = 0; p < kClPieces; ++p) {
            const uint32_t a = smem_addr(&full[p]);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(a, 0) && global_timer_ns() - t0 < wait_limit_ns) {
            }
        }
    }
    cluster_sync_all();  // no CTA leaves while a peer may still read its cta_part
}

// --------------------------------------------------------------- log_softmax, split rows

// Fixed-chunk multi-block variant for short batches.  The row is cut into chunks of
// kSplitChunk elements (a constant, so the cut depends on V alone); block (c, i) reduces
// chunk c of row i to a (max, sum of exp) partial, then, in a second launch, every block
// of row i merges the row's partials in the same fixed tree and writes its chunk of y.
// Within a chunk, thread t owns the 8-element groups t, t + T, ... in that order.
// Partials live in caller-provided scratch: one float2 (max, sum) per (row, chunk).
constexpr int kSplitThreads = 256;
constexpr int kSplitChunk = 4096;  // elements per chunk

__host__ __device__ inline int64_t split_chunks(int64_t V) { return (V + kSplitChunk - 1) / kSplitChunk; }

template <bool BF16>
__device__ __forceinline__ void split_load8(const uint8_t *row, int64_t e, float (&v)[8])
{
    if (BF16) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(row + 2 * e));
        v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
        v[4] = bf16lo(u.z); v[5] = bf16hi(u.z); v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
    } else {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(row + 4 * e));
        const float4 b = __ldg(reinterpret_cast<const float4 *>(row + 4 * e) + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
}

// Launch 1: grid (chunks, M).  V % 8 == 0, x 16-byte aligned.
template <bool BF16>
__global__ void __launch_bounds__(kSplitThreads) log_softmax_split_stats_kernel(
    const uint8_t *__restrict__ x, float2 *__restrict__ partial, int64_t V)
{
    __shared__ float red_m[32], red_s[32];
    constexpr int kElem = BF16 ? 2 : 4;
    const int64_t nch = split_chunks(V);
    const int64_t row = blockIdx.y, c = blockIdx.x;
    const uint8_t *xr = x + row * V * kElem;
    const int64_t e0 = c * kSplitChunk;
    MaxSum acc{kNegInf, 0.0f};
    for (int g = threadIdx.x; g < kSplitChunk / 8; g += kSplitThreads) {
        const int64_t e = e0 + 8 * (int64_t)g;
        if (e >= V) break;
        float v[8];
        split_load8<BF16>(xr, e, v);
        lsm_accumulate(acc, v);
    }
    const MaxSum part = block_merge(acc, red_m, red_s);
    if (threadIdx.x == 0) partial[row * nch + c] = make_float2(part.m, part.s);
}

// Launch 2: grid (chunks, M).  Merge the row's partials (lane l folds chunks l, l+32, ...
// in order, then a fixed xor butterfly), then write y for this block's chunk.
template <bool BF16>
__global__ void __launch_bounds__(kSplitThreads) log_softmax_split_write_kernel(
    const uint8_t *__restrict__ x, const float2 *__restrict__ partial, float *__restrict__ y, int64_t V)
{
    __shared__ float row_stats[2];
    constexpr int kElem = BF16 ? 2 : 4;
    const int64_t nch = split_chunks(V);
    const int64_t row = blockIdx.y, c = blockIdx.x;
    if (threadIdx.x < 32) {
        MaxSum acc{kNegInf, 0.0f};
        for (int64_t k = threadIdx.x; k < nch; k += 32) {
            const float2 pk = partial[row * nch + k];
            acc = merge(acc, MaxSum{pk.x, pk.y});
        }
        acc = warp_merge(acc);
        if (threadIdx.x == 0) {
            row_stats[0] = acc.m;
            row_stats[1] = __logf(acc.s);
        }
    }
    __syncthreads();
    const float m = row_stats[0], ls = row_stats[1];
    const uint8_t *xr = x + row * V * kElem;
    float *yr = y + row * V;
    const int64_t e0 = c * kSplitChunk;
    for (int g = threadIdx.x; g < kSplitChunk / 8; g += kSplitThreads) {
        const int64_t e = e0 + 8 * (int64_t)g;
        if (e >= V) break;
        float v[8];
        split_load8<BF16>(xr, e, v);
        float4 *dst = reinterpret_cast<float4 *>(yr + e);
        __stcs(dst, make_float4((v[0] - m) - ls, (v[1] - m) - ls, (v[2] - m) - ls, (v[3] - m) - ls));
        __stcs(dst + 1, make_float4((v[4] - m) - ls, (v[5] - m) - ls, (v[6] - m) - ls, (v[7] - m) - ls));
    }
}

// --------------------------------------------------------------- SiLU * up

__device__ __forceinline__ float silu_mul1(float g, float u)
{
    return __fmul_rn(g / (1.0f + __expf(-g)), u);
}

// F % 8 == 0: thread handles 8 outputs (one 16-byte chunk of h) per step.
__global__ void __launch_bounds__(256) silu_mul_vec_kernel(const uint4 *__restrict__ gu,
                                                          uint4 *__restrict__ h, int64_t M,
                                                          int64_t F)
{
    const int64_t fch = F / 8;
    const int64_t total = M * fch;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / fch, c = e % fch;
        const uint4 g = __ldg(gu + i * 2 * fch + c);
        const uint4 u = __ldg(gu + i * 2 * fch + fch + c);
        const uint32_t gq[4] = {g.x, g.y, g.z, g.w}, uq[4] = {u.x, u.y, u.z, u.w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
            o[k] = pack_bf16x2(silu_mul1(bf16lo(gq[k]), bf16lo(uq[k])),
                               silu_mul1(bf16hi(gq[k]), bf16hi(uq[k])));
        h[e] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

__global__ void __launch_bounds__(256) silu_mul_scalar_kernel(const __nv_bfloat16 *__restrict__ gu,
                                                             __nv_bfloat16 *__restrict__ h,
                                                             int64_t M, int64_t F)
{
    const int64_t total = M * F;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / F, j = e % F;
        h[e] = __float2bfloat16_rn(silu_mul1(__bfloat162float(gu[i * 2 * F + j]),
                                             __bfloat162float(gu[i * 2 * F + F + j])));
    }
}

}  // namespace bi
