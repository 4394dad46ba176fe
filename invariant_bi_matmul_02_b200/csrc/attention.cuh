// attention.cuh -- batch-invariant decode attention (one query token per sequence).
//
// The key/value cache of a sequence is cut into splits of kAttnSplit tokens, a cut fixed
// by the sequence's own length.  Launch 1 gives every (split, kv head, sequence) one block,
// which produces, for each query head of the kv head's group, the split's maximum score,
// its sum of exp(score - max) and the matching weighted sum of value rows.  Launch 2
// folds the splits of each (sequence, query head) in ascending split order.  Every
// reduction is a fixed sequence or a fixed tree, so a sequence's output depends on its own
// query, cache and length only -- not on the batch it is decoded in or its position there.
//
// Layouts (row-major, bf16): q [B, Hq, D]; k, v [B, Lmax, Hkv, D]; out [B, Hq, D].  Query
// head h reads kv head h / (Hq / Hkv).  D = 128.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "rowops.cuh"

namespace bi {

constexpr int kAttnD = 128;
constexpr int kAttnSplit = 128;       // tokens per split (one per thread in the score phase)
constexpr int kAttnThreads = 128;
constexpr int kAttnMaxGroup = 8;      // query heads per kv head
constexpr int kAttnKStride = kAttnD + 8;  // padded K row (bf16): conflict-free 16-byte reads

struct AttnSmem {
    __nv_bfloat16 k[kAttnSplit][kAttnKStride];
    __nv_bfloat16 v[kAttnSplit][kAttnD];
    __nv_bfloat16 q[kAttnMaxGroup][kAttnD];
    float p[kAttnMaxGroup][kAttnSplit];
    float red[kAttnMaxGroup][4];
    float stat[kAttnMaxGroup][2];
};

__host__ __device__ inline int64_t attn_splits(int64_t L) { return (L + kAttnSplit - 1) / kAttnSplit; }

// Launch 1: grid (ceil(Lmax / kAttnSplit), Hkv, B), kAttnThreads threads, sizeof(AttnSmem)
// bytes of dynamic shared memory.  part_ms: [B, Hq, S] float2 (max, sum); part_acc:
// [B, Hq, S, D] float, S = ceil(Lmax / kAttnSplit).
template <int G>  // query heads per kv head (1, 2, 4 or 8)
__global__ void __launch_bounds__(kAttnThreads)
    decode_attention_split_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                                  const __nv_bfloat16 *__restrict__ v, const int32_t *__restrict__ lens,
                                  float2 *__restrict__ part_ms, float *__restrict__ part_acc, int Hq, int Hkv,
                                  int64_t Lmax, float scale, int32_t *status)
{
    extern __shared__ __align__(16) uint8_t attn_raw[];
    AttnSmem &sm = *reinterpret_cast<AttnSmem *>(attn_raw);
    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t S = attn_splits(Lmax);
    int64_t L = lens[b];
    if (L < 1 || L > Lmax) {
        if (tid == 0) *reinterpret_cast<volatile int32_t *>(status) = 1;  // BI_ERR_INVALID_ARG
        L = L < 1 ? 1 : Lmax;
    }
    const int64_t t0 = (int64_t)split * kAttnSplit;
    if (t0 >= L) return;  // this split is past the sequence's end: it has no partial
    const int n_tok = (int)(L - t0 < kAttnSplit ? L - t0 : kAttnSplit);

    // Stage q for the group's query heads and the split's K rows (copy group 1), then the V rows
    // (copy group 2), all as 16-byte async copies; rows past the sequence are zero-filled.  The
    // scores only wait for group 1, so V lands while they are computed.
    for (int c = tid; c < G * (kAttnD / 8); c += kAttnThreads) {
        const int j = c / (kAttnD / 8), col = (c % (kAttnD / 8)) * 8;
        cp_async16(&sm.q[j][col], q + ((int64_t)b * Hq + (int64_t)g * G + j) * kAttnD + col, 16u);
    }
    for (int c = tid; c < kAttnSplit * (kAttnD / 8); c += kAttnThreads) {
        const int row = c / (kAttnD / 8), col = (c % (kAttnD / 8)) * 8;
        const bool in = row < n_tok;
        const int64_t off = in ? (((int64_t)b * Lmax + t0 + row) * Hkv + g) * kAttnD + col : 0;
        cp_async16(&sm.k[row][col], k + off, in ? 16u : 0u);
    }
    cp_async_commit();
    for (int c = tid; c < kAttnSplit * (kAttnD / 8); c += kAttnThreads) {
        const int row = c / (kAttnD / 8), col = (c % (kAttnD / 8)) * 8;
        const bool in = row < n_tok;
        const int64_t off = in ? (((int64_t)b * Lmax + t0 + row) * Hkv + g) * kAttnD + col : 0;
        cp_async16(&sm.v[row][col], v + off, in ? 16u : 0u);
    }
    cp_async_commit();
    cp_async_wait_pending<1>();  // q and K have landed (V may still be in flight)
    __syncthreads();

    // Scores: thread t takes token t0 + t; s_j = scale * sum_d q_j[d] k_t[d], d ascending.
    float s[G];
#pragma unroll
    for (int j = 0; j < G; ++j) s[j] = 0.0f;
#pragma unroll 2
    for (int d = 0; d < kAttnD; d += 8) {
        const uint4 kw = *reinterpret_cast<const uint4 *>(&sm.k[tid][d]);
        const float kf[8] = {bf16lo(kw.x), bf16hi(kw.x), bf16lo(kw.y), bf16hi(kw.y),
                             bf16lo(kw.z), bf16hi(kw.z), bf16lo(kw.w), bf16hi(kw.w)};
#pragma unroll
        for (int j = 0; j < G; ++j) {
            // q rows are read as 16-byte broadcasts (every thread the same address)
            const uint4 qw = *reinterpret_cast<const uint4 *>(&sm.q[j][d]);
            const float qv[8] = {bf16lo(qw.x), bf16hi(qw.x), bf16lo(qw.y), bf16hi(qw.y),
                                 bf16lo(qw.z), bf16hi(qw.z), bf16lo(qw.w), bf16hi(qw.w)};
#pragma unroll
            for (int e = 0; e < 8; ++e) s[j] = fmaf(qv[e], kf[e], s[j]);
        }
    }
    const bool live = tid < n_tok;
#pragma unroll
    for (int j = 0; j < G; ++j) s[j] = live ? s[j] * scale : kNegInf;

    // Per head: maximum over the split (fixed butterfly, then warp partials in order).
#pragma unroll
    for (int j = 0; j < G; ++j) {
        float m = s[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) sm.red[j][warp] = m;
    }
    __syncthreads();
    if (tid < G) {
        float m = sm.red[tid][0];
        for (int w = 1; w < kAttnThreads / 32; ++w) m = fmaxf(m, sm.red[tid][w]);
        sm.stat[tid][0] = m;
    }
    __syncthreads();
    // p = exp(s - m); per-head sums by the same fixed tree.
#pragma unroll
    for (int j = 0; j < G; ++j) {
        const float pj = live ? __expf(s[j] - sm.stat[j][0]) : 0.0f;
        sm.p[j][tid] = pj;
        const float w_sum = warp_sum(pj);
        if (lane == 0) sm.red[j][warp] = w_sum;
    }
    __syncthreads();
    if (tid < G) {
        float l = sm.red[tid][0];
        for (int w = 1; w < kAttnThreads / 32; ++w) l = __fadd_rn(l, sm.red[tid][w]);
        sm.stat[tid][1] = l;
    }
    __syncthreads();

    cp_async_wait_pending<0>();  // V has landed
    __syncthreads();

    // Weighted value sums: thread d accumulates sum_t p_j[t] v_t[d], t ascending.
    float acc[G];
#pragma unroll
    for (int j = 0; j < G; ++j) acc[j] = 0.0f;
    // Tokens four at a time (p rows read as 16-byte broadcasts); rows past n_tok hold p = 0
    // and zero-filled values, so the padded tail adds exact zeros.
    for (int t = 0; t < n_tok; t += 4) {
        const float v0 = __bfloat162float(sm.v[t][tid]), v1 = __bfloat162float(sm.v[t + 1][tid]),
                    v2 = __bfloat162float(sm.v[t + 2][tid]), v3 = __bfloat162float(sm.v[t + 3][tid]);
#pragma unroll
        for (int j = 0; j < G; ++j) {
            const float4 pj = *reinterpret_cast<const float4 *>(&sm.p[j][t]);
            acc[j] = fmaf(pj.x, v0, acc[j]);
            acc[j] = fmaf(pj.y, v1, acc[j]);
            acc[j] = fmaf(pj.z, v2, acc[j]);
            acc[j] = fmaf(pj.w, v3, acc[j]);
        }
    }
#pragma unroll
    for (int j = 0; j < G; ++j) {
        const int64_t bh = (int64_t)b * Hq + (int64_t)g * G + j;
        part_acc[(bh * S + split) * kAttnD + tid] = acc[j];
        if (tid == 0) part_ms[bh * S + split] = make_float2(sm.stat[j][0], sm.stat[j][1]);
    }
}

// Launch 2: grid (Hq, B), kAttnD threads.  Fold the sequence's splits in ascending order.
__global__ void __launch_bounds__(kAttnD)
    decode_attention_combine_kernel(const float2 *__restrict__ part_ms, const float *__restrict__ part_acc,
                                    const int32_t *__restrict__ lens, __nv_bfloat16 *__restrict__ out,
                                    int Hq, int64_t Lmax)
{
    const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
    const int64_t S = attn_splits(Lmax);
    int64_t L = lens[b];
    L = L < 1 ? 1 : (L > Lmax ? Lmax : L);
    const int64_t n = attn_splits(L);
    const int64_t bh = (int64_t)b * Hq + h;
    float m = kNegInf;
    for (int64_t s = 0; s < n; ++s) m = fmaxf(m, part_ms[bh * S + s].x);
    float l = 0.0f, o = 0.0f;
    for (int64_t s = 0; s < n; ++s) {
        const float2 ms = part_ms[bh * S + s];
        const float w = __expf(ms.x - m);
        l = fmaf(ms.y, w, l);
        o = fmaf(part_acc[(bh * S + s) * kAttnD + d], w, o);
    }
    out[bh * kAttnD + d] = __float2bfloat16_rn(o / l);
}

}  // namespace bi
