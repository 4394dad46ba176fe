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
constexpr int kAttnStride = kAttnD + 8;  // padded row (bf16): conflict-free ldmatrix rows
constexpr int kAttnWarps = kAttnThreads / 32;

struct AttnSmem {
    __nv_bfloat16 q[16][kAttnStride];           // the group's query heads, rows >= G zero
    union {
        __nv_bfloat16 k[kAttnSplit][kAttnStride];
        float o[kAttnWarps][kAttnMaxGroup][kAttnD];  // per-warp partial outputs, after the scores
    } ko;
    __nv_bfloat16 v[kAttnSplit][kAttnStride];
    float red[kAttnWarps][16];
    float stat[16][2];
};

__host__ __device__ inline int64_t attn_splits(int64_t L) { return (L + kAttnSplit - 1) / kAttnSplit; }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&p);
}

// Launch 1: grid (ceil(Lmax / kAttnSplit), Hkv, B), kAttnThreads threads, sizeof(AttnSmem)
// bytes of dynamic shared memory.  part_ms: [B, Hq, S] float2 (max, sum); part_acc:
// [B, Hq, S, D] float, S = ceil(Lmax / kAttnSplit).
//
// Tensor-core form (mma.sync m16n8k16, bf16 in, fp32 accumulate).  Warp w owns tokens
// 32w .. 32w+31 of the split.  Scores: S = Q . K^T with Q the group's heads padded to 16 rows;
// every score accumulates its eight 16-wide D steps in ascending order.  Then, per head, the
// split's maximum and sum of exp(s - max) (fp32) come from fixed trees: a thread's own values
// in order, the lane quad (xor 1, 2), the warps in order.  Weighted sums: O_w = P_w . V_w with
// P split into two bf16 terms (about 16 significant bits), two 16-token steps in ascending
// order; the four warps' O_w are added in warp order.
template <int G>  // query heads per kv head (1, 2, 4 or 8)
__global__ void __launch_bounds__(kAttnThreads, 3)
    decode_attention_split_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                                  const __nv_bfloat16 *__restrict__ v, const int32_t *__restrict__ lens,
                                  float2 *__restrict__ part_ms, float *__restrict__ part_acc, int Hq, int Hkv,
                                  int64_t Lmax, float scale, int32_t *status)
{
    extern __shared__ __align__(16) uint8_t attn_raw[];
    AttnSmem &sm = *reinterpret_cast<AttnSmem *>(attn_raw);
    griddep_wait();  // the previous kernel's output (q, the caches, the lengths) is complete
    griddep_launch_dependents();
    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    const int64_t S = attn_splits(Lmax);
    int64_t L = lens[b];
    if (L < 1 || L > Lmax) {
        if (tid == 0) *reinterpret_cast<volatile int32_t *>(status) = 1;  // BI_ERR_INVALID_ARG
        L = L < 1 ? 1 : Lmax;
    }
    const int64_t t0 = (int64_t)split * kAttnSplit;
    if (t0 >= L) return;  // this split is past the sequence's end: it has no partial
    const int n_tok = (int)(L - t0 < kAttnSplit ? L - t0 : kAttnSplit);

    // Stage Q (rows >= G zero) and K in copy group 1, V in copy group 2 (16-byte async
    // copies; rows past the sequence zero-filled).  The scores wait for group 1 only.
    for (int c = tid; c < 16 * (kAttnD / 8); c += kAttnThreads) {
        const int j = c / (kAttnD / 8), col = (c % (kAttnD / 8)) * 8;
        const bool in = j < G;
        cp_async16(&sm.q[j][col], q + (in ? ((int64_t)b * Hq + (int64_t)g * G + j) * kAttnD + col : 0),
                   in ? 16u : 0u);
    }
    for (int c = tid; c < kAttnSplit * (kAttnD / 8); c += kAttnThreads) {
        const int row = c / (kAttnD / 8), col = (c % (kAttnD / 8)) * 8;
        const bool in = row < n_tok;
        const int64_t off = in ? (((int64_t)b * Lmax + t0 + row) * Hkv + g) * kAttnD + col : 0;
        cp_async16(&sm.ko.k[row][col], k + off, in ? 16u : 0u);
    }
    cp_async_commit();
    for (int c = tid; c < kAttnSplit * (kAttnD / 8); c += kAttnThreads) {
        const int row = c / (kAttnD / 8), col = (c % (kAttnD / 8)) * 8;
        const bool in = row < n_tok;
        const int64_t off = in ? (((int64_t)b * Lmax + t0 + row) * Hkv + g) * kAttnD + col : 0;
        cp_async16(&sm.v[row][col], v + off, in ? 16u : 0u);
    }
    cp_async_commit();
    cp_async_wait_pending<1>();
    __syncthreads();

    // ---- scores: acc[nt] is the 16 x 8 tile (heads x tokens 32w + 8nt ..)
    float acc[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < kAttnD / 16; ++kk) {
        uint32_t af[4];
        ldsm_x4(af, &sm.q[(lane & 7) + 8 * ((lane >> 3) & 1)][16 * kk + 8 * (lane >> 4)]);
#pragma unroll
        for (int nt = 0; nt < 4; nt += 2) {
            // matrices: (tile nt, d 0-7), (nt, d 8-15), (nt+1, d 0-7), (nt+1, d 8-15) of this step
            uint32_t bf[4];
            ldsm_x4(bf, &sm.ko.k[32 * warp + 8 * (nt + (lane >> 4)) + (lane & 7)][16 * kk + 8 * ((lane >> 3) & 1)]);
            mma_16816_bf16(acc[nt], af, bf[0], bf[1]);
            mma_16816_bf16(acc[nt + 1], af, bf[2], bf[3]);
        }
    }
    // scale and mask: element (row gid / gid+8, token 32w + 8nt + 2tig + {0,1})
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int tok = 32 * warp + 8 * nt + 2 * tig + (e & 1);
            acc[nt][e] = tok < n_tok ? acc[nt][e] * scale : kNegInf;
        }

    // ---- per-head max: own values in order, quad butterfly, warps in order
    float mx[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float m = acc[0][2 * h];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) m = fmaxf(fmaxf(m, acc[nt][2 * h]), acc[nt][2 * h + 1]);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        mx[h] = m;
    }
    if (tig == 0) {
        sm.red[warp][gid] = mx[0];
        sm.red[warp][gid + 8] = mx[1];
    }
    __syncthreads();
    if (tid < 16) {
        float m = sm.red[0][tid];
        for (int w = 1; w < kAttnWarps; ++w) m = fmaxf(m, sm.red[w][tid]);
        sm.stat[tid][0] = m;
    }
    __syncthreads();
    // ---- p = exp(s - max); per-head sums by the same trees
    float sum[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const float m = sm.stat[gid + 8 * h][0];
        float l = 0.0f;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float &x = acc[nt][2 * h + e];
                x = x == kNegInf ? 0.0f : __expf(x - m);
                l = __fadd_rn(l, x);
            }
        l = __fadd_rn(l, __shfl_xor_sync(0xffffffffu, l, 1));
        l = __fadd_rn(l, __shfl_xor_sync(0xffffffffu, l, 2));
        sum[h] = l;
    }
    __syncthreads();  // every warp has read sm.stat / sm.red
    if (tig == 0) {
        sm.red[warp][gid] = sum[0];
        sm.red[warp][gid + 8] = sum[1];
    }
    cp_async_wait_pending<0>();  // V has landed
    __syncthreads();
    if (tid < 16) {
        float l = sm.red[0][tid];
        for (int w = 1; w < kAttnWarps; ++w) l = __fadd_rn(l, sm.red[w][tid]);
        sm.stat[tid][1] = l;
    }

    // ---- O_w = P_w . V_w: A from the score tiles (two 8-token tiles per 16-token step)
    float o[kAttnD / 8][4];
#pragma unroll
    for (int dt = 0; dt < kAttnD / 8; ++dt)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[dt][e] = 0.0f;
    // P enters the tensor cores as two bf16 terms, hi = bf16(p) and lo = bf16(p - hi), so the
    // weights keep about 16 significant bits; per 16-token step the hi product is added first.
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const float *p0 = acc[2 * j], *p1 = acc[2 * j + 1];
        const float pv[8] = {p0[0], p0[1], p0[2], p0[3], p1[0], p1[1], p1[2], p1[3]};
        float hi[8], lo[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            hi[e] = __bfloat162float(__float2bfloat16_rn(pv[e]));
            lo[e] = pv[e] - hi[e];
        }
        const uint32_t pa_hi[4] = {pack_bf16(hi[0], hi[1]), pack_bf16(hi[2], hi[3]), pack_bf16(hi[4], hi[5]),
                                   pack_bf16(hi[6], hi[7])};
        const uint32_t pa_lo[4] = {pack_bf16(lo[0], lo[1]), pack_bf16(lo[2], lo[3]), pack_bf16(lo[4], lo[5]),
                                   pack_bf16(lo[6], lo[7])};
        const int tok0 = 32 * warp + 16 * j;
#pragma unroll
        for (int dt = 0; dt < kAttnD / 8; dt += 2) {
            // matrices (transposed): (tokens 0-7, d tile dt), (tokens 8-15, dt), (0-7, dt+1), (8-15, dt+1)
            uint32_t vf[4];
            ldsm_x4_trans(vf, &sm.v[tok0 + (lane & 7) + 8 * ((lane >> 3) & 1)][8 * (dt + (lane >> 4))]);
            mma_16816_bf16(o[dt], pa_hi, vf[0], vf[1]);
            mma_16816_bf16(o[dt], pa_lo, vf[0], vf[1]);
            mma_16816_bf16(o[dt + 1], pa_hi, vf[2], vf[3]);
            mma_16816_bf16(o[dt + 1], pa_lo, vf[2], vf[3]);
        }
    }
    __syncthreads();  // K is no longer read: its space holds the per-warp outputs
#pragma unroll
    for (int dt = 0; dt < kAttnD / 8; ++dt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int row = gid + 8 * (e >> 1), col = 8 * dt + 2 * tig + (e & 1);
            if (row < G) sm.ko.o[warp][row][col] = o[dt][e];
        }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < G; ++j) {
        float r = sm.ko.o[0][j][tid];
        for (int w = 1; w < kAttnWarps; ++w) r = __fadd_rn(r, sm.ko.o[w][j][tid]);
        const int64_t bh = (int64_t)b * Hq + (int64_t)g * G + j;
        part_acc[(bh * S + split) * kAttnD + tid] = r;
        if (tid == 0) part_ms[bh * S + split] = make_float2(sm.stat[j][0], sm.stat[j][1]);
    }
}

// Launch 2: grid (Hq, B), kAttnD threads.  Fold the sequence's splits in ascending order.
__global__ void __launch_bounds__(kAttnD)
    decode_attention_combine_kernel(const float2 *__restrict__ part_ms, const float *__restrict__ part_acc,
                                    const int32_t *__restrict__ lens, __nv_bfloat16 *__restrict__ out,
                                    int Hq, int64_t Lmax)
{
    griddep_wait();  // every split's partials are complete
    griddep_launch_dependents();
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
