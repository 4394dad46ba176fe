// attention.cuh -- batch-invariant decode attention (one query token per sequence).
//
// The key/value cache of a sequence is cut into splits of kAttnSplit tokens, a cut fixed
// by the sequence's own length.  Launch 1 produces, for every (split, kv head, sequence) and
// each query head of the kv head's group, the split's maximum score, its sum of
// exp(score - max) and the matching weighted sum of value rows.  Launch 2 folds the splits of
// each (sequence, query head) in ascending split order.  Every reduction is a fixed sequence
// or a fixed tree, so a sequence's output depends on its own query, cache and length only --
// not on the batch it is decoded in, its position there, or which CTA computes a split.  When
// Lmax <= kAttnSplit every sequence is one split, and launch 1 does launch 2's fold of it itself
// (the same operations on the same values), so launch 2 is not made.
//
// Launch 1 is a persistent, warp-specialised kernel: one CTA per SM walks the (split, kv head,
// sequence) work items round-robin.  Its producer warp stages each split as the group's query
// rows (bulk copies) and K and V tiles (4-D TMA tensor loads of 128 tokens x 64 d boxes, 128-byte
// swizzle) into a ring of kAttnStages shared-memory stages, each completing on mbarriers; a stage
// holds 128 tokens of head size 128, or 256 tokens (two pieces of 128) of head size 64.  Two
// groups of four consumer warps take the CTA's splits alternately, so one group's compute
// overlaps the other's and the loads of the next stages.  The cache streams from HBM without a
// gap between items.  A split of kAttnSplit tokens keeps the partial results (written by launch 1,
// read by launch 2) at a few percent of the cache's bytes.  The arithmetic of a split is fixed and
// does not depend on the ring, the group or the CTA.
//
// Layouts (row-major, bf16): q [B, Hq, D]; k, v [B, Lmax, Hkv, D]; out [B, Hq, D].  Query
// head h reads kv head h / (Hq / Hkv).  D = 128.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "rowops.cuh"

namespace bi {

constexpr int kAttnD = 128;                             // largest head size; shared memory is laid out for it
constexpr int kAttnChunk = 128;                         // tokens per ring stage
constexpr int kAttnSplit = 4 * kAttnChunk;              // tokens per split (one partial result)
constexpr int kAttnConsumers = 4;                       // consumer warps per group, 32 tokens of a stage each
constexpr int kAttnGroups = 2;                          // consumer groups, alternate splits
constexpr int kAttnThreads = 32 * (1 + kAttnGroups * kAttnConsumers);  // warp 0 produces
constexpr int kAttnMaxGroup = 8;                        // query heads per kv head
constexpr int kAttnStages = 3;
constexpr int kAttnQStride = kAttnD + 8;                // padded query row (bf16): conflict-free ldmatrix
constexpr int kAttnBoxBytes = kAttnChunk * 64 * 2;      // one TMA box: 128 tokens x 64 d (16 KB)
constexpr int kAttnTileBytes = 2 * kAttnBoxBytes;       // K or V of one split: 32 KB
constexpr int kAttnQBytes = 16 * kAttnQStride * 2;      // query rows of a group, padded to 16 rows
constexpr int kAttnStageBytes = 2 * kAttnTileBytes + ((kAttnQBytes + 1023) / 1024) * 1024;
constexpr int kAttnSmem = kAttnStages * kAttnStageBytes + 1024;  // + alignment slack

constexpr int kAttnOStride = kAttnD + 8;                // per-warp output rows in shared memory (floats)
static_assert(kAttnChunk == 32 * kAttnConsumers, "each consumer warp owns 32 token rows of a stage");
static_assert(kAttnConsumers * kAttnMaxGroup * kAttnOStride * 4 <= kAttnTileBytes,
              "per-warp partial outputs fit in the K tile they replace");

struct AttnParams {
    const __nv_bfloat16 *q;
    const int32_t *lens;
    float2 *part_ms;  // [B, Hq, S] (max, sum)
    float *part_acc;  // [B, Hq, S, D]
    __nv_bfloat16 *out;  // non-null when every sequence is one split (S = 1): launch 1 writes out
    int32_t Hq, Hkv, B;
    int64_t Lmax, S;  // S = splits of Lmax
    float scale;
    int32_t *status;
    uint64_t wait_limit_ns;
};

__host__ __device__ inline int64_t attn_splits(int64_t L) { return (L + kAttnSplit - 1) / kAttnSplit; }
// Ring stages of a split that starts `rest` tokens before the sequence's end (rest >= 1).
__host__ __device__ inline int attn_chunks(int64_t rest)
{
    return rest >= kAttnSplit ? kAttnSplit / kAttnChunk : (int)((rest + kAttnChunk - 1) / kAttnChunk);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&p);
}

// Shared-memory address of 16-byte chunk `chunk` (0..15) of token row `row` of a K or V tile as
// the TMA writes it: two boxes of 64 d each (chunks 0..7 and 8..15), rows of 128 bytes, with the
// 128-byte swizzle (chunk c of row r lands at chunk c ^ (r mod 8)).
__device__ __forceinline__ const uint8_t *kv_chunk(const uint8_t *tile, int row, int chunk)
{
    return tile + (chunk >> 3) * kAttnBoxBytes + row * 128 + (((chunk & 7) ^ (row & 7)) << 4);
}

constexpr int kAttnLensCached = 4096;  // sequence lengths launch 1 keeps in shared memory

// Sequence length as the kernels use it: a value outside 1 .. Lmax is clamped (and reported).
// `cached` holds lens[0 .. kAttnLensCached) when non-null.
__device__ __forceinline__ int64_t attn_len(const AttnParams &p, int b, bool report, const int32_t *cached = nullptr)
{
    int64_t L = cached && b < kAttnLensCached ? cached[b] : p.lens[b];
    if (L < 1 || L > p.Lmax) {
        if (report) *reinterpret_cast<volatile int32_t *>(p.status) = 1;  // BI_ERR_INVALID_ARG
        L = L < 1 ? 1 : p.Lmax;
    }
    return L;
}

// 4-D tiled TMA load (coordinates innermost first), completion on `bar`, with an L2 cache
// policy: the caches are read once, so their lines go first (evict-first), and what is to be read
// again soon -- the splits' partial results, which the combine launch reads -- stays in L2.
// (B200, L2 flushed, same bits: B=8 L=4096 38.8 us against 41.9 without the policy; B=64 L=4000
// 178.2 against 183.1; one 32768-token sequence 39.9 against 42.5; head size 64 at B=64 L=4096
// 103.4 against 107.5; B=64 L=4096 unchanged.)
__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, uint64_t *bar, int32_t c0,
                                            int32_t c1, int32_t c2, int32_t c3, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
        "l"(policy)
        : "memory");
}

// All threads of one consumer group (named barrier `id`, 128 threads): true iff every one passes
// `ok`.
__device__ __forceinline__ bool consumers_all(int id, bool ok)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %2, 0;\n\t"
        "barrier.red.and.pred q, %1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(id), "r"(ok ? 1u : 0u)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void consumers_sync(int id) { asm volatile("barrier.sync %0, 128;" ::"r"(id) : "memory"); }

// Bounded wait until *flag >= v (a shared-memory progress counter written by another warp).
// On time-out it records BI_ERR_TIMEOUT and raises the abort flag, like wait_bounded.
__device__ __forceinline__ bool wait_flag_at_least(volatile int *flag, int v, volatile int *abort_flag,
                                                   int32_t *status, uint64_t limit_ns)
{
    if (*flag >= v) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (*flag >= v) return true;
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > limit_ns) {
            *reinterpret_cast<volatile int32_t *>(status) = 5;  // BI_ERR_TIMEOUT
            *abort_flag = 1;
            return false;
        }
    }
}

// Launch 1: grid = min(work items, SMs) CTAs of kAttnThreads threads, kAttnSmem bytes of dynamic
// shared memory.  Work item i: for D = 128 kv head i % Hkv, split (i / Hkv) % S, sequence
// i / (Hkv S); for D = 64 split i % S, kv head (i / S) % Hkv, sequence i / (S Hkv).  Items past
// their sequence's length have no partial and are skipped by every role alike.
//
// Arithmetic per split (mma.sync m16n8k16, bf16 in, fp32 accumulate), over its pieces of
// kAttnChunk tokens in ascending order (one or two per ring stage, by the head size; the
// arithmetic is the same either way); warp w owns tokens 32w .. 32w+31 of each piece.  Scores:
// S = Q . K^T with Q the group's heads padded to 16 rows; every score accumulates its eight
// 16-wide D steps in ascending order.  Per head and piece, the piece's maximum comes from a fixed
// tree (a thread's own values in order, the lane quad xor 1, 2, the warps in order) and raises the
// running maximum m; what is accumulated so far -- each thread's sum of exp(s - m) and each warp's
// weighted sums -- is multiplied by exp(m_old - m) (0 at the first piece), then the piece's
// exp(s - m) are added in order.  Weighted sums: O_w^T += V_w^T . P_w^T with P split into two bf16
// terms (about 16 significant bits), two 16-token steps in ascending order.  At the split's end the
// threads' sums meet in the lane quad (xor 1, 2), then the four warps' sums and O_w are added in
// warp order.  Value rows past the sequence's end are zeroed in shared memory before use, so stale
// cache contents never reach the sums.
template <int G, int D>  // G query heads per kv head (1, 2, 4 or 8); head size D (64 or 128)
__global__ void __launch_bounds__(kAttnThreads, 1)
    decode_attention_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                                  const AttnParams p)
{
    static_assert(D == 64 || D == 128, "head size 64 or 128");
    // A K or V tile is two 64-d TMA boxes of 128 tokens.  D = 128: both halves of the same 128
    // tokens' rows.  D = 64: two consecutive 128-token pieces, so a stage carries as many bytes.
    constexpr int kPieces = D == 64 ? 2 : 1;            // 128-token pieces per stage
    extern __shared__ uint8_t attn_raw[];
    uint8_t *smem = attn_raw + ((1024u - (smem_addr(attn_raw) & 1023u)) & 1023u);
    __shared__ uint64_t kfull[kAttnStages], vfull[kAttnStages], empty[kAttnStages];
    __shared__ float red_m_all[kAttnGroups][kAttnConsumers][8];  // per-warp maxima of the 8 head rows
    __shared__ float red_s_all[kAttnGroups][kAttnConsumers][8];  // per-warp sums of exp
    __shared__ float mrun_all[kAttnGroups][8];                   // a split's running maxima, per head
    __shared__ int abort_flag_s;
    __shared__ int slot_use_s[kAttnStages];  // uses of each ring slot that a consumer group has passed
    // Every role walks all of the CTA's items and needs each one's sequence length: read once here
    // rather than from global memory per item.
    __shared__ int32_t lens_s[kAttnLensCached];
    volatile int *abort_flag = &abort_flag_s;
    volatile int *slot_use = slot_use_s;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto k_tile = [&](int s) { return smem + s * kAttnStageBytes; };
    auto v_tile = [&](int s) { return smem + s * kAttnStageBytes + kAttnTileBytes; };
    auto q_rows = [&](int s) { return reinterpret_cast<__nv_bfloat16 *>(smem + s * kAttnStageBytes + 2 * kAttnTileBytes); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kAttnStages; ++s) {
            mbar_init(&kfull[s], 1);
            mbar_init(&vfull[s], 1);
            mbar_init(&empty[s], kAttnConsumers);  // one arrival per consumer warp
        }
        abort_flag_s = 0;
        for (int st = 0; st < kAttnStages; ++st) slot_use_s[st] = 0;
        fence_mbar_init();
    }
    // Query rows G .. 15 of every stage stay zero (the copies fill rows 0 .. G-1 only).
    for (int i = threadIdx.x; i < kAttnStages * (16 - G) * kAttnQStride / 2; i += kAttnThreads) {
        const int s = i / ((16 - G) * kAttnQStride / 2), r = i % ((16 - G) * kAttnQStride / 2);
        reinterpret_cast<uint32_t *>(q_rows(s) + G * kAttnQStride)[r] = 0u;
    }
    fence_proxy_async_smem();
    __syncthreads();
    griddep_wait();  // the previous kernel's output (q, the caches, the lengths) is complete
    griddep_launch_dependents();
    for (int i = threadIdx.x; i < p.B && i < kAttnLensCached; i += kAttnThreads) lens_s[i] = p.lens[i];
    __syncthreads();

    // The host guarantees B * Hkv * S < 2^31, so item indices and their coordinates are 32-bit.
    const uint32_t items = (uint32_t)p.B * (uint32_t)p.Hkv * (uint32_t)p.S;
    const uint32_t n_splits = (uint32_t)p.S, n_kv = (uint32_t)p.Hkv;
    // Item order (a property of the head size, not of the batch; no item's arithmetic depends on
    // it): D = 128, kv head fastest, so the heads of the same tokens -- adjacent pieces of the same
    // cache rows -- are fetched by neighbouring CTAs at about the same time; D = 64, split fastest
    // (measured faster there).
    auto item_coords = [&](uint32_t it, int &split, int &g, int &b) {
        if (D == 128) {
            const uint32_t sg = it / n_kv;
            g = (int)(it - sg * n_kv);
            split = (int)(sg % n_splits);
            b = (int)(sg / n_splits);
        } else {
            const uint32_t sg = it / n_splits;
            split = (int)(it - sg * n_splits);
            g = (int)(sg % n_kv);
            b = (int)(sg / n_kv);
        }
    };
    const uint64_t lim = p.wait_limit_ns;

    if (warp == 0) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t kv_policy = l2_policy_evict_first();  // every cache byte is read once
            uint32_t stage = 0, phase = 0;
            int issued = 0;
            bool ok = true;
            for (uint32_t it = blockIdx.x; ok && it < items; it += gridDim.x) {
                int split, g, b;
                item_coords(it, split, g, b);
                const int64_t t0 = (int64_t)split * kAttnSplit, L = attn_len(p, b, false, lens_s);
                if (t0 >= L) continue;
                // The split's stages in token order; each carries the group's query rows too.
                const int nc = attn_chunks(L - t0), ns = (nc + kPieces - 1) / kPieces;
                for (int c = 0; c < ns; ++c) {
                    const int32_t tc = (int32_t)(t0 + (int64_t)c * kPieces * kAttnChunk);
                    if (!(ok = wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.status, lim))) break;
                    mbar_arrive_expect_tx(&kfull[stage], G * D * 2 + kAttnTileBytes);
                    for (int j = 0; j < G; ++j)
                        bulk_load(q_rows(stage) + j * kAttnQStride,
                                  p.q + ((int64_t)b * p.Hq + (int64_t)g * G + j) * D, D * 2, &kfull[stage]);
                    // Box x: d offset 64 x (D = 128), or tokens tc + 128 x (D = 64; past the sequence
                    // the box is loaded but never read).
#pragma unroll
                    for (int x = 0; x < 2; ++x)
                        tma_load_4d(k_tile(stage) + x * kAttnBoxBytes, &tm_k, &kfull[stage], kPieces == 1 ? 64 * x : 0, g,
                                    tc + (kPieces == 1 ? 0 : x * kAttnChunk), b, kv_policy);
                    mbar_arrive_expect_tx(&vfull[stage], kAttnTileBytes);
#pragma unroll
                    for (int x = 0; x < 2; ++x)
                        tma_load_4d(v_tile(stage) + x * kAttnBoxBytes, &tm_v, &vfull[stage], kPieces == 1 ? 64 * x : 0, g,
                                    tc + (kPieces == 1 ? 0 : x * kAttnChunk), b, kv_policy);
                    ++issued;
                    advance(stage, phase, kAttnStages);
                }
            }
            if (!ok) {
                // A wait ran out: let every copy already issued land before shared memory goes
                // away (the last kAttnStages stages at most).
                for (int j = issued > kAttnStages ? issued - kAttnStages : 0; j < issued; ++j) {
                    const uint32_t par = (uint32_t)(j / kAttnStages) & 1u;
                    const uint64_t t0 = global_timer_ns();
                    while ((!mbar_try_wait(smem_addr(&kfull[j % kAttnStages]), par) ||
                            !mbar_try_wait(smem_addr(&vfull[j % kAttnStages]), par)) &&
                           global_timer_ns() - t0 < lim) {
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------------------------ consumers
        // Group grp takes the CTA's splits with local index i = grp, grp + 2, ...  Stages are
        // numbered across all of the CTA's splits in producer order: stage number q sits in ring
        // slot q % kAttnStages, that slot's use q / kAttnStages.
        const int grp = (warp - 1) / kAttnConsumers;
        const int cw = (warp - 1) % kAttnConsumers, ct = threadIdx.x - 32 - 32 * kAttnConsumers * grp;
        const int bar_id = 1 + grp;
        const int gid = lane >> 2, tig = lane & 3;
        float (*red_m)[8] = red_m_all[grp];
        float (*red_s)[8] = red_s_all[grp];
        uint32_t local = 0, q0 = 0;  // the split's local index and its first stage number
        bool alive = true;
        for (uint32_t it = blockIdx.x; alive && it < items; it += gridDim.x) {
            int split, g, b;
            item_coords(it, split, g, b);
            const int64_t t0 = (int64_t)split * kAttnSplit;
            const int64_t L = attn_len(p, b, ct == 0 && grp == 0 && split == 0, lens_s);
            if (t0 >= L) continue;
            const int nc = attn_chunks(L - t0), ns = (nc + kPieces - 1) / kPieces;
            const uint32_t mine = local++, first = q0;
            q0 += (uint32_t)ns;
            if (mine % kAttnGroups != (uint32_t)grp) continue;

            // Per head (row gid of the score tiles): the running maximum over the split's stages so
            // far, and this thread's running sum of exp(s - m_run) over its tokens.  o holds this
            // warp's weighted sums O_w^T (d 16 mt + gid (+ 8), heads 2 tig and 2 tig + 1), scaled to
            // the same running maximum.
            float m_run = kNegInf, l_t = 0.0f;
            float o[D / 16][4];
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) o[mt][e] = 0.0f;
            int stage = 0;
            for (int c = 0; c < ns; ++c) {
                const uint32_t qn = first + (uint32_t)c;
                stage = (int)(qn % kAttnStages);
                const uint32_t use = qn / kAttnStages;
                const __nv_bfloat16 *qs = q_rows(stage);
                // Uses of a slot are passed in order: once the slot's previous use has been passed
                // (by either group), the slot's barriers are at most one phase from the one wanted,
                // so a parity wait is exact.  V is released with K, so the V wait needs no more.
                bool ok = wait_flag_at_least(&slot_use[stage], (int)use, abort_flag, p.status, lim);
                ok = ok && wait_bounded(&kfull[stage], use & 1u, abort_flag, p.status, lim);
                if (!consumers_all(bar_id, ok)) {
                    alive = false;
                    break;
                }
                if (ct == 0) slot_use[stage] = (int)use + 1;

              // The stage's 128-token pieces in token order (one for D = 128, two for D = 64); the
              // piece's K and V rows start at box hp of the tile.
              for (int hp = 0; hp < kPieces && c * kPieces + hp < nc; ++hp) {
                const int64_t tc = t0 + (int64_t)(c * kPieces + hp) * kAttnChunk;
                const int n_tok = (int)(L - tc < kAttnChunk ? L - tc : kAttnChunk);
                const uint8_t *ks = k_tile(stage) + hp * kAttnBoxBytes;
                uint8_t *vs = v_tile(stage) + hp * kAttnBoxBytes;

                // ---- scores: acc[nt] is the 16 x 8 tile (heads x tokens 32 cw + 8 nt ..)
                float acc[4][4];
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.0f;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    uint32_t af[4];
                    ldsm_x4(af, qs + ((lane & 7) + 8 * ((lane >> 3) & 1)) * kAttnQStride + 16 * kk + 8 * (lane >> 4));
#pragma unroll
                    for (int nt = 0; nt < 4; nt += 2) {
                        // matrices: (tile nt, d 0-7), (nt, d 8-15), (nt+1, d 0-7), (nt+1, d 8-15) of this step
                        uint32_t bf[4];
                        ldsm_x4(bf, kv_chunk(ks, 32 * cw + 8 * (nt + (lane >> 4)) + (lane & 7), 2 * kk + ((lane >> 3) & 1)));
                        mma_16816_bf16(acc[nt], af, bf[0], bf[1]);
                        mma_16816_bf16(acc[nt + 1], af, bf[2], bf[3]);
                    }
                }
                // scale and mask: element (row gid / gid+8, token 32 cw + 8 nt + 2 tig + {0,1})
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int tok = 32 * cw + 8 * nt + 2 * tig + (e & 1);
                        acc[nt][e] = tok < n_tok ? acc[nt][e] * p.scale : kNegInf;
                    }

                // ---- the stage's maximum per head: own values in order, quad butterfly, warps in
                // order.  Only rows 0..7 (e = 0, 1) hold heads; rows 8..15 are padding.
                {
                    float m = acc[0][0];
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt) m = fmaxf(fmaxf(m, acc[nt][0]), acc[nt][1]);
                    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
                    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
                    if (tig == 0) red_m[cw][gid] = m;
                }
                consumers_sync(bar_id);  // every warp's maxima are posted; the K tile is no longer read
                // ---- new running maximum, rescale what is accumulated, p = exp(s - m_new), sums.
                float alpha;
                {
                    float m_c = red_m[0][gid];
#pragma unroll
                    for (int w = 1; w < kAttnConsumers; ++w) m_c = fmaxf(m_c, red_m[w][gid]);
                    const float m_new = fmaxf(m_run, m_c);  // finite: the stage has a token
                    alpha = __expf(m_run - m_new);          // 0 for the first stage
                    m_run = m_new;
                    float l = __fmul_rn(l_t, alpha);
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            float &x = acc[nt][e];
                            x = x == kNegInf ? 0.0f : __expf(x - m_new);
                            l = __fadd_rn(l, x);
                        }
                    l_t = l;
                }
                {
                    // o's columns are heads 2 tig and 2 tig + 1, whose factors the lanes of rows
                    // gid = 2 tig (lane 8 tig) and 2 tig + 1 (lane 8 tig + 4) hold.
                    const float a0 = __shfl_sync(0xffffffffu, alpha, 8 * tig);
                    const float a1 = __shfl_sync(0xffffffffu, alpha, 8 * tig + 4);
#pragma unroll
                    for (int mt = 0; mt < D / 16; ++mt) {
                        o[mt][0] = __fmul_rn(o[mt][0], a0);
                        o[mt][1] = __fmul_rn(o[mt][1], a1);
                        o[mt][2] = __fmul_rn(o[mt][2], a0);
                        o[mt][3] = __fmul_rn(o[mt][3], a1);
                    }
                }
                if (hp == 0 && !consumers_all(bar_id, wait_bounded(&vfull[stage], use & 1u, abort_flag, p.status, lim))) {
                    alive = false;
                    break;
                }
                if (n_tok < kAttnChunk) {
                    // Value rows past the sequence's end: zero, whatever the cache holds there.
                    for (int i = ct; i < (kAttnChunk - n_tok) * (D / 8); i += 32 * kAttnConsumers)
                        *reinterpret_cast<uint4 *>(const_cast<uint8_t *>(kv_chunk(vs, n_tok + i / (D / 8), i % (D / 8)))) =
                            make_uint4(0u, 0u, 0u, 0u);
                    consumers_sync(bar_id);
                }

                // ---- O_w^T += V_w^T . P_w^T: d on the MMA's M (8 tiles of 16 rows), the group's heads
                // on N (8 columns; columns G .. 7 are padding), tokens on K in two 16-token steps in
                // ascending order.  Rows 0..7 of the score tiles (e = 0, 1: head gid, tokens 2 tig and
                // 2 tig + 1 of tiles 2j and 2j + 1) are exactly the B fragments of P^T for step j, and
                // the transposed ldmatrix of V yields the A fragments of V^T, so nothing is reshuffled.
                // P enters as two bf16 terms, hi = bf16(p) and lo = bf16(p - hi), so the weights keep
                // about 16 significant bits; per 16-token step hi is added first.
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const float pv[4] = {acc[2 * j][0], acc[2 * j][1], acc[2 * j + 1][0], acc[2 * j + 1][1]};
                    float hi[4], lo[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        hi[e] = __bfloat162float(__float2bfloat16_rn(pv[e]));
                        lo[e] = pv[e] - hi[e];
                    }
                    const uint32_t pb_hi0 = pack_bf16(hi[0], hi[1]), pb_hi1 = pack_bf16(hi[2], hi[3]);
                    const uint32_t pb_lo0 = pack_bf16(lo[0], lo[1]), pb_lo1 = pack_bf16(lo[2], lo[3]);
                    const int tok0 = 32 * cw + 16 * j;
#pragma unroll
                    for (int dt = 0; dt < D / 8; dt += 2) {
                        // matrices (transposed): (tokens 0-7, d tile dt), (8-15, dt), (0-7, dt+1),
                        // (8-15, dt+1); as A of V^T (rows d, columns tokens): a0 = (dt, 0-7),
                        // a1 = (dt+1, 0-7), a2 = (dt, 8-15), a3 = (dt+1, 8-15).
                        uint32_t vf[4];
                        ldsm_x4_trans(vf, kv_chunk(vs, tok0 + (lane & 7) + 8 * ((lane >> 3) & 1), dt + (lane >> 4)));
                        const uint32_t va[4] = {vf[0], vf[2], vf[1], vf[3]};
                        mma_16816_bf16(o[dt / 2], va, pb_hi0, pb_hi1);
                        mma_16816_bf16(o[dt / 2], va, pb_lo0, pb_lo1);
                    }
                }
              }
                if (!alive) break;
                if (c + 1 < ns) {
                    // Release the stage, one arrival per warp: the generic-proxy writes into it
                    // (zeroed rows) are ordered before the next TMA writes.
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[stage]);
                }
            }
            if (!alive) break;

            // ---- the split's partial result.  The last stage's K tile (read by every warp before
            // that stage's maxima barrier) holds the per-warp outputs, rows kAttnOStride floats
            // apart: a store's lanes cover d 16 mt + gid (+ 8) of heads 2 tig (+ 1); for up to four
            // heads, rows 0 and 2 (or 1 and 3) sit 16 banks apart, so the 16 lanes that store land in
            // distinct banks; eight heads share banks two ways.  The running maxima and the warps'
            // sums go to arrays that nothing else reads before the barrier below.
            float *so = reinterpret_cast<float *>(const_cast<uint8_t *>(k_tile(stage)));
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int head = 2 * tig + (e & 1), col = 16 * mt + gid + 8 * (e >> 1);
                    if (head < G) so[(cw * kAttnMaxGroup + head) * kAttnOStride + col] = o[mt][e];
                }
            {
                float l = __fadd_rn(l_t, __shfl_xor_sync(0xffffffffu, l_t, 1));
                l = __fadd_rn(l, __shfl_xor_sync(0xffffffffu, l, 2));
                if (tig == 0) red_s[cw][gid] = l;
                if (tig == 0 && cw == 0) mrun_all[grp][gid] = m_run;
            }
            consumers_sync(bar_id);
#pragma unroll
            for (int j = 0; j < G; ++j) {
                const int64_t bh = (int64_t)b * p.Hq + (int64_t)g * G + j;
                if (ct < D) {  // thread ct sums column d = ct over the warps, in warp order
                    float r = so[j * kAttnOStride + ct];
                    for (int w = 1; w < kAttnConsumers; ++w)
                        r = __fadd_rn(r, so[(w * kAttnMaxGroup + j) * kAttnOStride + ct]);
                    if (p.out != nullptr) {
                        // Every sequence is one split: the combine launch's fold of one split,
                        // here, with the same operations on the same values (so the same bits).
                        float l = red_s[0][j];
                        for (int w = 1; w < kAttnConsumers; ++w) l = __fadd_rn(l, red_s[w][j]);
                        const float m = mrun_all[grp][j];
                        const float wt = __expf(m - m);
                        p.out[bh * D + ct] = __float2bfloat16_rn(fmaf(r, wt, 0.0f) / fmaf(l, wt, 0.0f));
                    } else {
                        p.part_acc[(bh * p.S + split) * D + ct] = r;
                    }
                }
                if (ct == 0 && p.out == nullptr) {
                    float l = red_s[0][j];
                    for (int w = 1; w < kAttnConsumers; ++w) l = __fadd_rn(l, red_s[w][j]);
                    p.part_ms[bh * p.S + split] = make_float2(mrun_all[grp][j], l);
                }
            }
            // Release the last stage, one arrival per warp: the generic-proxy writes into it
            // (partial outputs, zeroed rows) are ordered before the next TMA writes.
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
        }
    }
    __syncthreads();
}

// Launch 2: grid (Hq, B), D threads (one per column of the head).  Fold the sequence's splits
// in ascending order.  The splits' maximum is exact in any order, so the block takes it in parallel; the weights
// w_s = exp(m_s - max) and the split sums go to shared memory a chunk at a time, and each thread
// folds l += sum_s w_s and o += acc_s w_s in ascending s with its value loads issued ahead.
template <int D>
__global__ void __launch_bounds__(D)
    decode_attention_combine_kernel(const float2 *__restrict__ part_ms, const float *__restrict__ part_acc,
                                    const int32_t *__restrict__ lens, __nv_bfloat16 *__restrict__ out,
                                    int Hq, int64_t Lmax)
{
    constexpr int kCombineChunk = D;  // splits whose weights are staged at a time
    __shared__ float w_s[kCombineChunk], l_s[kCombineChunk], red[D / 32];
    griddep_wait();  // every split's partials are complete
    griddep_launch_dependents();
    const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
    const int64_t S = attn_splits(Lmax);
    int64_t L = lens[b];
    L = L < 1 ? 1 : (L > Lmax ? Lmax : L);
    const int64_t n = attn_splits(L);
    const int64_t bh = (int64_t)b * Hq + h;
    const float2 *ms = part_ms + bh * S;
    const float *acc = part_acc + bh * S * D + d;
    float m = kNegInf;
    for (int64_t s = d; s < n; s += D) m = fmaxf(m, ms[s].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((d & 31) == 0) red[d >> 5] = m;
    __syncthreads();
    m = red[0];
#pragma unroll
    for (int w = 1; w < D / 32; ++w) m = fmaxf(m, red[w]);
    float l = 0.0f, o = 0.0f;
    for (int64_t s0 = 0; s0 < n; s0 += kCombineChunk) {
        const int cnt = (int)(n - s0 < kCombineChunk ? n - s0 : kCombineChunk);
        __syncthreads();  // the previous chunk's weights have been read
        if (d < cnt) {
            const float2 v = ms[s0 + d];
            w_s[d] = __expf(v.x - m);
            l_s[d] = v.y;
        }
        __syncthreads();
        int j = 0;
        for (; j + 8 <= cnt; j += 8) {
            float a[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) a[u] = acc[(s0 + j + u) * D];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                l = fmaf(l_s[j + u], w_s[j + u], l);
                o = fmaf(a[u], w_s[j + u], o);
            }
        }
        for (; j < cnt; ++j) {
            l = fmaf(l_s[j], w_s[j], l);
            o = fmaf(acc[(s0 + j) * D], w_s[j], o);
        }
    }
    out[bh * D + d] = __float2bfloat16_rn(o / l);
}

}  // namespace bi
