// gemm_pair.cuh -- the batch-invariant bf16 GEMM: tcgen05 on CTA pairs (cta_group::2).
//
// A CTA pair (a 2-CTA cluster on one TPC) owns a 256 x BN output tile.  Each CTA stages,
// per pipeline stage of SK values of K, its own 128 rows of A and its own BN/2 rows
// (columns of C) of B; the leader CTA issues tcgen05.mma.cta_group::2 (M = 256, N = BN,
// K = 16), which reads both CTAs' shared memory and accumulates each CTA's 128 x BN half
// of the tile in fp32 in that CTA's tensor memory.  Per output element the order is the
// same as for any single tcgen05 MMA: the first 16-wide K step overwrites the
// accumulator, every later step adds in ascending K.  It depends only on K -- not on M,
// N, the row's position, or which pair computes the tile.  No split-K, no stream-K.
//
// Three instantiations exist, and the host picks one from the weight's number of rows
// alone (never from M; pair_config below): the wide tile (BN = 256, SK = 64), the 192-column
// tile (BN = 192, SK = 128) where its smaller tiles fill the GPU's CTA pairs in fewer
// cost-weighted waves, and for weights of up to 1024 rows the narrow tile (BN = 128,
// SK = 128), whose more numerous tiles fill more of the GPU.  Eight MMAs per 128-deep stage
// amortise the issuing thread's per-stage barrier wait and commit at the narrower widths.  All
// run the same 16-wide K steps in the same order, so a row's bits do not depend on which one
// ran (the tests compare them).
//
// Pipeline, per CTA pair:
//   full[s]   (leader)  armed by the leader's producer with both CTAs' bytes; both
//                       CTAs' TMA loads complete on it.
//   empty[s]  (both)    the leader's MMA commit, multicast to both CTAs, frees stage s.
//   tfull[b]  (both)    the leader's commit after a tile's last MMA: accumulator b ready.
//   tempty[b] (leader)  one arrival per epilogue warp of both CTAs: accumulator b drained.
// TMA loads are plain tiled loads (no cluster multicast); only the tcgen05.commit
// arrivals are multicast.
//
// Warp roles (192 threads per CTA): warp 0 TMA producer lane, warp 1 TMEM owner (both
// CTAs) and MMA issuer (leader only), warps 2..5 epilogue.  Every wait is bounded.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "gemm.cuh"
#include "ptx.cuh"

namespace bi {

constexpr int kPairBM = 256;  // rows of C per CTA pair

// Shared-memory layout of one tile configuration.  A stage holds SK / 64 swizzle atoms
// (64 values of K, 128 bytes per row) of A and of B.
template <int BN, int SK>
struct PairTile {
    static constexpr int kBN = BN;                      // columns of C per CTA pair
    static constexpr int kHalf = BN / 2;                // B rows staged by each CTA
    static constexpr int kStageK = SK;                  // K per pipeline stage
    static constexpr int kAtoms = SK / kBK;             // 64-wide K atoms per stage
    static constexpr int kAAtom = 128 * kBK * 2;        // one atom of A per CTA
    static constexpr int kBAtom = kHalf * kBK * 2;      // one atom of B ([N, K] storage) per CTA
    static constexpr int kABytes = kAtoms * kAAtom;     // A slice per CTA per stage
    static constexpr int kBBytes = kAtoms * kBAtom;     // B slice per CTA per stage
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStagesRaw = (kSmemBudget - kSmemMisc) / kStageBytes;
    static constexpr int kStages = kStagesRaw > 12 ? 12 : kStagesRaw;
    static constexpr int kSmem = kStages * kStageBytes + kSmemMisc;
    static constexpr uint32_t kTmemCols = pow2_at_least(2 * BN);

    static_assert(BN % 64 == 0 && BN <= 256, "pair tile N: a multiple of 64 up to 256");
    static constexpr bool kKNOk = kHalf % 64 == 0;   // [K, N] B is staged in 64-column groups
    static_assert(SK % kBK == 0 && SK >= kBK, "a stage holds whole swizzle atoms");
    static_assert(kStages >= 2 && kStages <= 32, "two to 32 stages (one producer lane per stage at the tail)");
    static_assert(kSmem + 1024 <= 256 * 1024, "shared addresses fit the 14-bit descriptor address field");
    static_assert(kTmemCols <= 512, "accumulators must fit in tensor memory");
    static_assert(kSmem > 114 * 1024, "one CTA per SM keeps the TMEM allocation uncontended");
};

using WideTile = PairTile<256, 64>;     // 7 stages of 64 K
using MidTile = PairTile<192, 128>;     // 4 stages of 128 K ([N, K] weights only)
using NarrowTile = PairTile<128, 128>;  // 4 stages of 128 K
constexpr int64_t kNarrowMaxN = 1024;   // weights of up to this many rows use NarrowTile

// Which configuration a weight runs, from its number of rows R alone (N of a plain product, 2F
// of the fused gate/up product; either way a tile row of 256 outputs needs ceil(R / BN) tiles):
// NarrowTile up to kNarrowMaxN rows; above that MidTile if, for a reference batch of 1024 rows
// (4 tile rows) on the B200's 74 CTA pairs, its waves of tiles weighted by the measured cost of a
// 192-column wave (0.8 of a 256-column one: 20.6 against 25.7 us per LM-head wave) come out
// fewer than WideTile's, else WideTile.  [K, N] weights, staged in 64-column groups per CTA, take
// WideTile where the rule says MidTile.  The rule never sees M, and every configuration takes the
// same 16-wide K steps in ascending order, so the choice does not change a bit of the result.
enum PairConfig { kPairNarrow = 0, kPairMid = 1, kPairWide = 2 };
constexpr int64_t kRefPairs = 74, kRefTileRows = 4;
__host__ inline PairConfig pair_config(int64_t weight_rows, bool nk)
{
    if (weight_rows <= kNarrowMaxN) return kPairNarrow;
    if (!nk) return kPairWide;
    auto waves = [&](int64_t bn) { return (kRefTileRows * ((weight_rows + bn - 1) / bn) + kRefPairs - 1) / kRefPairs; };
    return 4 * waves(MidTile::kBN) < 5 * waves(WideTile::kBN) ? kPairMid : kPairWide;
}

template <int BN, int SK>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_pair_kernel(const __grid_constant__ CUtensorMap tm_a,
                          const __grid_constant__ CUtensorMap tm_b, const GemmParams p)
{
    using T = PairTile<BN, SK>;
    constexpr int kPairBN = T::kBN, kHalfBN = T::kHalf, kPStages = T::kStages;
    constexpr int kPABytes = T::kABytes, kPBBytes = T::kBBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint8_t *sA = smem;
    uint8_t *sB = smem + kPStages * kPABytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(sB + kPStages * kPBBytes);
    uint64_t *empty = full + kPStages;
    uint64_t *tfull = empty + kPStages;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 2 * 4);  // one arrival per epilogue warp of both CTAs
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensor_map(&tm_a);
        prefetch_tensor_map(&tm_b);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_holder, T::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA signal
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;
    // Everything above touched only this cluster's shared and tensor memory; global memory is
    // read and written only after the previous kernel in the stream has completed.
    griddep_wait();
    griddep_launch_dependents();

    // Fused SiLU * up: a pair tile yields kHalfBN columns of h; CTA 0 stages gate rows
    // n0 .. n0 + kHalfBN - 1 and CTA 1 the up rows F + n0 .., so each CTA's accumulator holds gate
    // in columns [0, kHalfBN) and up in [kHalfBN, kPairBN) for its 128 rows.
    const int out_cols = p.fuse_silu ? kHalfBN : kPairBN;
    const int m_blocks = (p.M + kPairBM - 1) / kPairBM;
    const int n_blocks = (p.N + out_cols - 1) / out_cols;
    const int num_tiles = m_blocks * n_blocks;
    const int first = (int)cluster_id_x(), stride = (int)num_clusters_x();
    const uint64_t lim = p.wait_limit_ns;

    if (warp == 0) {
        uint32_t stage = 0, phase = 0;
        bool ok = true;
        if (lane == 0) {
            // ---------------------------------------------------------- TMA producer (both CTAs)
            for (int tile = first; ok && tile < num_tiles; tile += stride) {
                const int m_pair = (tile % m_blocks) * kPairBM;
                const int m0 = m_pair + 128 * (int)rank;
                const int nh0 = p.fuse_silu ? (tile / m_blocks) * kHalfBN + (rank ? p.N : 0)
                                            : (tile / m_blocks) * kPairBN + kHalfBN * (int)rank;
                // A rows are copied only where they exist: the box holds p.a_box_rows rows (M
                // rounded up to 8, at most 128), and the second CTA's half is not copied at all
                // when no row of it is below M.  Shared-memory rows left uncopied feed only
                // accumulator rows at or beyond M, which are never stored.
                const bool a_hi = m_pair + 128 < p.M;
                const uint32_t a_bytes = (uint32_t)p.a_box_rows * (SK * 2);
                const uint32_t stage_bytes = (a_hi ? 2u : 1u) * a_bytes + 2u * kPBBytes;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.status, lim)) {
                        ok = false;
                        break;
                    }
                    if (leader) mbar_arrive_expect_tx(&full[stage], stage_bytes);
                    const uint32_t bar = map_to_rank(smem_addr(&full[stage]), 0);
                    const int k0 = kb * SK;
                    if (leader || a_hi) {
#pragma unroll
                        for (int at = 0; at < T::kAtoms; ++at)
                            tma_load_2d_pair(sA + stage * kPABytes + at * T::kAAtom, &tm_a, bar, k0 + at * kBK, m0);
                    }
                    uint8_t *dstB = sB + stage * kPBBytes;
                    if (p.b_mn_major) {
                        // [K, N] storage: one box of 64 columns x SK values of K per 64-column group.
#pragma unroll
                        for (int g = 0; g < kHalfBN / 64; ++g)
                            tma_load_2d_pair(dstB + g * (64 * SK * 2), &tm_b, bar, nh0 + g * 64, k0);
                    } else {
#pragma unroll
                        for (int at = 0; at < T::kAtoms; ++at)
                            tma_load_2d_pair(dstB + at * T::kBAtom, &tm_b, bar, k0 + at * kBK, nh0);
                    }
                    advance(stage, phase, kPStages);
                }
            }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        stage = __shfl_sync(0xffffffffu, stage, 0);
        phase = __shfl_sync(0xffffffffu, phase, 0);
        if (ok) {
            // Tail: every stage released by the leader's MMA, so no multicast arrival is still
            // on its way to this CTA when it exits.  Lane j waits for the j-th stage after the
            // last one filled (the same barriers and parities a sequential walk would take); a
            // wait that completes still costs a few hundred cycles, so the lanes take them at once.
            if (lane < kPStages) {
                const uint32_t j = stage + (uint32_t)lane;
                const uint32_t st = j < (uint32_t)kPStages ? j : j - kPStages;
                const uint32_t ph = j < (uint32_t)kPStages ? phase : phase ^ 1u;
                wait_bounded(&empty[st], ph ^ 1u, abort_flag, p.status, lim);
            }
            __syncwarp();
        } else if (lane == 0) {
            // Abort: loads already issued complete on the leader's barrier, which this CTA
            // cannot observe; give them a bounded grace period to land.
            const uint64_t t0 = global_timer_ns();
            while (global_timer_ns() - t0 < 2000000ull) {
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ---------------------------------------------------------- MMA issuer (leader)
            const uint32_t idesc = mma_idesc_bf16(kPairBM, kPairBN, 0u, p.b_mn_major ? 1u : 0u);
            // Descriptors of stage 0's first K step.  A stage or a K step moves only the start
            // address field (address / 16 in the low 14 bits; every shared address of this CTA
            // fits, so the sum never carries into the next field): one add per MMA instead of a
            // descriptor rebuilt on the issuing thread's critical path.
            const uint64_t a_desc0 = sw128_desc(smem_addr(sA), 16, 1024);
            const uint64_t b_desc0 = p.b_mn_major ? sw128_desc(smem_addr(sB), 64 * SK * 2, 1024)
                                                  : sw128_desc(smem_addr(sB), 16, 1024);
            const bool b_mn = p.b_mn_major != 0;
            uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
            bool ok = true;
            for (int tile = first; ok && tile < num_tiles; tile += stride) {
                if (!wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, p.status, lim)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + acc * kPairBN;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!wait_bounded(&full[stage], phase, abort_flag, p.status, lim)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint64_t a_desc = a_desc0 + stage * (uint32_t)(kPABytes >> 4);
                    const uint64_t b_desc = b_desc0 + stage * (uint32_t)(kPBBytes >> 4);
#pragma unroll
                    for (int kk = 0; kk < SK / kMmaK; ++kk) {
                        // K step kk: atom kk / 4, 32-byte column (kk % 4) of its 128-byte rows;
                        // [K, N] storage advances 16 rows of 128 bytes instead.
                        constexpr int kPerAtom = kBK / kMmaK;
                        const uint32_t in_atom = (kk % kPerAtom) * ((kMmaK * 2) >> 4);
                        const uint32_t a_off = (kk / kPerAtom) * (T::kAAtom >> 4) + in_atom;
                        const uint32_t b_off =
                            b_mn ? kk * ((kMmaK * 128) >> 4) : (kk / kPerAtom) * (T::kBAtom >> 4) + in_atom;
                        tc_mma_bf16_pair(d_tmem, a_desc + a_off, b_desc + b_off, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit_pair_mc(&empty[stage], 0x3);
                    advance(stage, phase, kPStages);
                }
                if (!ok) break;
                tc_commit_pair_mc(&tfull[acc], 0x3);
                advance(acc, acc_phase, 2);
            }
            if (!ok) {
                tc_commit_pair_mc(drain, 0x1);
                const uint32_t a = smem_addr(drain);
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(a, 0) && global_timer_ns() - t0 < lim) {
                }
            }
        }
    } else {
        // -------------------------------------------------------------- epilogue (both CTAs)
        const int quarter = warp & 3;
        const int row_in_half = quarter * 32 + lane;
        const uint32_t tempty_leader0 = map_to_rank(smem_addr(&tempty[0]), 0);
        uint32_t acc = 0, acc_phase = 0;
        for (int tile = first; tile < num_tiles; tile += stride) {
            const bool ready = wait_bounded(&tfull[acc], acc_phase, abort_flag, p.status, lim);
            if (!__all_sync(0xffffffffu, ready)) break;
            tc_fence_after_sync();
            const int64_t row = (int64_t)(tile % m_blocks) * kPairBM + 128 * rank + row_in_half;
            const int64_t n0 = (int64_t)(tile / m_blocks) * out_cols;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * kPairBN;
#pragma unroll 1
            for (int c = 0; p.fuse_silu && c < kHalfBN / 32; ++c) {
                uint32_t rg[32], ru[32];
                tmem_load_32x32(t_row + c * 32, rg);
                tmem_load_32x32(t_row + kHalfBN + c * 32, ru);
                tmem_wait_ld();
                const int64_t col0 = n0 + c * 32;
                if (row < p.M && col0 < p.N) {
                    float gv[32], uv[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        gv[j] = __uint_as_float(rg[j]);
                        uv[j] = __uint_as_float(ru[j]);
                    }
                    store_silu_chunk(p, row, col0, gv, uv);
                }
            }
#pragma unroll 1
            for (int c = 0; !p.fuse_silu && c < kPairBN / 32; ++c) {
                uint32_t r[32];
                tmem_load_32x32(t_row + c * 32, r);
                tmem_wait_ld();
                const int64_t col0 = n0 + c * 32;
                if (row < p.M && col0 < p.N) {
                    float v[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
                    const bool full_chunk = col0 + 32 <= p.N;
                    add_addend(p, row, col0, full_chunk, v);
                    store_row_chunk(p, row, col0, full_chunk, v);
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty_leader0 + acc * sizeof(uint64_t));
            advance(acc, acc_phase, 2);
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    cluster_sync_all();  // no CTA leaves while its peer may still signal its barriers
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem_base, T::kTmemCols);
    }
}

}  // namespace bi
