// gemm.cuh -- the batch-invariant bf16 GEMM for sm_100a: C = A . B (+ input).
//
// One tile configuration for every call: a 128 x BN output tile per CTA, K sliced
// 64 at a time into a ring of shared-memory stages by TMA, multiplied by tcgen05.mma
// (M = 128, N = BN, K = 16 per instruction) into an fp32 accumulator in tensor
// memory, and read back by four epilogue warps.  Each output element therefore sums
// its K products in one order that depends only on K: 16-wide tensor-core steps in
// ascending K, the first overwriting the accumulator.  The tile shape, the K slicing
// and the instruction sequence never change with M, N or the position of a row in
// the batch; there is no split-K or stream-K, so no partial sums ever meet across
// CTAs.  Rows past M and columns past N/K are zero-filled by TMA and never stored.
//
// Persistent schedule: gridDim.x CTAs (at most one per SM) walk the tile list with
// stride gridDim.x.  The tensor-memory accumulator is double-buffered, so the
// epilogue of one tile overlaps the main loop of the next.  Which CTA computes a tile
// does not affect its arithmetic.
//
// Warp roles (192 threads):
//   warp 0      TMA producer (one lane)
//   warp 1      TMEM owner + MMA issuer (one lane)
//   warps 2..5  epilogue: TMEM -> registers -> (+ bias / residual) -> global
//
// Every wait on an mbarrier is bounded.  A wait that runs out records a timeout in
// the device status word and raises a shared abort flag; every role then leaves its
// loop, outstanding TMA loads and MMAs are drained (again with a bound), TMEM is
// freed and the kernel returns.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

#ifndef BI_GEMM_BN
#define BI_GEMM_BN 256
#endif

namespace bi {

constexpr int kBM = 128;
constexpr int kBN = BI_GEMM_BN;
constexpr int kBK = 64;          // one 128-byte swizzle row of bf16
constexpr int kMmaK = 16;        // K of one tcgen05.mma kind::f16
constexpr int kGemmThreads = 192;
constexpr int kABytes = kBM * kBK * 2;
constexpr int kBBytes = kBN * kBK * 2;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kSmemBudget = 227 * 1024;
constexpr int kSmemMisc = 1024 /*alignment slack*/ + 512 /*barriers, flags*/;
constexpr int kStagesRaw = (kSmemBudget - kSmemMisc) / kStageBytes;
constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
constexpr int kGemmSmem = kStages * kStageBytes + kSmemMisc;
constexpr uint32_t pow2_at_least(uint32_t v, uint32_t p = 32) { return p >= v ? p : pow2_at_least(v, p * 2); }
constexpr uint32_t kTmemCols = pow2_at_least(2 * kBN);

static_assert(kBN % 32 == 0 && kBN >= 32 && kBN <= 256, "tile N must be a multiple of 32 in [32, 256]");
static_assert(kBN % 64 == 0, "the [K, N] operand is loaded as 64-column boxes");
static_assert(kStages >= 2, "need at least two pipeline stages");
static_assert(kTmemCols <= 512, "accumulators must fit in tensor memory");
static_assert(kGemmSmem > 114 * 1024, "one CTA per SM keeps the TMEM allocation uncontended");

enum AddendMode : int { kAddNone = 0, kAddBias = 1, kAddMatrix = 2 };

struct GemmParams {
    int32_t M, N, K;
    int32_t m_blocks, n_blocks, k_blocks;
    int32_t b_mn_major;     // 1: B stored [K, N] (MN-major operand); 0: B stored [N, K]
    int32_t c_f32;          // 1: C is fp32; 0: C is bf16
    int32_t addend_mode;    // AddendMode
    int64_t ldc;
    int64_t ld_addend;
    void *C;
    const __nv_bfloat16 *addend;
    int32_t *status;        // device status word
    uint64_t wait_limit_ns;
};

// Bounded wait on (bar, parity).  Returns false if the wait ran out (after recording
// the timeout and raising the abort flag) or if another role already aborted.
__device__ __forceinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                             int32_t *status, uint64_t limit_ns)
{
    const uint32_t a = smem_addr(bar);
    if (mbar_try_wait(a, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(a, parity)) return true;
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > limit_ns) {
            *reinterpret_cast<volatile int32_t *>(status) = 5;  // BI_ERR_TIMEOUT
            *abort_flag = 1;
            return false;
        }
    }
}

__device__ __forceinline__ void advance(uint32_t &idx, uint32_t &phase, uint32_t n)
{
    if (++idx == n) {
        idx = 0;
        phase ^= 1u;
    }
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) { return __uint_as_float(b16 << 16); }

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi)
{
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&p);
}

// Add the bias / residual to 32 accumulator values of one row (columns col0..col0+31).
__device__ __forceinline__ void add_addend(const GemmParams &p, int64_t row, int64_t col0, bool full,
                                           float (&v)[32])
{
    if (p.addend_mode == kAddNone) return;
    const __nv_bfloat16 *src =
        p.addend_mode == kAddBias ? p.addend + col0 : p.addend + row * p.ld_addend + col0;
    if (full) {
        const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 u = __ldg(s4 + q);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                v[q * 8 + 2 * k] += bf16_bits_to_f32(w[k] & 0xffffu);
                v[q * 8 + 2 * k + 1] += bf16_bits_to_f32(w[k] >> 16);
            }
        }
    } else {
        for (int j = 0; j < 32 && col0 + j < p.N; ++j) v[j] += __bfloat162float(src[j]);
    }
}

__device__ __forceinline__ void store_row_chunk(const GemmParams &p, int64_t row, int64_t col0,
                                                bool full, const float (&v)[32])
{
    if (p.c_f32) {
        float *dst = reinterpret_cast<float *>(p.C) + row * p.ldc + col0;
        if (full) {
            float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                d4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        } else {
            for (int j = 0; j < 32 && col0 + j < p.N; ++j) dst[j] = v[j];
        }
    } else {
        __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(p.C) + row * p.ldc + col0;
        if (full) {
            uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                d4[q] = make_uint4(pack2_bf16(v[8 * q], v[8 * q + 1]), pack2_bf16(v[8 * q + 2], v[8 * q + 3]),
                                   pack2_bf16(v[8 * q + 4], v[8 * q + 5]),
                                   pack2_bf16(v[8 * q + 6], v[8 * q + 7]));
        } else {
            for (int j = 0; j < 32 && col0 + j < p.N; ++j) dst[j] = __float2bfloat16_rn(v[j]);
        }
    }
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_tcgen05_kernel(const __grid_constant__ CUtensorMap tm_a,
                             const __grid_constant__ CUtensorMap tm_b, const GemmParams p)
{
    extern __shared__ uint8_t smem_raw[];
    // 128-byte swizzle atoms need 1024-byte aligned stage buffers (shared-window offset).
    uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint8_t *sA = smem;
    uint8_t *sB = smem + kStages * kABytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(sB + kStages * kBBytes);
    uint64_t *empty = full + kStages;
    uint64_t *tfull = empty + kStages;   // [2] accumulator ready for the epilogue
    uint64_t *tempty = tfull + 2;        // [2] accumulator drained by the epilogue
    uint64_t *drain = tempty + 2;        // [1] used only when aborting
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4 * 32);
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
        tmem_alloc(tmem_holder, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;

    const int num_tiles = p.m_blocks * p.n_blocks;
    const uint64_t lim = p.wait_limit_ns;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------- TMA producer
            uint32_t stage = 0, phase = 0;
            uint32_t filled = 0;        // bit s: stage s has a load whose landing is unobserved
            uint32_t fill_parity = 0;   // bit s: parity of that load's phase
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                const int m0 = (tile % p.m_blocks) * kBM;
                const int n0 = (tile / p.m_blocks) * kBN;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.status, lim)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], kStageBytes);
                    tma_load_2d(sA + stage * kABytes, &tm_a, &full[stage], kb * kBK, m0);
                    uint8_t *dstB = sB + stage * kBBytes;
                    if (p.b_mn_major) {
                        // [K, N] operand: kBN/64 boxes of 64 columns x 64 k-rows each.
#pragma unroll
                        for (int g = 0; g < kBN / 64; ++g)
                            tma_load_2d(dstB + g * (64 * kBK * 2), &tm_b, &full[stage], n0 + g * 64,
                                        kb * kBK);
                    } else {
                        tma_load_2d(dstB, &tm_b, &full[stage], kb * kBK, n0);
                    }
                    filled |= 1u << stage;
                    fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
                    advance(stage, phase, kStages);
                }
            }
            if (ok) {
                // Tail: wait until the MMA warp has released every stage, so no
                // tensor-core read or barrier arrival is still in flight at exit.
                for (int s = 0; s < kStages; ++s) {
                    if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.status, lim)) break;
                    advance(stage, phase, kStages);
                }
            } else {
                // Abort: let every issued TMA load land before the CTA's shared memory goes away.
                for (int s = 0; s < kStages; ++s) {
                    if (!(filled >> s & 1u)) continue;
                    const uint32_t a = smem_addr(&full[s]);
                    const uint32_t par = fill_parity >> s & 1u;
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(a, par) && global_timer_ns() - t0 < lim) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------- MMA issuer
            const uint32_t idesc = mma_idesc_bf16(kBM, kBN, p.b_mn_major ? 1u : 0u);
            uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                if (!wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, p.status, lim)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + acc * kBN;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!wait_bounded(&full[stage], phase, abort_flag, p.status, lim)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_base = smem_addr(sA + stage * kABytes);
                    const uint32_t b_base = smem_addr(sB + stage * kBBytes);
#pragma unroll
                    for (int kk = 0; kk < kBK / kMmaK; ++kk) {
                        const uint64_t a_desc = sw128_desc(a_base + kk * (kMmaK * 2), 16, 1024);
                        const uint64_t b_desc =
                            p.b_mn_major ? sw128_desc(b_base + kk * (kMmaK * 128), 64 * kBK * 2, 1024)
                                         : sw128_desc(b_base + kk * (kMmaK * 2), 16, 1024);
                        tc_mma_bf16(d_tmem, a_desc, b_desc, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit(&empty[stage]);
                    advance(stage, phase, kStages);
                }
                if (!ok) break;
                tc_commit(&tfull[acc]);
                advance(acc, acc_phase, 2);
            }
            if (!ok) {
                // Abort: wait for every MMA already issued before TMEM is released.
                tc_commit(drain);
                const uint32_t a = smem_addr(drain);
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(a, 0) && global_timer_ns() - t0 < lim) {
                }
            }
        }
    } else {
        // -------------------------------------------------------------- epilogue
        const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31 are this warp's
        const int row_in_tile = quarter * 32 + lane;
        uint32_t acc = 0, acc_phase = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            // All lanes take the same branch: tcgen05.ld below is warp-collective.
            const bool ready = wait_bounded(&tfull[acc], acc_phase, abort_flag, p.status, lim);
            if (!__all_sync(0xffffffffu, ready)) break;
            tc_fence_after_sync();
            const int64_t row = (int64_t)(tile % p.m_blocks) * kBM + row_in_tile;
            const int64_t n0 = (int64_t)(tile / p.m_blocks) * kBN;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * kBN;
#pragma unroll 1
            for (int c = 0; c < kBN / 32; ++c) {
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
            mbar_arrive(&tempty[acc]);
            advance(acc, acc_phase, 2);
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// K = 0: the product is empty, so C = input (addmm) or 0.
__global__ void gemm_k0_fill_kernel(const GemmParams p)
{
    const int64_t total = (int64_t)p.M * p.N;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / p.N, j = e % p.N;
        float v = 0.0f;
        if (p.addend_mode == kAddBias) v = __bfloat162float(p.addend[j]);
        if (p.addend_mode == kAddMatrix) v = __bfloat162float(p.addend[i * p.ld_addend + j]);
        if (p.c_f32)
            reinterpret_cast<float *>(p.C)[i * p.ldc + j] = v;
        else
            reinterpret_cast<__nv_bfloat16 *>(p.C)[i * p.ldc + j] = __float2bfloat16_rn(v);
    }
}

}  // namespace bi
