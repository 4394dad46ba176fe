// gemm.cuh -- pieces shared by the GEMM kernel: launch parameters, the bounded
// mbarrier wait, ring-index arithmetic and the epilogue's addend/store helpers.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace bi {

constexpr int kBM = 128;          // rows of C per CTA (one TMEM lane per row)
constexpr int kBK = 64;           // K per pipeline stage: one 128-byte swizzle row of bf16
constexpr int kMmaK = 16;         // K of one tcgen05.mma kind::f16
constexpr int kGemmThreads = 192; // warp 0 TMA, warp 1 TMEM/MMA, warps 2..5 epilogue
constexpr int kSmemBudget = 227 * 1024;
constexpr int kSmemMisc = 1024 /*alignment slack*/ + 512 /*barriers, flags*/;
constexpr uint32_t pow2_at_least(uint32_t v, uint32_t p = 32) { return p >= v ? p : pow2_at_least(v, p * 2); }

enum AddendMode : int { kAddNone = 0, kAddBias = 1, kAddMatrix = 2 };

struct GemmParams {
    int32_t M, N, K;
    int32_t m_blocks, n_blocks, k_blocks;
    int32_t b_mn_major;     // 1: B stored [K, N] (MN-major operand); 0: B stored [N, K]
    int32_t c_f32;          // 1: C is fp32; 0: C is bf16
    int32_t addend_mode;    // AddendMode
    int32_t fuse_silu;      // 1: B is [gate; up] (2F rows), C = silu(A.gate^T) * (A.up^T), N = F
    int64_t ldc;
    int64_t ld_addend;
    void *C;
    const __nv_bfloat16 *addend;
    int32_t *status;        // device status word
    uint64_t wait_limit_ns;
    int32_t a_box_rows;     // rows of A one TMA box copies: M rounded up to 8, at most 128
};

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

// silu(g) * u of one row chunk, fp32 inside, stored as bf16 (columns col0 .. col0+31 of h).
__device__ __forceinline__ void store_silu_chunk(const GemmParams &p, int64_t row, int64_t col0,
                                                 const float (&g)[32], const float (&u)[32])
{
    float h[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) h[j] = __fmul_rn(g[j] / (1.0f + __expf(-g[j])), u[j]);
    store_row_chunk(p, row, col0, col0 + 32 <= p.N, h);
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
