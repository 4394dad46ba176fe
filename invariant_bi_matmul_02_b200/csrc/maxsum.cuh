// maxsum.cuh -- the running (max, sum of exp) pair behind every log_softmax in the library:
// the one-block-per-row kernels, the split-row kernels and the GEMM epilogue that reduces each
// output tile of a row to one pair.  All merges here are fixed sequences or fixed xor
// butterflies, so a row's pair depends on its values alone.
#pragma once

#include <cstdint>

namespace bi {

#define kNegInf (-__builtin_huge_valf())

// (max, sum of exp(x - max)) pairs.  The merge is symmetric in its two arguments
// (no contracted multiply-adds), so both lanes of a butterfly pair hold equal bits.
struct MaxSum {
    float m, s;
};

__device__ __forceinline__ MaxSum merge(MaxSum a, MaxSum b)
{
    const float m = fmaxf(a.m, b.m);
    if (m == kNegInf) return {m, 0.0f};
    const float s = __fadd_rn(__fmul_rn(a.s, __expf(a.m - m)), __fmul_rn(b.s, __expf(b.m - m)));
    return {m, s};
}

__device__ __forceinline__ MaxSum warp_merge(MaxSum v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        MaxSum w{__shfl_xor_sync(0xffffffffu, v.m, o), __shfl_xor_sync(0xffffffffu, v.s, o)};
        v = merge(v, w);
    }
    return v;
}

// Running (max, sum) update with a group of values already reduced to their max `gm`.
__device__ __forceinline__ void rescale_to(MaxSum &acc, float gm)
{
    if (gm > acc.m) {
        acc.s = acc.m == kNegInf ? 0.0f : acc.s * __expf(acc.m - gm);
        acc.m = gm;
    }
}

template <int P>
__device__ __forceinline__ void lsm_accumulate(MaxSum &acc, const float (&v)[P])
{
    float gm = v[0];
#pragma unroll
    for (int k = 1; k < P; ++k) gm = fmaxf(gm, v[k]);
    rescale_to(acc, gm);
    if (acc.m != kNegInf) {
#pragma unroll
        for (int k = 0; k < P; ++k) acc.s += __expf(v[k] - acc.m);
    }
}

}  // namespace bi
