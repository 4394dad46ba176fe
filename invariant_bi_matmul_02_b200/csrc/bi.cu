// bi.cu -- host side of libbi.so: argument checks, TMA tensor-map encoding and
// stream-ordered launches behind the C ABI declared in include/bi.h.
//
// The library allocates no device memory.  Per device it caches the SM count, the
// address of its status word and the GEMM kernel's shared-memory attribute.  No
// launch decision depends on M except the grid size (how many CTAs share the tile
// list, or how many rows there are), which never changes a row's arithmetic.
#include "bi.h"

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstddef>
#include <cstdint>
#include <mutex>

#include "gemm.cuh"
#include "attention.cuh"
#include "gemm_pair.cuh"
#include "ptx.cuh"
#include "rowops.cuh"

// Per-device status word: 0, or the first error a kernel recorded (BI_ERR_TIMEOUT).
__device__ int32_t g_bi_status = 0;

namespace {

constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s per device-side wait
constexpr int kMaxDevices = 64;
constexpr int64_t kI32Max = 2147483647;

struct DeviceState {
    bool ready = false;
    int sms = 0;
    int gemm_clusters_wide = 0;    // CTA pairs of each GEMM configuration that fit on the device at once
    int gemm_clusters_narrow = 0;
    int gemm_clusters_mid = 0;
    int mean_rows_blocks_per_sm = 0;  // co-resident 1024-thread blocks of the persistent mean
    int32_t *status = nullptr;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Opt the decode-attention kernels of head size D into their shared memory.
template <int D>
bi_status attn_smem_opt_in()
{
    const void *fns[4] = {reinterpret_cast<const void *>(bi::decode_attention_split_kernel<1, D>),
                          reinterpret_cast<const void *>(bi::decode_attention_split_kernel<2, D>),
                          reinterpret_cast<const void *>(bi::decode_attention_split_kernel<4, D>),
                          reinterpret_cast<const void *>(bi::decode_attention_split_kernel<8, D>)};
    for (const void *fn : fns)
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bi::kAttnSmem) != cudaSuccess)
            return BI_ERR_CUDA;
    return BI_OK;
}

// Opt the GEMM configuration T into its shared memory and count the CTA pairs that fit at once.
template <typename T>
bi_status pair_clusters(int sms, int *out)
{
    const void *fn = reinterpret_cast<const void *>(bi::gemm_bf16_pair_kernel<T::kBN, T::kStageK>);
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, T::kSmem) != cudaSuccess)
        return BI_ERR_CUDA;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * sms, 1, 1);
    cfg.blockDim = dim3(bi::kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = T::kSmem;
    cudaLaunchAttribute attr{};
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess || n < 1) return BI_ERR_CUDA;
    *out = n;
    return BI_OK;
}

bi_status device_state(DeviceState **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BI_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return BI_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState &d = g_dev[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return BI_ERR_CUDA;
        void *sym = nullptr;
        if (cudaGetSymbolAddress(&sym, g_bi_status) != cudaSuccess) return BI_ERR_CUDA;
        d.status = static_cast<int32_t *>(sym);
        if (pair_clusters<bi::WideTile>(d.sms, &d.gemm_clusters_wide) != BI_OK ||
            pair_clusters<bi::NarrowTile>(d.sms, &d.gemm_clusters_narrow) != BI_OK ||
            pair_clusters<bi::MidTile>(d.sms, &d.gemm_clusters_mid) != BI_OK)
            return BI_ERR_CUDA;
        if (attn_smem_opt_in<64>() != BI_OK || attn_smem_opt_in<128>() != BI_OK) return BI_ERR_CUDA;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.mean_rows_blocks_per_sm, bi::mean_rows_kernel,
                                                          bi::kMeanRowsThreads, 0) !=
                cudaSuccess ||
            d.mean_rows_blocks_per_sm < 1)
            return BI_ERR_CUDA;
        if (cudaFuncSetAttribute(bi::log_softmax_stream_kernel<true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, bi::kLsmSmem) != cudaSuccess ||
            cudaFuncSetAttribute(bi::log_softmax_stream_kernel<false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, bi::kLsmSmem) != cudaSuccess ||
            cudaFuncSetAttribute(bi::log_softmax_cluster_kernel<true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, bi::kClSliceBytesMax) != cudaSuccess ||
            cudaFuncSetAttribute(bi::log_softmax_cluster_kernel<false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, bi::kClSliceBytesMax) != cudaSuccess)
            return BI_ERR_CUDA;
        if (bi::kRowCluster > 8 &&  // clusters above the portable size must be allowed per kernel
            (cudaFuncSetAttribute(bi::log_softmax_cluster_kernel<true>,
                                  cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess ||
             cudaFuncSetAttribute(bi::log_softmax_cluster_kernel<false>,
                                  cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess))
            return BI_ERR_CUDA;
        d.ready = true;
    }
    *out = &d;
    return BI_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D bf16 tensor map over a row-major matrix: `inner` contiguous elements per row,
// `outer` rows `ld` elements apart, box inner x outer, 128-byte swizzle, zero fill.
bi_status encode_map_uncached(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer, uint64_t ld,
                              uint32_t box_inner, uint32_t box_outer)
{
    auto enc = tensor_map_encoder();
    if (!enc) return BI_ERR_CUDA;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {ld * 2};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? BI_OK : BI_ERR_CUDA;
}

// Encoded tensor maps, keyed by everything the encoding reads (base address, extents, row
// stride, box).  A map is a pure function of its key, so a hit returns exactly the map a fresh
// encoding would; a freed and re-allocated buffer at the same address with the same shape gets
// the same, still correct, map.  Direct-mapped with kMapCacheSlots slots under one mutex: a
// colliding key replaces the slot.  A GEMM call looks up two maps.
struct MapKey {
    uint64_t base, inner, outer, ld;
    uint32_t box_inner, box_outer;
    bool operator==(const MapKey &o) const
    {
        return base == o.base && inner == o.inner && outer == o.outer && ld == o.ld &&
               box_inner == o.box_inner && box_outer == o.box_outer;
    }
};
struct MapSlot {
    bool used = false;
    MapKey key{};
    CUtensorMap map{};
};
constexpr int kMapCacheSlots = 256;
std::mutex g_map_mu;
MapSlot g_map_cache[kMapCacheSlots];
uint64_t g_map_hits = 0, g_map_misses = 0;

inline uint32_t map_slot(const MapKey &k)
{
    uint64_t h = 0x9E3779B97F4A7C15ull;
    for (uint64_t v : {k.base, k.inner, k.outer, k.ld, (uint64_t)k.box_inner << 32 | k.box_outer}) {
        h ^= v + 0x9E3779B97F4A7C15ull + (h << 6) + (h >> 2);
    }
    return (uint32_t)(h % kMapCacheSlots);
}

bi_status encode_map(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer, uint64_t ld,
                     uint32_t box_inner, uint32_t box_outer)
{
    const MapKey key{reinterpret_cast<uint64_t>(base), inner, outer, ld, box_inner, box_outer};
    const uint32_t slot = map_slot(key);
    std::lock_guard<std::mutex> lock(g_map_mu);
    MapSlot &e = g_map_cache[slot];
    if (e.used && e.key == key) {
        ++g_map_hits;
        *map = e.map;
        return BI_OK;
    }
    ++g_map_misses;
    const bi_status st = encode_map_uncached(map, base, inner, outer, ld, box_inner, box_outer);
    if (st != BI_OK) return st;
    e.used = true;
    e.key = key;
    e.map = *map;
    return BI_OK;
}

// 4-D bf16 tensor map over a decode cache [B, Lmax, Hkv, D] (row-major): dims innermost first
// (D, Hkv, Lmax, B); box 64 d x 1 head x 128 tokens x 1 sequence, 128-byte swizzle, zero fill
// past Lmax.
bi_status encode_kv_map(CUtensorMap *map, const void *base, uint64_t D, uint64_t Hkv, uint64_t Lmax, uint64_t B)
{
    auto enc = tensor_map_encoder();
    if (!enc) return BI_ERR_CUDA;
    const cuuint64_t dims[4] = {D, Hkv, Lmax, B};
    const cuuint64_t strides[3] = {D * 2, Hkv * D * 2, Lmax * Hkv * D * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)bi::kAttnChunk, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? BI_OK : BI_ERR_CUDA;
}

// Launch `kernel` on `s` and report the launch's own result.  cudaLaunchKernelEx returns the
// error of this launch, so a failure left behind by some other library's launch on this thread
// is neither reported as ours nor cleared.
template <typename... KArgs, typename... Args>
bi_status launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = nullptr;
    cfg.numAttrs = 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

// Launch `kernel` with programmatic stream serialization: it may start while the previous kernel
// in the stream finishes, and waits (griddep_wait) for it before touching global memory.
template <typename... KArgs, typename... Args>
bi_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr{};
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

// Launch `kernel` with one cluster of bi::kRowCluster CTAs per row, rows on grid.y in slices of
// at most 65535; the kernel takes the slice's first row as its `row0` argument.
template <typename... KArgs, typename... Args>
bi_status launch_row_clusters(void (*kernel)(KArgs...), int64_t M, size_t smem, cudaStream_t s, Args... args)
{
    for (int64_t row0 = 0; row0 < M; row0 += 65535) {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(bi::kRowCluster, (unsigned)(M - row0 < 65535 ? M - row0 : 65535), 1);
        cfg.blockDim = dim3(bi::kClThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr{};
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = bi::kRowCluster;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, kernel, args..., row0) != cudaSuccess) return BI_ERR_CUDA;
    }
    return BI_OK;
}

// N is the number of output columns.  With fuse_silu, B holds 2N rows ([gate; up]) and
// the output is silu(A . gate^T) * (A . up^T).
// Launch 1 (group size G chosen at run time, head size D) and launch 2 of the decode attention.
template <int D>
bi_status launch_attention(int64_t group, dim3 grid, size_t smem, cudaStream_t s, const CUtensorMap &tm_k,
                           const CUtensorMap &tm_v, const bi::AttnParams &p, const int32_t *seq_lens, void *out,
                           int64_t B)
{
    bi_status st;
    switch (group) {
    case 1: st = launch_pdl(bi::decode_attention_split_kernel<1, D>, grid, dim3(bi::kAttnThreads), smem, s, tm_k, tm_v, p); break;
    case 2: st = launch_pdl(bi::decode_attention_split_kernel<2, D>, grid, dim3(bi::kAttnThreads), smem, s, tm_k, tm_v, p); break;
    case 4: st = launch_pdl(bi::decode_attention_split_kernel<4, D>, grid, dim3(bi::kAttnThreads), smem, s, tm_k, tm_v, p); break;
    case 8: st = launch_pdl(bi::decode_attention_split_kernel<8, D>, grid, dim3(bi::kAttnThreads), smem, s, tm_k, tm_v, p); break;
    default: return BI_ERR_UNSUPPORTED;
    }
    if (st != BI_OK || p.out != nullptr) return st;  // one split per sequence: launch 1 wrote out
    return launch_pdl(bi::decode_attention_combine_kernel<D>, dim3((unsigned)p.Hq, (unsigned)B), dim3(D), 0, s,
                      static_cast<const float2 *>(p.part_ms), static_cast<const float *>(p.part_acc), seq_lens,
                      static_cast<__nv_bfloat16 *>(out), (int)p.Hq, p.Lmax);
}

// Tile counts, tensor maps and the launch of the pair GEMM in configuration T.
template <typename T>
bi_status launch_pair(bi::GemmParams p, const void *A, int64_t lda, const void *B, int64_t ldb, int b_layout,
                      int64_t b_rows, int pairs, cudaStream_t s)
{
    // [K, N] weights are staged in 64-column groups per CTA; pair_config never sends them to a
    // tile whose half-width is not a multiple of 64.
    if (b_layout == BI_B_KN && !T::kKNOk) return BI_ERR_UNSUPPORTED;
    const int64_t M = p.M, N = p.N, K = p.K;
    p.m_blocks = (int32_t)((M + bi::kPairBM - 1) / bi::kPairBM);
    p.n_blocks = (int32_t)(p.fuse_silu ? (N + T::kHalf - 1) / T::kHalf : (N + T::kBN - 1) / T::kBN);
    p.k_blocks = (int32_t)((K + T::kStageK - 1) / T::kStageK);
    const int64_t tiles = (int64_t)p.m_blocks * p.n_blocks;
    if (tiles > kI32Max) return BI_ERR_UNSUPPORTED;

    CUtensorMap tm_a, tm_b;
    // The A box copies the rows that exist: M rounded up to 8, at most the CTA's 128.  The tile,
    // the MMA shape and every element's K order are the same for every M.
    p.a_box_rows = (int32_t)(M >= bi::kBM ? bi::kBM : (M + 7) / 8 * 8);
    bi_status st = encode_map(&tm_a, A, (uint64_t)K, (uint64_t)M, (uint64_t)lda, bi::kBK, (uint32_t)p.a_box_rows);
    if (st != BI_OK) return st;
    if (b_layout == BI_B_NK)
        st = encode_map(&tm_b, B, (uint64_t)K, (uint64_t)b_rows, (uint64_t)ldb, bi::kBK, (uint32_t)T::kHalf);
    else
        st = encode_map(&tm_b, B, (uint64_t)b_rows, (uint64_t)K, (uint64_t)ldb, 64, (uint32_t)T::kStageK);
    if (st != BI_OK) return st;

    const int grid = 2 * (int)(tiles < pairs ? tiles : pairs);
    return launch_pdl(bi::gemm_bf16_pair_kernel<T::kBN, T::kStageK>, dim3(grid), dim3(bi::kGemmThreads),
                      (size_t)T::kSmem, s, tm_a, tm_b, p);
}

bi_status gemm_common(const void *input, int64_t ld_input, int addend_mode, const void *A, int64_t lda,
                      const void *B, int64_t ldb, int b_layout, void *C, int64_t ldc, int c_dtype,
                      int64_t M, int64_t N, int64_t K, void *stream, int fuse_silu = 0)
{
    if (M < 0 || N < 0 || K < 0) return BI_ERR_INVALID_ARG;
    if (b_layout != BI_B_KN && b_layout != BI_B_NK) return BI_ERR_INVALID_ARG;
    if (c_dtype != BI_BF16 && c_dtype != BI_F32) return BI_ERR_INVALID_ARG;
    if (M > kI32Max || (fuse_silu ? 2 * N : N) > kI32Max || K > kI32Max) return BI_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return BI_OK;
    const int64_t b_rows = fuse_silu ? 2 * N : N;  // extent of B along the output dimension
    if (!C || ldc < N) return BI_ERR_INVALID_ARG;
    if (addend_mode != bi::kAddNone) {
        if (!input || ld_input < 0 || (ld_input != 0 && ld_input < N)) return BI_ERR_INVALID_ARG;
        if (!aligned16(input) || ld_input % 8 != 0) return BI_ERR_ALIGNMENT;
    }
    const bool c_f32 = c_dtype == BI_F32;
    if (!aligned16(C) || ldc % (c_f32 ? 4 : 8) != 0) return BI_ERR_ALIGNMENT;
    if (K > 0) {
        if (!A || !B) return BI_ERR_INVALID_ARG;
        if (lda < K || ldb < (b_layout == BI_B_KN ? b_rows : K)) return BI_ERR_INVALID_ARG;
        if (!aligned16(A) || !aligned16(B) || lda % 8 != 0 || ldb % 8 != 0) return BI_ERR_ALIGNMENT;
        // [K, 2F] gate/up weights: the up half starts at column F, the innermost coordinate of its
        // tile loads, which a TMA copy needs at a multiple of 16 bytes (8 bf16 elements).
        if (fuse_silu && b_layout == BI_B_KN && N % 8 != 0) return BI_ERR_ALIGNMENT;
    }

    DeviceState *dev = nullptr;
    bi_status st = device_state(&dev);
    if (st != BI_OK) return st;

    bi::GemmParams p{};
    p.M = (int32_t)M;
    p.N = (int32_t)N;
    p.K = (int32_t)K;
    p.fuse_silu = fuse_silu;
    p.b_mn_major = b_layout == BI_B_KN ? 1 : 0;
    p.c_f32 = c_f32 ? 1 : 0;
    p.addend_mode = addend_mode;
    p.ldc = ldc;
    p.ld_addend = ld_input;
    p.C = C;
    p.addend = static_cast<const __nv_bfloat16 *>(input);
    p.status = dev->status;
    p.wait_limit_ns = kWaitLimitNs;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    if (K == 0 && !fuse_silu) {
        const int64_t total = M * N;
        int64_t blocks = (total + 255) / 256;
        if (blocks > (int64_t)dev->sms * 16) blocks = (int64_t)dev->sms * 16;
        return launch(bi::gemm_k0_fill_kernel, dim3((unsigned)blocks), dim3(256), 0, s, p);
    }

    // The tile configuration is a function of the weight alone (its rows and storage); every M of
    // a given weight runs the same one.
    switch (bi::pair_config(b_rows, b_layout == BI_B_NK)) {
    case bi::kPairNarrow:
        return launch_pair<bi::NarrowTile>(p, A, lda, B, ldb, b_layout, b_rows, dev->gemm_clusters_narrow, s);
    case bi::kPairMid:
        return launch_pair<bi::MidTile>(p, A, lda, B, ldb, b_layout, b_rows, dev->gemm_clusters_mid, s);
    default:
        break;
    }
    return launch_pair<bi::WideTile>(p, A, lda, B, ldb, b_layout, b_rows, dev->gemm_clusters_wide, s);
}

__global__ void selftest_wait_kernel(int32_t *status, uint64_t limit_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        bi::mbar_init(&bar, 1);
        abort_flag = 0;
        bi::fence_mbar_init();
    }
    __syncthreads();
    // Phase 0 of `bar` never completes: nothing arrives on it.
    if (threadIdx.x == 0) bi::wait_bounded(&bar, 0, &abort_flag, status, limit_ns);
    __syncthreads();
}

// The two launches of the split log_softmax: per-(row, chunk) partials, then the merge and write.
bi_status split_launches(bool bf16, dim3 grid, cudaStream_t s, const uint8_t *xb, float2 *part, float *y, int64_t V)
{
    bi_status st = bf16 ? launch(bi::log_softmax_split_stats_kernel<true>, grid, dim3(bi::kSplitThreads), 0, s, xb,
                                 part, V)
                        : launch(bi::log_softmax_split_stats_kernel<false>, grid, dim3(bi::kSplitThreads), 0, s, xb,
                                 part, V);
    if (st != BI_OK) return st;
    return bf16 ? launch(bi::log_softmax_split_write_kernel<true>, grid, dim3(bi::kSplitThreads), 0, s, xb,
                         static_cast<const float2 *>(part), y, V)
                : launch(bi::log_softmax_split_write_kernel<false>, grid, dim3(bi::kSplitThreads), 0, s, xb,
                         static_cast<const float2 *>(part), y, V);
}

inline unsigned elementwise_blocks(int64_t work, int sms)
{
    int64_t blocks = (work + 255) / 256;
    const int64_t cap = (int64_t)sms * 8;
    return (unsigned)(blocks < 1 ? 1 : (blocks > cap ? cap : blocks));
}

}  // namespace

extern "C" {

bi_status bi_matmul(const void *A, int64_t lda, const void *B, int64_t ldb, bi_b_layout b_layout,
                    void *C, int64_t ldc, bi_dtype c_dtype, int64_t M, int64_t N, int64_t K,
                    void *stream)
{
    return gemm_common(nullptr, 0, bi::kAddNone, A, lda, B, ldb, b_layout, C, ldc, c_dtype, M, N, K,
                       stream);
}

bi_status bi_addmm(const void *input, int64_t ld_input, const void *A, int64_t lda, const void *B,
                   int64_t ldb, bi_b_layout b_layout, void *C, int64_t ldc, bi_dtype c_dtype,
                   int64_t M, int64_t N, int64_t K, void *stream)
{
    return gemm_common(input, ld_input, ld_input == 0 ? bi::kAddBias : bi::kAddMatrix, A, lda, B, ldb,
                       b_layout, C, ldc, c_dtype, M, N, K, stream);
}

bi_status bi_matmul_silu_mul(const void *A, int64_t lda, const void *B, int64_t ldb,
                             bi_b_layout b_layout, void *H, int64_t ldh, int64_t M, int64_t F, int64_t K,
                             void *stream)
{
    if (K == 0)  // empty products: silu(0) * 0 = 0
        return gemm_common(nullptr, 0, bi::kAddNone, A, lda, B, ldb, b_layout, H, ldh, BI_BF16, M, F, 0,
                           stream, 0);
    return gemm_common(nullptr, 0, bi::kAddNone, A, lda, B, ldb, b_layout, H, ldh, BI_BF16, M, F, K, stream,
                       1);
}

bi_status bi_rmsnorm(const void *x, const void *w, void *y, int64_t M, int64_t H, float eps,
                     void *stream)
{
    if (M < 0 || H < 0 || !(eps >= 0.0f)) return BI_ERR_INVALID_ARG;
    if (M > kI32Max || H > kI32Max) return BI_ERR_UNSUPPORTED;
    if (M == 0) return BI_OK;
    if (H == 0 || !x || !w || !y) return BI_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int T = bi::rmsnorm_threads(H);
    bi_status st = BI_OK;
    if (H % 8 == 0) {
        if (!aligned16(x) || !aligned16(w) || !aligned16(y)) return BI_ERR_ALIGNMENT;
        const int64_t cpt = (H / 8 + T - 1) / T;
        const uint4 *xv = static_cast<const uint4 *>(x);
        const uint4 *wv = static_cast<const uint4 *>(w);
        uint4 *yv = static_cast<uint4 *>(y);
        switch (cpt) {
        case 1: st = launch_pdl(bi::rmsnorm_vec_kernel<1>, dim3((unsigned)M), dim3(T), 0, s, xv, wv, yv, H, eps); break;
        case 2: st = launch_pdl(bi::rmsnorm_vec_kernel<2>, dim3((unsigned)M), dim3(T), 0, s, xv, wv, yv, H, eps); break;
        case 3: st = launch_pdl(bi::rmsnorm_vec_kernel<3>, dim3((unsigned)M), dim3(T), 0, s, xv, wv, yv, H, eps); break;
        case 4: st = launch_pdl(bi::rmsnorm_vec_kernel<4>, dim3((unsigned)M), dim3(T), 0, s, xv, wv, yv, H, eps); break;
        default:
            st = launch(bi::rmsnorm_scalar_kernel, dim3((unsigned)M), dim3(T), 0, s,
                        static_cast<const __nv_bfloat16 *>(x), static_cast<const __nv_bfloat16 *>(w),
                        static_cast<__nv_bfloat16 *>(y), H, eps);
        }
        return st;
    }
    return launch(bi::rmsnorm_scalar_kernel, dim3((unsigned)M), dim3(T), 0, s,
                  static_cast<const __nv_bfloat16 *>(x), static_cast<const __nv_bfloat16 *>(w),
                  static_cast<__nv_bfloat16 *>(y), H, eps);
}

bi_status bi_mean(const float *x, float *y, int64_t M, int64_t H, void *stream)
{
    if (M < 0 || H < 0) return BI_ERR_INVALID_ARG;
    if (M > kI32Max || H > kI32Max) return BI_ERR_UNSUPPORTED;
    if (M == 0) return BI_OK;
    if (H == 0 || !x || !y) return BI_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int T = bi::mean_threads(H);
    bi_status st = BI_OK;
    if (H % 4 == 0) {
        if (!aligned16(x)) return BI_ERR_ALIGNMENT;
        if (H / 4 >= 8 * (int64_t)T && T == bi::kMeanRowsThreads) {
            DeviceState *dev = nullptr;
            st = device_state(&dev);
            if (st != BI_OK) return st;
            const int64_t fit = (int64_t)dev->sms * dev->mean_rows_blocks_per_sm;
            st = launch_pdl(bi::mean_rows_kernel, dim3((unsigned)(M < fit ? M : fit)), dim3(T), 0, s,
                            reinterpret_cast<const float4 *>(x), y, H, M);
        } else
            st = launch_pdl(bi::mean_vec_kernel, dim3((unsigned)M), dim3(T), 0, s,
                            reinterpret_cast<const float4 *>(x), y, H);
        return st;
    }
    return launch(bi::mean_scalar_kernel, dim3((unsigned)M), dim3(T), 0, s, x, y, H);
}

bi_status bi_log_softmax(const void *x, bi_dtype x_dtype, float *y, int64_t M, int64_t V, void *stream)
{
    if (M < 0 || V < 0) return BI_ERR_INVALID_ARG;
    if (x_dtype != BI_BF16 && x_dtype != BI_F32) return BI_ERR_INVALID_ARG;
    if (M > kI32Max || V > kI32Max) return BI_ERR_UNSUPPORTED;
    if (M == 0) return BI_OK;
    if (V == 0 || !x || !y) return BI_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int T = bi::log_softmax_threads(V);
    const bool bf16 = x_dtype == BI_BF16;
    const int per = bf16 ? 8 : 4;
    if (V % per == 0) {
        if (!aligned16(x) || !aligned16(y)) return BI_ERR_ALIGNMENT;
        DeviceState *dev = nullptr;
        bi_status st = device_state(&dev);
        if (st != BI_OK) return st;
        const uint8_t *xb = static_cast<const uint8_t *>(x);
        st = bf16 ? launch_pdl(bi::log_softmax_stream_kernel<true>, dim3((unsigned)M), dim3(bi::kLsmThreads),
                               (size_t)bi::kLsmSmem, s, xb, y, V, dev->status, kWaitLimitNs)
                  : launch_pdl(bi::log_softmax_stream_kernel<false>, dim3((unsigned)M), dim3(bi::kLsmThreads),
                               (size_t)bi::kLsmSmem, s, xb, y, V, dev->status, kWaitLimitNs);
        return st;
    }
    return bf16 ? launch(bi::log_softmax_scalar_kernel<true>, dim3((unsigned)M), dim3(T), 0, s, x, y, V)
                : launch(bi::log_softmax_scalar_kernel<false>, dim3((unsigned)M), dim3(T), 0, s, x, y, V);
}

bi_status bi_log_softmax_cluster(const void *x, bi_dtype x_dtype, float *y, int64_t M, int64_t V, void *stream)
{
    if (M < 0 || V < 0) return BI_ERR_INVALID_ARG;
    if (x_dtype != BI_BF16 && x_dtype != BI_F32) return BI_ERR_INVALID_ARG;
    if (M > kI32Max || V > kI32Max) return BI_ERR_UNSUPPORTED;
    if (M == 0) return BI_OK;
    if (V == 0 || !x || !y) return BI_ERR_INVALID_ARG;
    const bool bf16 = x_dtype == BI_BF16;
    const int elem = bf16 ? 2 : 4;
    const int64_t slice_bytes = bi::cluster_slice(V) * elem;
    if (V % (bf16 ? 8 : 4) != 0 || V * elem < bi::kClusterRowBytes || slice_bytes > bi::kClSliceBytesMax)
        return BI_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(y)) return BI_ERR_ALIGNMENT;
    DeviceState *dev = nullptr;
    bi_status st = device_state(&dev);
    if (st != BI_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uint8_t *xb = static_cast<const uint8_t *>(x);
    st = bf16 ? launch_row_clusters(bi::log_softmax_cluster_kernel<true>, M, (size_t)slice_bytes, s, xb, y, V,
                                    dev->status, kWaitLimitNs)
              : launch_row_clusters(bi::log_softmax_cluster_kernel<false>, M, (size_t)slice_bytes, s, xb, y, V,
                                    dev->status, kWaitLimitNs);
    return st;
}

size_t bi_log_softmax_split_scratch_bytes(int64_t M, int64_t V)
{
    if (M <= 0 || V <= 0) return 0;
    return (size_t)M * (size_t)bi::split_chunks(V) * sizeof(float2);
}

bi_status bi_log_softmax_split(const void *x, bi_dtype x_dtype, float *y, int64_t M, int64_t V, void *scratch,
                               size_t scratch_bytes, void *stream)
{
    if (M < 0 || V < 0) return BI_ERR_INVALID_ARG;
    if (x_dtype != BI_BF16 && x_dtype != BI_F32) return BI_ERR_INVALID_ARG;
    if (M > 65535 || V > kI32Max) return BI_ERR_UNSUPPORTED;  // rows on grid.y
    if (M == 0) return BI_OK;
    if (V == 0 || !x || !y || !scratch) return BI_ERR_INVALID_ARG;
    if (V % 8 != 0) return BI_ERR_UNSUPPORTED;
    if (scratch_bytes < bi_log_softmax_split_scratch_bytes(M, V)) return BI_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y) || !aligned16(scratch)) return BI_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const dim3 grid((unsigned)bi::split_chunks(V), (unsigned)M);
    const uint8_t *xb = static_cast<const uint8_t *>(x);
    float2 *part = static_cast<float2 *>(scratch);
    return split_launches(x_dtype == BI_BF16, grid, s, xb, part, y, V);
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// Allocation-free split log_softmax.
//
// Some callers cannot hand the library a scratch buffer because they cannot allocate device
// memory when they call it: code that runs under a memory budget fixed at start-up (every
// byte already reserved by a pool it does not own), plugins living inside a host framework
// that controls all device allocation, or callers on a hot path where a cudaMalloc's
// implicit synchronisation is not acceptable.  For them the partials of the split path live
// in this file-scope device array.  It has a fixed size and is part of the module image, so
// every GPU that loads libbi.so holds it until the process exits, and no call allocates.
namespace {

constexpr int64_t kNoAllocPartials = 65536;  // (row, chunk) partials: 512 KiB per device
static __device__ __align__(256) float2 g_noalloc_partials[kNoAllocPartials];

std::mutex g_noalloc_mu;
float2 *g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_partials on the current device.  In host code the array's name
// only stands in for the symbol, so its address is looked up once per device, with that device
// current, and cached.
bi_status noalloc_partials(float2 **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BI_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return BI_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_partials) != cudaSuccess || !p) return BI_ERR_CUDA;
        g_noalloc_ptr[dev] = static_cast<float2 *>(p);
    }
    *out = g_noalloc_ptr[dev];
    return BI_OK;
}

}  // namespace

extern "C" {

bi_status bi_log_softmax_split_noalloc(const void *x, bi_dtype x_dtype, float *y, int64_t M, int64_t V,
                                       void *stream)
{
    if (M < 0 || V < 0) return BI_ERR_INVALID_ARG;
    if (x_dtype != BI_BF16 && x_dtype != BI_F32) return BI_ERR_INVALID_ARG;
    if (M > 65535 || V > kI32Max) return BI_ERR_UNSUPPORTED;
    if (M == 0) return BI_OK;
    if (V == 0 || !x || !y) return BI_ERR_INVALID_ARG;
    if (V % 8 != 0) return BI_ERR_UNSUPPORTED;
    if (M * bi::split_chunks(V) > kNoAllocPartials) return BI_ERR_UNSUPPORTED;  // beyond the fixed array
    if (!aligned16(x) || !aligned16(y)) return BI_ERR_ALIGNMENT;
    float2 *part = nullptr;
    bi_status st = noalloc_partials(&part);
    if (st != BI_OK) return st;
    // Launch 1 overwrites every partial that launch 2 reads, so nothing needs clearing.
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const dim3 grid((unsigned)bi::split_chunks(V), (unsigned)M);
    const uint8_t *xb = static_cast<const uint8_t *>(x);
    return split_launches(x_dtype == BI_BF16, grid, s, xb, part, y, V);
}

size_t bi_decode_attention_scratch_bytes(int64_t B, int64_t Hq, int64_t D, int64_t Lmax)
{
    if (B <= 0 || Hq <= 0 || D <= 0 || Lmax <= 0) return 0;
    const size_t parts = (size_t)B * (size_t)Hq * (size_t)bi::attn_splits(Lmax);
    return parts * ((size_t)D * sizeof(float) + sizeof(float2));
}

bi_status bi_decode_attention(const void *q, const void *k_cache, const void *v_cache, const int32_t *seq_lens,
                              void *out, int64_t B, int64_t Hq, int64_t Hkv, int64_t D, int64_t Lmax, float scale,
                              void *scratch, size_t scratch_bytes, void *stream)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Lmax <= 0) return B == 0 ? BI_OK : BI_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return BI_ERR_INVALID_ARG;
    const int64_t group = Hq / Hkv;
    if ((D != 64 && D != 128) || (group != 1 && group != 2 && group != 4 && group != 8)) return BI_ERR_UNSUPPORTED;
    if (B > 65535 || Hkv > 65535 || Hq > 65535 || bi::attn_splits(Lmax) > kI32Max) return BI_ERR_UNSUPPORTED;
    if (B * Hkv * bi::attn_splits(Lmax) > kI32Max) return BI_ERR_UNSUPPORTED;  // work items are 32-bit indices
    if (B == 0) return BI_OK;
    if (!q || !k_cache || !v_cache || !seq_lens || !out || !scratch) return BI_ERR_INVALID_ARG;
    if (scratch_bytes < bi_decode_attention_scratch_bytes(B, Hq, D, Lmax)) return BI_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(scratch) ||
        (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
        return BI_ERR_ALIGNMENT;
    DeviceState *dev = nullptr;
    bi_status st = device_state(&dev);
    if (st != BI_OK) return st;
    const int64_t S = bi::attn_splits(Lmax);
    CUtensorMap tm_k, tm_v;
    st = encode_kv_map(&tm_k, k_cache, (uint64_t)D, (uint64_t)Hkv, (uint64_t)Lmax, (uint64_t)B);
    if (st != BI_OK) return st;
    st = encode_kv_map(&tm_v, v_cache, (uint64_t)D, (uint64_t)Hkv, (uint64_t)Lmax, (uint64_t)B);
    if (st != BI_OK) return st;
    bi::AttnParams p{};
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.lens = seq_lens;
    p.part_acc = static_cast<float *>(scratch);
    p.part_ms = reinterpret_cast<float2 *>(p.part_acc + (size_t)B * Hq * S * D);
    // With Lmax <= 512 every sequence is one split, whose fold launch 1 does itself.
    p.out = S == 1 ? static_cast<__nv_bfloat16 *>(out) : nullptr;
    p.Hq = (int32_t)Hq;
    p.Hkv = (int32_t)Hkv;
    p.B = (int32_t)B;
    p.Lmax = Lmax;
    p.S = S;
    p.scale = scale;
    p.status = dev->status;
    p.wait_limit_ns = kWaitLimitNs;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // Persistent: one CTA per SM walks the (split, kv head, sequence) items; the grid size only
    // decides which CTA computes an item, never an item's arithmetic.
    const int64_t items = B * Hkv * S;
    const dim3 grid((unsigned)(items < dev->sms ? items : dev->sms));
    const size_t smem = (size_t)bi::kAttnSmem;
    // The group size and the head size are properties of the model, not of the batch.
    return D == 64 ? launch_attention<64>(Hq / Hkv, grid, smem, s, tm_k, tm_v, p, seq_lens, out, B)
                   : launch_attention<128>(Hq / Hkv, grid, smem, s, tm_k, tm_v, p, seq_lens, out, B);
}

bi_status bi_silu_mul(const void *gu, void *h, int64_t M, int64_t F, void *stream)
{
    if (M < 0 || F < 0) return BI_ERR_INVALID_ARG;
    if (M > kI32Max || F > kI32Max) return BI_ERR_UNSUPPORTED;
    if (M == 0 || F == 0) return BI_OK;
    if (!gu || !h) return BI_ERR_INVALID_ARG;
    DeviceState *dev = nullptr;
    bi_status st = device_state(&dev);
    if (st != BI_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (F % 8 == 0) {
        if (!aligned16(gu) || !aligned16(h)) return BI_ERR_ALIGNMENT;
        const int64_t work = M * (F / 8);
        return launch(bi::silu_mul_vec_kernel, dim3(elementwise_blocks(work, dev->sms)), dim3(256), 0, s,
                      static_cast<const uint4 *>(gu), static_cast<uint4 *>(h), M, F);
    }
    return launch(bi::silu_mul_scalar_kernel, dim3(elementwise_blocks(M * F, dev->sms)), dim3(256), 0, s,
                  static_cast<const __nv_bfloat16 *>(gu), static_cast<__nv_bfloat16 *>(h), M, F);
}

bi_status bi_get_device_status(void *stream, int32_t *out)
{
    if (!out) return BI_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return BI_ERR_CUDA;
    int32_t v = 0;
    if (cudaMemcpyFromSymbol(&v, g_bi_status, sizeof v) != cudaSuccess) return BI_ERR_CUDA;
    const int32_t zero = 0;
    if (cudaMemcpyToSymbol(g_bi_status, &zero, sizeof zero) != cudaSuccess) return BI_ERR_CUDA;
    *out = v;
    return BI_OK;
}

bi_status bi_selftest_wait_timeout(int64_t limit_ns, void *stream)
{
    if (limit_ns < 1000 || limit_ns > 10000000000ll) return BI_ERR_INVALID_ARG;
    DeviceState *dev = nullptr;
    bi_status st = device_state(&dev);
    if (st != BI_OK) return st;
    return launch(selftest_wait_kernel, dim3(1), dim3(32), 0, static_cast<cudaStream_t>(stream), dev->status,
                  (uint64_t)limit_ns);
}

const char *bi_status_string(bi_status status)
{
    switch (status) {
    case BI_OK: return "BI_OK";
    case BI_ERR_INVALID_ARG: return "BI_ERR_INVALID_ARG";
    case BI_ERR_UNSUPPORTED: return "BI_ERR_UNSUPPORTED";
    case BI_ERR_ALIGNMENT: return "BI_ERR_ALIGNMENT";
    case BI_ERR_CUDA: return "BI_ERR_CUDA";
    case BI_ERR_TIMEOUT: return "BI_ERR_TIMEOUT";
    }
    return "BI_ERR_UNKNOWN";
}

void bi_gemm_config(int64_t weight_rows, int32_t *bm, int32_t *bn, int32_t *bk, int32_t *stages, int32_t *mma_k)
{
    const bi::PairConfig c = weight_rows > 0 ? bi::pair_config(weight_rows, true) : bi::kPairWide;
    if (bm) *bm = bi::kPairBM;
    if (bn) *bn = c == bi::kPairNarrow ? bi::NarrowTile::kBN : c == bi::kPairMid ? bi::MidTile::kBN : bi::WideTile::kBN;
    if (stages)
        *stages = c == bi::kPairNarrow ? bi::NarrowTile::kStages : c == bi::kPairMid ? bi::MidTile::kStages
                                                                                      : bi::WideTile::kStages;
    if (bk)
        *bk = c == bi::kPairNarrow ? bi::NarrowTile::kStageK : c == bi::kPairMid ? bi::MidTile::kStageK
                                                                                  : bi::WideTile::kStageK;
    if (mma_k) *mma_k = bi::kMmaK;
}

void bi_tensor_map_cache_stats(int64_t *hits, int64_t *misses)
{
    std::lock_guard<std::mutex> lock(g_map_mu);
    if (hits) *hits = (int64_t)g_map_hits;
    if (misses) *misses = (int64_t)g_map_misses;
}

int32_t bi_version(void) { return 201; }

}  // extern "C"
