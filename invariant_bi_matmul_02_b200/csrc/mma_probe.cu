// mma_probe.cu -- measurement program: clock cycles per tcgen05.mma (kind::f16, bf16 inputs,
// fp32 accumulator, K = 16) issued back to back from shared memory, for the instruction shapes
// a batch-invariant GEMM tile could be built from.  One CTA (cta_group::1) or one CTA pair
// (cta_group::2) issues 4096 MMAs into one accumulator (or alternately two) and times them with
// clock64 up to the commit; the operands are zeros.  It prints cycles per MMA and the implied
// MAC/clk per SM.  Every wait is bounded (2 s).  Built by csrc/build.py, run by
// `bench.py --mma-probe`.
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
#include "ptx.cuh"

using namespace bi;

template <int CG, int M, int N, int NACC>
__global__ void __launch_bounds__(128, 1) probe(uint32_t iters, unsigned long long *out, int *status)
{
    extern __shared__ uint8_t raw[];
    uint8_t *sm = raw + ((1024u - (smem_addr(raw) & 1023u)) & 1023u);
    __shared__ uint64_t bar;
    __shared__ uint32_t holder;
    constexpr int ROWS_A = CG == 2 ? M / 2 : M;
    constexpr int ROWS_B = CG == 2 ? N / 2 : N;
    uint8_t *A = sm;
    uint8_t *B = sm + ROWS_A * 128;
    for (int i = threadIdx.x; i < (ROWS_A + ROWS_B) * 128 / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(sm)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
    const uint32_t rank = CG == 2 ? cluster_ctarank() : 0;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    if (threadIdx.x < 32) {
        if (CG == 2) { tmem_alloc_pair(&holder, 512); tmem_relinquish_pair(); }
        else { tmem_alloc(&holder, 512); tmem_relinquish(); }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (CG == 2) cluster_sync_all();
    tc_fence_after_sync();
    const uint32_t tmem = holder;
    if (threadIdx.x == 0 && rank == 0) {
        const uint32_t idesc = mma_idesc_bf16(M, N, 0, 0);
        const uint64_t a = sw128_desc(smem_addr(A), 16, 1024), b = sw128_desc(smem_addr(B), 16, 1024);
        const unsigned long long t0 = clock64();
        for (uint32_t i = 0; i < iters; ++i) {
            const uint32_t d = tmem + (NACC > 1 ? (i % NACC) * 256 : 0);
            if (CG == 2) tc_mma_bf16_pair(d, a, b, idesc, i >= NACC ? 1u : 0u);
            else tc_mma_bf16(d, a, b, idesc, i >= NACC ? 1u : 0u);
        }
        if (CG == 2) tc_commit_pair_mc(&bar, 0x3);
        else tc_commit(&bar);
        const uint32_t ba = smem_addr(&bar);
        const uint64_t g0 = global_timer_ns();
        bool ok = false;
        while (global_timer_ns() - g0 < 2000000000ull) {
            if (mbar_try_wait(ba, 0)) { ok = true; break; }
        }
        const unsigned long long t1 = clock64();
        if (!ok) *status = 1;
        out[0] = t1 - t0;
    }
    if (CG == 2 && threadIdx.x == 0 && rank == 1) {
        const uint32_t ba = smem_addr(&bar);
        const uint64_t g0 = global_timer_ns();
        while (!mbar_try_wait(ba, 0) && global_timer_ns() - g0 < 2000000000ull) {
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (CG == 2) cluster_sync_all();
    if (threadIdx.x < 32) {
        tc_fence_after_sync();
        if (CG == 2) tmem_dealloc_pair(tmem, 512);
        else tmem_dealloc(tmem, 512);
    }
}

template <int CG, int M, int N, int NACC>
void run(const char *name)
{
    unsigned long long *d_out;
    int *d_st;
    cudaMalloc(&d_out, 8);
    cudaMalloc(&d_st, 4);
    cudaMemset(d_st, 0, 4);
    const int smem = (M + N) * 128 + 1024;
    cudaFuncSetAttribute(probe<CG, M, N, NACC>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(CG, 1, 1);
    cfg.blockDim = dim3(128, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr{};
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = CG;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    const uint32_t iters = 4096;
    for (int rep = 0; rep < 3; ++rep) {
        cudaError_t e = cudaLaunchKernelEx(&cfg, probe<CG, M, N, NACC>, iters, d_out, d_st);
        if (e != cudaSuccess) { printf("%s launch error %s\n", name, cudaGetErrorString(e)); return; }
        e = cudaDeviceSynchronize();
        if (e != cudaSuccess) { printf("%s error %s\n", name, cudaGetErrorString(e)); return; }
    }
    unsigned long long cyc = 0;
    int st = 0;
    cudaMemcpy(&cyc, d_out, 8, cudaMemcpyDeviceToHost);
    cudaMemcpy(&st, d_st, 4, cudaMemcpyDeviceToHost);
    const double per = (double)cyc / iters;
    const double macs_per_sm = (double)M * N * 16 / CG;
    printf("{\"shape\": \"%s\", \"cycles_per_mma\": %.1f, \"mac_per_clk_per_sm\": %.0f, \"timed_out\": %d}\n", name,
           per, macs_per_sm / per, st);
    cudaFree(d_out);
    cudaFree(d_st);
}

int main()
{
    run<1, 128, 256, 1>("cg1 M128 N256");
    run<1, 128, 128, 1>("cg1 M128 N128");
    run<1, 128, 64, 1>("cg1 M128 N64");
    run<1, 128, 128, 2>("cg1 M128 N128 2acc");
    run<1, 64, 256, 1>("cg1 M64 N256");
    run<1, 64, 128, 1>("cg1 M64 N128");
    run<2, 256, 256, 1>("cg2 M256 N256");
    run<2, 256, 128, 1>("cg2 M256 N128");
    run<2, 256, 128, 2>("cg2 M256 N128 2acc");
    run<2, 256, 64, 1>("cg2 M256 N64");
    run<2, 128, 256, 1>("cg2 M128 N256");
    run<2, 128, 128, 1>("cg2 M128 N128");
    return 0;
}
