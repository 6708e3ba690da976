// calibration: cycles per tcgen05.mma (kind::f16, M=128, K=16) for SS / TS operands and N
#include <cstdio>
#include <cuda_runtime.h>
#include "sm100.cuh"
using namespace fa;

template <int N, bool TS>
__global__ void __launch_bounds__(128, 1) mma_bench(long long* out, int iters)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    __shared__ uint64_t bar;
    __shared__ uint32_t tslot;
    __shared__ int abort_f;
    // operands: A 128 rows x 64 bf16 (16 KB), B 256 rows x 64 bf16 (32 KB); contents irrelevant
    for (int i = threadIdx.x; i < (48 * 1024) / 16; i += 128)
        reinterpret_cast<uint4*>(smem)[i] = make_uint4(0x3f803f80u, 0u, 0x3f803f80u, 0u);
    fence_proxy_async_smem();
    if (threadIdx.x == 0) { mbar_init(&bar, 1); abort_f = 0; fence_barrier_init(); }
    if (threadIdx.x < 32) { tmem_alloc(&tslot, 512); tmem_relinquish(); }
    tc_fence_before(); __syncthreads(); tc_fence_after();
    const uint32_t tmem = tslot;
    if (threadIdx.x == 0) {
        const uint32_t sa = smem_u32(smem), sb = sa + 16384;
        const uint64_t da = sdesc_sw128(sa, 16, 1024), db = sdesc_sw128(sb, 16, 1024);
        const uint32_t id = idesc_bf16_f32(128, N, false, false);
        // warm up
        for (int i = 0; i < 16; ++i) {
            if (TS) mma_ts(tmem + 256, tmem + (uint32_t)((i & 3) * 8), db + (uint64_t)((i & 3) * 2), id, 1u);
            else mma_ss(tmem + 256, da + (uint64_t)((i & 3) * 2), db + (uint64_t)((i & 3) * 2), id, 1u);
        }
        mma_commit(&bar);
        mbar_wait_limited(&bar, 0, 2000000000ll);
        const long long t0 = clock64();
        for (int i = 0; i < iters; ++i) {
            if (TS) mma_ts(tmem + 256, tmem + (uint32_t)((i & 3) * 8), db + (uint64_t)((i & 3) * 2), id, 1u);
            else mma_ss(tmem + 256, da + (uint64_t)((i & 3) * 2), db + (uint64_t)((i & 3) * 2), id, 1u);
        }
        const long long t_issue = clock64();
        mma_commit(&bar);
        const bool ok = mbar_wait_limited(&bar, 1, 2000000000ll);
        const long long t1 = clock64();
        if (blockIdx.x == 0) { out[0] = t_issue - t0; out[1] = t1 - t0; out[2] = ok; }
    }
    tc_fence_before(); __syncthreads();
    if (threadIdx.x < 32) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

template <int N, bool TS>
void run(const char* name, long long* d, int sms)
{
    const int iters = 4096;
    auto k = mma_bench<N, TS>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
    k<<<sms, 128, 64 * 1024>>>(d, iters);
    cudaError_t e = cudaDeviceSynchronize();
    long long h[3];
    cudaMemcpy(h, d, sizeof h, cudaMemcpyDeviceToHost);
    const double ideal = 128.0 * N * 16 / 4096.0;
    printf("%-12s N=%3d  issue %.1f cyc/mma  complete %.1f cyc/mma  ideal %.1f  -> %.0f%% of peak  ok=%lld err=%s\n",
           name, N, (double)h[0] / iters, (double)h[1] / iters, ideal, 100.0 * ideal / ((double)h[1] / iters), h[2],
           cudaGetErrorString(e));
}

int main()
{
    long long* d;
    cudaMalloc(&d, 64);
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
    for (int s : {1, sms}) {
        printf("--- %d CTAs (one per SM)\n", s);
        run<64, false>("SS", d, s);
        run<128, false>("SS", d, s);
        run<256, false>("SS", d, s);
        run<64, true>("TS", d, s);
        run<128, true>("TS", d, s);
        run<256, true>("TS", d, s);
    }
    return 0;
}
