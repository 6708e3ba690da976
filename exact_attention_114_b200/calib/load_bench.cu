// calibration: the forward kernel's MMA sequence (one issuing warp, fwd-like commits) while
// eight other warps run a chosen load: MUFU, FMA, tcgen05.ld / st on the S columns, or a
// softmax-like mix.  Reports MMA cycles per block of 32 MMAs (ideal 2048).
#include <cstdio>
#include <cuda_runtime.h>
#include "sm100.cuh"
using namespace fa;

template <int LOAD, int SMSP_MASK = 15, int MMA_WARP = 9>
__global__ void __launch_bounds__(384, 1) load_bench(long long* out, int iters, int load_iters)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    __shared__ uint64_t bar;
    __shared__ uint64_t dummy[4];
    __shared__ uint32_t tslot;
    for (int i = threadIdx.x; i < (192 * 1024) / 16; i += 384)
        reinterpret_cast<uint4*>(smem)[i] = make_uint4(0x3f803f80u, 0u, 0x3f803f80u, 0u);
    fence_proxy_async_smem();
    if (threadIdx.x == 0) { mbar_init(&bar, 1); for (int i = 0; i < 4; ++i) mbar_init(&dummy[i], 1); fence_barrier_init(); }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == MMA_WARP) { tmem_alloc(&tslot, 512); tmem_relinquish(); }
    tc_fence_before(); __syncthreads(); tc_fence_after();
    const uint32_t tmem = tslot;
    if (warp == MMA_WARP && lane == 0) {
        const uint32_t sq = smem_u32(smem), skv = sq + 65536;
        const uint64_t dq = sdesc_sw128(sq, 16, 1024), dk = sdesc_sw128(skv, 16, 1024),
                       dv = sdesc_sw128(skv, 16384, 1024);
        const uint32_t idS = idesc_bf16_f32(128, 128, false, false), idPV = idesc_bf16_f32(128, 128, false, true);
        long long t0 = 0;
        for (int j = -2; j < iters; ++j) {
            if (j == 0) t0 = clock64();
            const uint32_t slotK = (uint32_t)(((2 * j + 8) % 4) * 32768), slotV = (uint32_t)(((2 * j + 9) % 4) * 32768);
            for (int t = 0; t < 2; ++t) {
                const uint32_t tS = tmem + 128u * t, tO = tmem + 256u + 128u * t;
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tO, tS + (uint32_t)(kk * 8), dv + (uint64_t)((slotV + kk * 2048) >> 4), idPV, 1u);
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t o = (uint32_t)((kk >> 2) * 16384 + (kk & 3) * 32);
                    mma_ss(tS, dq + (uint64_t)((t * 32768 + o) >> 4), dk + (uint64_t)((slotK + o) >> 4), idS,
                           kk > 0 ? 1u : 0u);
                }
                mma_commit(&dummy[t]);
                mma_commit(&dummy[2 + t]);
            }
        }
        mma_commit(&bar);
        mbar_wait_limited(&bar, 0, 2000000000ll);
        const long long t1 = clock64();
        if (blockIdx.x == 0) out[0] = t1 - t0;
    } else if ((MMA_WARP == 9 ? warp < 8 : (warp >= 4 && warp < 12)) && LOAD > 0 && ((SMSP_MASK >> (warp & 3)) & 1)) {
        const int t = (MMA_WARP == 9 ? warp : warp - 4) >> 2;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + 128u * (uint32_t)t;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = 0.001f * (float)(i + lane);
        const long long t0 = clock64();
        for (int it = 0; it < load_iters; ++it) {
            if (LOAD == 3 || LOAD == 5 || LOAD == 6) {
                uint32_t r[128];
                tmem_ld128(tS, r);
#pragma unroll
                for (int i = 0; i < 128; ++i) x[i & 15] += __uint_as_float(r[i]) * 1e-30f;
            }
            if (LOAD == 1 || LOAD == 6) {
#pragma unroll
                for (int k = 0; k < 6; ++k)
#pragma unroll
                    for (int i = 0; i < 16; ++i) x[i] = ex2_approx(x[i] * -0.5f);
            }
            if (LOAD == 2) {
#pragma unroll
                for (int k = 0; k < 24; ++k)
#pragma unroll
                    for (int i = 0; i < 16; ++i) x[i] = fmaf(x[i], 0.999f, 0.001f);
            }
            if (LOAD == 7) {   // packed f32x2 FMA
#pragma unroll
                for (int k = 0; k < 24; ++k)
#pragma unroll
                    for (int i = 0; i < 16; i += 2) {
                        float2 v = ffma2(make_float2(x[i], x[i + 1]), make_float2(0.999f, 0.999f),
                                         make_float2(0.001f, 0.001f));
                        x[i] = v.x; x[i + 1] = v.y;
                    }
            }
            if (LOAD == 8) {   // integer ALU
                uint32_t u[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) u[i] = __float_as_uint(x[i]);
#pragma unroll
                for (int k = 0; k < 24; ++k)
#pragma unroll
                    for (int i = 0; i < 16; ++i) u[i] = (u[i] ^ (u[(i + 1) & 15] >> 3)) + 0x9e3779b9u;
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = __uint_as_float(u[i] & 0x3f7fffffu);
            }
            if (LOAD == 9) {   // max (FMNMX)
#pragma unroll
                for (int k = 0; k < 24; ++k)
#pragma unroll
                    for (int i = 0; i < 16; ++i) x[i] = fmax3(x[i], x[(i + 3) & 15], x[(i + 7) & 15]);
            }
            if (LOAD == 10) {  // the same S bytes in four x32 loads
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t r[32];
                    tmem_ld32(tS + (uint32_t)(32 * q), r);
#pragma unroll
                    for (int i = 0; i < 32; ++i) x[i & 15] += __uint_as_float(r[i]) * 1e-30f;
                }
            }
            if (LOAD == 4 || LOAD == 5 || LOAD == 6) {
                uint32_t w[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) w[i] = pack_bf16x2(x[i & 15], x[(i + 1) & 15]);
                tmem_st32(tS, w);
                tmem_st32(tS + 32u, w);
                tmem_st_wait();
            }
        }
        const long long t1 = clock64();
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) s += x[i];
        if (blockIdx.x == 0 && lane == 0) out[1 + (MMA_WARP == 9 ? warp : warp - 4)] = (t1 - t0) + (s == 12345.f ? 1 : 0);
    }
    tc_fence_before(); __syncthreads();
    if (warp == MMA_WARP) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

template <int LOAD, int SMSP_MASK = 15, int MMA_WARP = 9>
void run(const char* name, long long* d, int sms, int load_iters)
{
    const int iters = 512;
    auto k = load_bench<LOAD, SMSP_MASK, MMA_WARP>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 194 * 1024);
    cudaMemset(d, 0, 16 * sizeof(long long));
    k<<<sms, 384, 194 * 1024>>>(d, iters, load_iters);
    cudaError_t e = cudaDeviceSynchronize();
    long long h[16] = {};
    cudaMemcpy(h, d, sizeof h, cudaMemcpyDeviceToHost);
    printf("%-34s MMA %.0f cyc/block (ideal 2048) -> %3.0f%%   load warp time %.2f x MMA time  err=%s\n", name,
           (double)h[0] / iters, 100.0 * 2048.0 / ((double)h[0] / iters),
           (double)(h[1] ? h[1] : h[2] ? h[2] : h[3] ? h[3] : h[4]) / (double)h[0],
           cudaGetErrorString(e));
}

int main()
{
    long long* d;
    cudaMalloc(&d, 16 * sizeof(long long));
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
    run<0>("no load", d, sms, 0);
    run<2>("FFMA (8 warps), MMA warp 9", d, sms, 3000);
    run<2, 15, 1>("FFMA (8 warps), MMA warp 1", d, sms, 3000);
    run<2, 2>("FFMA own SMSP, MMA warp 9", d, sms, 6000);
    run<2, 2, 1>("FFMA own SMSP, MMA warp 1", d, sms, 6000);
    run<3>("ld x128, MMA warp 9", d, sms, 3000);
    run<3, 15, 1>("ld x128, MMA warp 1", d, sms, 3000);
    run<6>("softmax-like, MMA warp 9", d, sms, 1500);
    run<6, 15, 1>("softmax-like, MMA warp 1", d, sms, 1500);
    run<8>("integer ALU, MMA warp 9", d, sms, 6000);
    run<8, 15, 1>("integer ALU, MMA warp 1", d, sms, 6000);
    return 0;
}
