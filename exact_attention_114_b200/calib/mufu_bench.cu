// calibration: MUFU ex2 throughput per SM per clock for f32, f16x2, bf16x2
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

template <int KIND>   // 0 f32, 1 f16x2, 2 bf16x2
__global__ void __launch_bounds__(512) mufu(float* out, int iters, long long* cyc)
{
    float a[8]; uint32_t h[8];
    for (int i = 0; i < 8; ++i) { a[i] = -0.001f * (threadIdx.x + i); h[i] = 0xBC00BC00u + i; }
    __syncthreads();
    long long t0 = clock64();
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (KIND == 0) asm volatile("ex2.approx.ftz.f32 %0, %0;" : "+f"(a[i]));
            else if (KIND == 1) asm volatile("ex2.approx.f16x2 %0, %0;" : "+r"(h[i]));
            else asm volatile("ex2.approx.ftz.bf16x2 %0, %0;" : "+r"(h[i]));
        }
    }
    __syncthreads();
    long long t1 = clock64();
    float s = 0.f; for (int i = 0; i < 8; ++i) s += a[i] + __uint_as_float(h[i]);
    if (s == 123.f) out[0] = s;
    if (threadIdx.x == 0 && blockIdx.x == 0) *cyc = t1 - t0;
}

template <int KIND>
void run(const char* name, float* d, long long* c, int sms)
{
    const int iters = 4096, threads = 512;
    mufu<KIND><<<sms, threads>>>(d, iters, c);
    cudaError_t e = cudaDeviceSynchronize();
    long long h = 0; cudaMemcpy(&h, c, sizeof h, cudaMemcpyDeviceToHost);
    const double instr = (double)threads * iters * 8;            // per SM (one CTA per SM)
    const double vals = instr * (KIND == 0 ? 1 : 2);
    printf("%-8s %.2f MUFU lane-ops/clk/SM, %.2f exp values/clk/SM  (%s)\n", name, instr / h, vals / h, cudaGetErrorString(e));
}

int main()
{
    float* d; long long* c; cudaMalloc(&d, 64); cudaMalloc(&c, 64);
    int sms = 0; cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
    run<0>("f32", d, c, sms); run<1>("f16x2", d, c, sms); run<2>("bf16x2", d, c, sms);
    return 0;
}
