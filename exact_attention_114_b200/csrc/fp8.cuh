// fp8.cuh -- preparation of e4m3 inputs for the forward kernel.
//
// The P.V product of kind::f8f6f4 takes V as a K-major operand (keys
// contiguous), while V is stored with d contiguous.  fp8_vt_kernel writes
// V^T [B * Hkv, d, Nk_pad] once per call; keys Nk .. Nk_pad-1 are written as
// zero bytes so that a padded key contributes 0 * 0 to P.V (e4m3 0x7f would be
// a NaN).  Nk_pad is Nk rounded up to 16 so every V^T row starts 16-byte
// aligned for the tensor map.
#pragma once

#include <cstdint>

#include "sm100.cuh"

namespace fa {

// grid (Nk_pad / 64 rounded up, B * Hkv), 256 threads; D = 128
template <int D>
__global__ void __launch_bounds__(256) fp8_vt_kernel(const uint8_t* __restrict__ v, uint8_t* __restrict__ vt,
                                                     int Nk, int Nk_pad)
{
    __shared__ __align__(16) uint8_t tile[64][D + 16];   // 64 keys x D bytes (+16: fewer bank conflicts)
    griddep_launch_dependents();   // the forward may start its set-up
    const int kb = (int)blockIdx.x * 64;
    const size_t bh = blockIdx.y;
    const uint8_t* src = v + bh * (size_t)Nk * D;
    constexpr int kChunks = D / 16;   // 16-byte chunks of one key row
    for (int idx = threadIdx.x; idx < 64 * kChunks; idx += 256) {
        const int r = idx / kChunks, c = idx % kChunks;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (kb + r < Nk)
            val = *reinterpret_cast<const uint4*>(src + (size_t)(kb + r) * D + c * 16);
        *reinterpret_cast<uint4*>(&tile[r][c * 16]) = val;
    }
    __syncthreads();
    // thread -> (16-key group g, d row c): 16 key bytes of V^T row c
    uint8_t* dst = vt + bh * (size_t)D * Nk_pad;
    for (int idx = threadIdx.x; idx < 4 * D; idx += 256) {
        const int g = idx / D, c = idx % D;
        const int key0 = kb + 16 * g;
        if (key0 >= Nk_pad)
            continue;
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            w[q] = (uint32_t)tile[16 * g + 4 * q][c] | ((uint32_t)tile[16 * g + 4 * q + 1][c] << 8) |
                   ((uint32_t)tile[16 * g + 4 * q + 2][c] << 16) | ((uint32_t)tile[16 * g + 4 * q + 3][c] << 24);
        *reinterpret_cast<uint4*>(dst + (size_t)c * Nk_pad + key0) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

}  // namespace fa
