// The block-int4 dequantisation of the frozen weights.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

namespace lmlp {

// Block-int4 weight element -> bf16: (fp32(q) * fp32(scale)) / 7 in IEEE fp32
// (the product is exact; the divide is correctly rounded), then round to
// nearest-even bf16.
__device__ __forceinline__ __nv_bfloat16 dequant_one(int q, float scale) {
    return __float2bfloat16_rn(__fdiv_rn(__fmul_rn(static_cast<float>(q), scale), 7.0f));
}

__device__ __forceinline__ uint32_t bf16_bits(__nv_bfloat16 v) {
    return static_cast<uint32_t>(__bfloat16_as_ushort(v));
}

// One thread per 64-element block (one scale): the magnitudes for |q| = 0..8
// are computed once with dequant_one, then every code is a lookup plus a sign
// flip.  This equals dequant_one(q, scale) bit for bit, because q*scale is
// exact and round-to-nearest-even is symmetric in sign: fl(-x) = -fl(x).
// Packed rows are [rows, cols/2] bytes, scales [rows, cols/64], both row-major,
// so block i's 32 code bytes start at byte 32*i and its outputs at element 64*i.
__global__ void __launch_bounds__(256) dequant_int4_kernel(const uint4* __restrict__ packed,
                                                           const __half* __restrict__ scales, long long rows,
                                                           long long cols, __nv_bfloat16* __restrict__ w) {
    const long long total = rows * (cols / 64);
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const float sc = __half2float(scales[i]);
        uint32_t mag[9];
#pragma unroll
        for (int m = 0; m < 9; ++m) mag[m] = bf16_bits(dequant_one(m, sc));
        const uint4 p0 = packed[2 * i], p1 = packed[2 * i + 1];
        const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
        uint4* out = reinterpret_cast<uint4*>(w + i * 64);
#pragma unroll
        for (int wd = 0; wd < 8; ++wd) {
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                uint32_t half2[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int nib = static_cast<int>((words[wd] >> (8 * e + 4 * h)) & 0xFu);
                    const int q = nib >= 8 ? nib - 16 : nib;
                    const uint32_t m = mag[q < 0 ? -q : q];
                    half2[h] = q < 0 ? (m ^ 0x8000u) : m;
                }
                o[e] = half2[0] | (half2[1] << 16);
            }
            out[wd] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

}  // namespace lmlp
