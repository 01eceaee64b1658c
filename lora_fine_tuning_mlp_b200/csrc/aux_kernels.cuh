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

// Each thread expands one 32-bit word (8 codes) into 8 bf16 (one 16-byte store).
__global__ void __launch_bounds__(256) dequant_int4_kernel(const uint32_t* __restrict__ packed,
                                                           const __half* __restrict__ scales, long long rows,
                                                           long long cols, __nv_bfloat16* __restrict__ w) {
    const long long words_per_row = cols / 8;
    const long long total = rows * words_per_row;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long row = i / words_per_row;
        const long long c8 = (i - row * words_per_row) * 8;
        const uint32_t word = packed[i];
        const float sc = __half2float(scales[row * (cols / 64) + c8 / 64]);
        __align__(16) __nv_bfloat16 v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            int q = static_cast<int>((word >> (4 * e)) & 0xFu);
            q = q >= 8 ? q - 16 : q;
            v[e] = dequant_one(q, sc);
        }
        *reinterpret_cast<uint4*>(w + row * cols + c8) = *reinterpret_cast<const uint4*>(v);
    }
}

}  // namespace lmlp
