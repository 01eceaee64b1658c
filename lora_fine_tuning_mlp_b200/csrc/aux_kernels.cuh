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

// Warp-cooperative dequantisation.  Packed codes [rows, cols/2] bytes and
// scales [rows, cols/64] are row-major, so flat block i (64 elements, one
// scale) has its 32 code bytes at byte 32*i and its outputs at element 64*i.
// A warp takes kDqPasses passes of 8 consecutive blocks (512 elements) per
// iteration:
//  1. every lane issues its loads first (the scale of block L/4 and two
//     4-byte code words per pass), so their latencies overlap;
//  2. lane L computes magnitudes L%4 and L%4+4 (and 8 when L%4 = 0) of block
//     L/4 with dequant_one and writes them to that block's 16-entry table in
//     shared memory at the code's two's-complement nibble, the negative code
//     -m at nibble 16-m with the sign bit flipped.  This equals
//     dequant_one(-m, scale) bit for bit: q*scale is exact and round to
//     nearest even is symmetric in sign, fl(-x) = -fl(x);
//  3. lane L converts the 8 codes of elements 8L .. 8L+7 and 256+8L ..
//     256+8L+7 of each pass with table lookups: one 4-byte load and one
//     16-byte store each, so a warp's loads and stores cover contiguous
//     128 B and 512 B spans.
constexpr int kDqWarps = 8;
#ifndef LMLP_DQ_PASSES
#define LMLP_DQ_PASSES 2
#endif
constexpr int kDqPasses = LMLP_DQ_PASSES;

__global__ void __launch_bounds__(kDqWarps * 32) dequant_int4_kernel(const uint32_t* __restrict__ packed,
                                                                     const __half* __restrict__ scales,
                                                                     long long nblocks,
                                                                     __nv_bfloat16* __restrict__ w) {
    __shared__ uint32_t tab[kDqWarps][kDqPasses * 8 * 16];
    const int lane = threadIdx.x & 31;
    const int wid = threadIdx.x >> 5;
    uint32_t* t = tab[wid];
    const long long nchunks = (nblocks + 8 * kDqPasses - 1) / (8 * kDqPasses);
    for (long long c = static_cast<long long>(blockIdx.x) * kDqWarps + wid; c < nchunks;
         c += static_cast<long long>(gridDim.x) * kDqWarps) {
        const long long cb = c * (8 * kDqPasses);  // first block of this iteration
        float sc[kDqPasses];
        uint32_t word[kDqPasses][2];
#pragma unroll
        for (int p = 0; p < kDqPasses; ++p) {
            const long long b = cb + p * 8 + (lane >> 2);
            sc[p] = b < nblocks ? __half2float(scales[b]) : 0.0f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int e0 = h * 256 + lane * 8;
                const long long e = (cb + p * 8) * 64 + e0;
                word[p][h] = (cb + p * 8 + (e0 >> 6)) < nblocks ? packed[e >> 3] : 0u;
            }
        }
#pragma unroll
        for (int p = 0; p < kDqPasses; ++p) {
            uint32_t* tb = t + (p * 8 + (lane >> 2)) * 16;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int m = (lane & 3) + 4 * j;
                const uint32_t v = bf16_bits(dequant_one(m, sc[p]));
                tb[m] = v;
                if (m != 0) tb[16 - m] = v ^ 0x8000u;
            }
            if ((lane & 3) == 0) tb[8] = bf16_bits(dequant_one(8, sc[p])) ^ 0x8000u;
        }
        __syncwarp();
#pragma unroll
        for (int p = 0; p < kDqPasses; ++p) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int e0 = h * 256 + lane * 8;
                const int lb = p * 8 + (e0 >> 6);
                if (cb + lb < nblocks) {
                    const uint32_t* tb = t + lb * 16;
                    const uint32_t wd = word[p][h];
                    uint32_t o[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        o[k] = tb[(wd >> (8 * k)) & 0xFu] | (tb[(wd >> (8 * k + 4)) & 0xFu] << 16);
                    *reinterpret_cast<uint4*>(w + (cb + p * 8) * 64 + e0) = make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
        }
        __syncwarp();
    }
}

}  // namespace lmlp
