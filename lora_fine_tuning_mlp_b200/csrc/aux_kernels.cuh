// The block-int4 dequantisation of the frozen weights.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "f32x2.cuh"

namespace lmlp {

// x / 7 correctly rounded in fp32 for x = fp32(q) * fp32(scale), q an int4
// code and scale an fp16 (so x has at most 14 significant bits): the product
// y = x * fl(1/7), then one correction by the exact residual e = x - 7y,
// y + e * fl(1/7) rounded once by the FMA.  Checked exhaustively with exact
// rational arithmetic against the correctly rounded quotient for every code
// 1..8 and every positive finite fp16 scale (253,944 cases); negative x
// follow from the sign symmetry of round-to-nearest-even.  It is evaluated
// from -x (y = (-x)(-1/7), e' = 7y + (-x) = -e, result = e'(-1/7) + y): the
// same values, and a zero x keeps its sign (a residual sum of +0 and -0
// would otherwise turn -0 into +0).  Two lanes at a time; neg_x = -x.
__device__ __forceinline__ uint64_t div7_rn_neg2(uint64_t neg_x) {
    const uint64_t nr = f2_packf(-1.0f / 7.0f, -1.0f / 7.0f);  // -fl(1/7)
    const uint64_t seven = f2_packf(7.0f, 7.0f);
    const uint64_t y = f2_mul(neg_x, nr);
    const uint64_t e = f2_fma(y, seven, neg_x);
    return f2_fma(e, nr, y);
}

// fp32 bits of 2^23 + (q + 8) for the two's-complement nibble n (0..15) of
// code q: q + 8 = n ^ 8, and 2^23 + m is exact in fp32 for m < 2^23.
__device__ __forceinline__ uint32_t nibble_bits(uint32_t n) { return 0x4B000000u | (n ^ 8u); }

// Eight codes (one 4-byte word, element 2k in the low nibble of byte k) ->
// eight bf16 values (fp32(q) * fp32(scale)) / 7, rounded to nearest-even
// bf16.  The product is exact and the quotient correctly rounded (div7_rn);
// a non-finite scale takes IEEE's own divide (inf / 7 = inf, NaN stays NaN).
template <bool kFinite>
__device__ __forceinline__ uint4 dequant_word(uint32_t word, float scale) {
    uint32_t o[4];
    const uint64_t c8 = f2_packf(8388616.0f, 8388616.0f);  // 2^23 + 8
    const uint64_t ns2 = f2_packf(-scale, -scale);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t bl = nibble_bits((word >> (8 * j)) & 0xFu);
        const uint32_t bh = nibble_bits((word >> (8 * j + 4)) & 0xFu);
        // (2^23 + q + 8) - (2^23 + 8) = q exactly (+0 for code 0); q * (-scale)
        // is -(q * scale) exactly, the sign of a zero included
        const uint64_t neg_x = f2_mul(f2_sub(f2_pack(bl, bh), c8), ns2);
        float lo, hi;
        if (kFinite) {
            f2_unpack(div7_rn_neg2(neg_x), lo, hi);
        } else {
            f2_unpack(neg_x, lo, hi);
            lo = __fdiv_rn(lo, -7.0f);
            hi = __fdiv_rn(hi, -7.0f);
        }
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        o[j] = *reinterpret_cast<uint32_t*>(&h);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// One thread per 8-code group per step: packed codes [rows, cols/2] bytes
// and scales [rows, cols/64] are row-major, so group g (elements 8g .. 8g+7)
// is the 4-byte code word g, its scale is scale g/8 and its output the 16
// bytes at element 8g.  A CTA takes kDqUnroll x 256 consecutive groups and
// issues all their loads before converting, so a warp's loads and stores
// cover contiguous 128-byte and 512-byte spans and several are in flight.
// Everything runs on the FMA and integer pipes, two lanes per fp32
// instruction.
constexpr int kDqThreads = 256;
constexpr int kDqUnroll = 4;

__global__ void __launch_bounds__(kDqThreads) dequant_int4_kernel(const uint32_t* __restrict__ packed,
                                                                  const __half* __restrict__ scales,
                                                                  long long ngroups,
                                                                  __nv_bfloat16* __restrict__ w) {
    const long long span = static_cast<long long>(kDqThreads) * kDqUnroll;
    for (long long g0 = static_cast<long long>(blockIdx.x) * span + threadIdx.x; g0 < ngroups;
         g0 += static_cast<long long>(gridDim.x) * span) {
        uint32_t word[kDqUnroll];
        float sc[kDqUnroll];
#pragma unroll
        for (int k = 0; k < kDqUnroll; ++k) {
            const long long g = g0 + k * kDqThreads;
            word[k] = g < ngroups ? __ldcs(packed + g) : 0u;
            sc[k] = g < ngroups ? __half2float(scales[g >> 3]) : 0.0f;
        }
#pragma unroll
        for (int k = 0; k < kDqUnroll; ++k) {
            const long long g = g0 + k * kDqThreads;
            if (g >= ngroups) break;
            const uint4 v = fabsf(sc[k]) <= 65504.0f ? dequant_word<true>(word[k], sc[k])  // finite scale
                                                     : dequant_word<false>(word[k], sc[k]);
            __stcs(reinterpret_cast<uint4*>(w) + g, v);
        }
    }
}

}  // namespace lmlp
