// Small bandwidth-bound kernels around the GEMMs: the deterministic split-K
// reduction that finishes every rank-r product, the transpose of the adapter
// B matrices into K-major operands, and the block-int4 dequantisation.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

namespace lmlp {

constexpr int kRedRows = 32;
constexpr int kRedMaxCols = 256;

// Sum `splits` fp32 partial tiles P[s][m][col0 + j] in split order, scale, and
// write bf16 to up to two places: row-major rm[m][j] and transposed tr[j][m].
// One block handles 32 rows and all `ncols` (<= 256) columns.
__global__ void __launch_bounds__(256) reduce_partials_kernel(const float* __restrict__ P, int splits,
                                                              long long split_stride, int M, int ldp, int col0,
                                                              int ncols, float scale, __nv_bfloat16* rm,
                                                              long long ld_rm, __nv_bfloat16* tr, long long ld_tr) {
    __shared__ float tile[kRedRows][kRedMaxCols + 1];
    const int m0 = blockIdx.x * kRedRows;
    for (int i = threadIdx.x; i < kRedRows * ncols; i += blockDim.x) {
        const int rr = i / ncols, j = i - rr * ncols;
        const int m = m0 + rr;
        float acc = 0.0f;
        if (m < M) {
            const float* p = P + static_cast<long long>(m) * ldp + col0 + j;
            for (int s = 0; s < splits; ++s) acc += p[s * split_stride];
        }
        acc *= scale;
        tile[rr][j] = acc;
        if (rm != nullptr && m < M) rm[static_cast<long long>(m) * ld_rm + j] = __float2bfloat16_rn(acc);
    }
    if (tr == nullptr) return;
    __syncthreads();
    for (int i = threadIdx.x; i < kRedRows * ncols; i += blockDim.x) {
        const int j = i / kRedRows, rr = i - j * kRedRows;
        const int m = m0 + rr;
        if (m < M) tr[static_cast<long long>(j) * ld_tr + m] = __float2bfloat16_rn(tile[rr][j]);
    }
}

// out[c][r] = in[r][c] for a bf16 [R, C] matrix with C <= 256 (an adapter B).
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const __nv_bfloat16* __restrict__ in, int R, int C,
                                                             __nv_bfloat16* __restrict__ out) {
    __shared__ __nv_bfloat16 tile[kRedRows][kRedMaxCols + 2];
    const int r0 = blockIdx.x * kRedRows;
    for (int i = threadIdx.x; i < kRedRows * C; i += blockDim.x) {
        const int rr = i / C, c = i - rr * C;
        if (r0 + rr < R) tile[rr][c] = in[static_cast<long long>(r0 + rr) * C + c];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kRedRows * C; i += blockDim.x) {
        const int c = i / kRedRows, rr = i - c * kRedRows;
        if (r0 + rr < R) out[static_cast<long long>(c) * R + r0 + rr] = tile[rr][c];
    }
}

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
