// RMSNorm over the rows of a bf16 matrix [N, d] (d a multiple of 8), forward
// and backward, for the pre-norm MLP block.  Memory-bound: one warp per row,
// 16-byte coalesced loads and stores, fp32 arithmetic.  Per row x with frozen
// gain gamma:
//   rstd = 1 / sqrt(mean(x^2) + eps),   y = x * rstd * gamma
//   dx   = rstd * (dy*gamma - x_hat * mean(dy*gamma*x_hat)),  x_hat = x * rstd
// The backward takes rstd from the forward instead of recomputing the mean of
// squares ("Unsloth支持哪些模型？主流LLM兼容性一览", section 4.2).  Sums run in a
// fixed per-lane order followed by a fixed butterfly across the warp, so the
// results are deterministic.
//
// For the block with gamma folded into the gate/up weights: with y ==
// nullptr the forward only computes rstd, and with gamma == nullptr both
// passes take gamma = 1 (the backward then maps dy*gamma, computed by the dX
// GEMM on the folded weights, to dx).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace lmlp {

constexpr int kRmsWarps = 8;
constexpr uint32_t kBf16One2 = 0x3F803F80u;  // two bf16 ones

__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ uint4 pack8(const float* f) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// y = RMSNorm(x) * gamma.  With rstd_in == nullptr the kernel computes rstd
// (and writes it to rstd_out if that is not null); otherwise it reuses
// rstd_in, which reproduces the forward's y bit for bit.
__global__ void __launch_bounds__(kRmsWarps * 32) rmsnorm_fwd_kernel(const __nv_bfloat16* __restrict__ x,
                                                                     const __nv_bfloat16* __restrict__ gamma,
                                                                     long long N, int d, float eps,
                                                                     const float* __restrict__ rstd_in,
                                                                     float* __restrict__ rstd_out,
                                                                     __nv_bfloat16* __restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int nc = d >> 3;
    const uint4* g4 = reinterpret_cast<const uint4*>(gamma);
    for (long long row = static_cast<long long>(blockIdx.x) * kRmsWarps + (threadIdx.x >> 5); row < N;
         row += static_cast<long long>(gridDim.x) * kRmsWarps) {
        const uint4* x4 = reinterpret_cast<const uint4*>(x + row * d);
        float r;
        if (rstd_in != nullptr) {
            r = rstd_in[row];
        } else {
            float ss = 0.0f;
            for (int c = lane; c < nc; c += 32) {
                float f[8];
                unpack8(__ldg(x4 + c), f);
#pragma unroll
                for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
            }
            ss = warp_sum(ss);
            r = 1.0f / sqrtf(ss / static_cast<float>(d) + eps);
            if (lane == 0 && rstd_out != nullptr) rstd_out[row] = r;
        }
        if (y == nullptr) continue;
        uint4* y4 = reinterpret_cast<uint4*>(y + row * d);
        for (int c = lane; c < nc; c += 32) {
            float f[8], g[8];
            unpack8(__ldg(x4 + c), f);
            unpack8(gamma != nullptr ? __ldg(g4 + c) : make_uint4(kBf16One2, kBf16One2, kBf16One2, kBf16One2), g);
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = f[i] * r * g[i];
            y4[c] = pack8(f);
        }
    }
}

// dx for upstream dy (the gradient of y), reusing the forward's rstd.
__global__ void __launch_bounds__(kRmsWarps * 32) rmsnorm_bwd_kernel(const __nv_bfloat16* __restrict__ x,
                                                                     const __nv_bfloat16* __restrict__ gamma,
                                                                     const float* __restrict__ rstd,
                                                                     const __nv_bfloat16* __restrict__ dy,
                                                                     long long N, int d,
                                                                     __nv_bfloat16* __restrict__ dx) {
    const int lane = threadIdx.x & 31;
    const int nc = d >> 3;
    const uint4* g4 = reinterpret_cast<const uint4*>(gamma);
    for (long long row = static_cast<long long>(blockIdx.x) * kRmsWarps + (threadIdx.x >> 5); row < N;
         row += static_cast<long long>(gridDim.x) * kRmsWarps) {
        const uint4* x4 = reinterpret_cast<const uint4*>(x + row * d);
        const uint4* d4 = reinterpret_cast<const uint4*>(dy + row * d);
        const float r = rstd[row];
        float dot = 0.0f;
        const uint4 ones = make_uint4(kBf16One2, kBf16One2, kBf16One2, kBf16One2);
        for (int c = lane; c < nc; c += 32) {
            float f[8], g[8], e[8];
            unpack8(__ldg(x4 + c), f);
            unpack8(gamma != nullptr ? __ldg(g4 + c) : ones, g);
            unpack8(__ldg(d4 + c), e);
#pragma unroll
            for (int i = 0; i < 8; ++i) dot = fmaf(e[i] * g[i], f[i] * r, dot);
        }
        const float m = warp_sum(dot) / static_cast<float>(d);
        uint4* o4 = reinterpret_cast<uint4*>(dx + row * d);
        for (int c = lane; c < nc; c += 32) {
            float f[8], g[8], e[8];
            unpack8(__ldg(x4 + c), f);
            unpack8(gamma != nullptr ? __ldg(g4 + c) : ones, g);
            unpack8(__ldg(d4 + c), e);
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = r * (e[i] * g[i] - f[i] * r * m);
            o4[c] = pack8(f);
        }
    }
}

// Row-per-CTA variants for rows of up to NCH * 1024 elements: a CTA of
// kRowThreads threads takes one row at a time; every thread issues the loads
// of all its NCH 8-element chunks (x, gamma and, backward, dy) at once and
// keeps them in registers between the row reduction and the output pass.  The
// row sum adds each warp's butterfly total in warp order, so the results are
// deterministic.
constexpr int kRowThreads = 128;

__device__ __forceinline__ float block_row_sum(float v, float* red, int parity) {
    v = warp_sum(v);
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[parity * 4 + warp] = v;
    __syncthreads();
    return ((red[parity * 4 + 0] + red[parity * 4 + 1]) + red[parity * 4 + 2]) + red[parity * 4 + 3];
}

template <int NCH>
__global__ void __launch_bounds__(kRowThreads) rmsnorm_fwd_row_kernel(const __nv_bfloat16* __restrict__ x,
                                                                      const __nv_bfloat16* __restrict__ gamma,
                                                                      long long N, int d, float eps,
                                                                      const float* __restrict__ rstd_in,
                                                                      float* __restrict__ rstd_out,
                                                                      __nv_bfloat16* __restrict__ y) {
    __shared__ float red[8];
    const int nc = d >> 3;
    const uint4* g4 = reinterpret_cast<const uint4*>(gamma);
    int parity = 0;
    for (long long row = blockIdx.x; row < N; row += gridDim.x, parity ^= 1) {
        const uint4* x4 = reinterpret_cast<const uint4*>(x + row * d);
        uint4 v[NCH], gv[NCH];
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            const int c = threadIdx.x + kRowThreads * i;
            v[i] = c < nc ? __ldg(x4 + c) : make_uint4(0u, 0u, 0u, 0u);
            gv[i] = c < nc && y != nullptr
                        ? (gamma != nullptr ? __ldg(g4 + c) : make_uint4(kBf16One2, kBf16One2, kBf16One2, kBf16One2))
                        : make_uint4(0u, 0u, 0u, 0u);
        }
        float r;
        if (rstd_in != nullptr) {
            r = rstd_in[row];
        } else {
            float ss = 0.0f;
#pragma unroll
            for (int i = 0; i < NCH; ++i) {
                float f[8];
                unpack8(v[i], f);
#pragma unroll
                for (int k = 0; k < 8; ++k) ss = fmaf(f[k], f[k], ss);
            }
            ss = block_row_sum(ss, red, parity);
            r = 1.0f / sqrtf(ss / static_cast<float>(d) + eps);
            if (threadIdx.x == 0 && rstd_out != nullptr) rstd_out[row] = r;
        }
        if (y == nullptr) continue;
        uint4* y4 = reinterpret_cast<uint4*>(y + row * d);
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            const int c = threadIdx.x + kRowThreads * i;
            if (c < nc) {
                float f[8], g[8];
                unpack8(v[i], f);
                unpack8(gv[i], g);
#pragma unroll
                for (int k = 0; k < 8; ++k) f[k] = f[k] * r * g[k];
                y4[c] = pack8(f);
            }
        }
    }
}

template <int NCH>
__global__ void __launch_bounds__(kRowThreads) rmsnorm_bwd_row_kernel(const __nv_bfloat16* __restrict__ x,
                                                                      const __nv_bfloat16* __restrict__ gamma,
                                                                      const float* __restrict__ rstd,
                                                                      const __nv_bfloat16* __restrict__ dy,
                                                                      long long N, int d,
                                                                      __nv_bfloat16* __restrict__ dx) {
    __shared__ float red[8];
    const int nc = d >> 3;
    const uint4* g4 = reinterpret_cast<const uint4*>(gamma);
    int parity = 0;
    for (long long row = blockIdx.x; row < N; row += gridDim.x, parity ^= 1) {
        const uint4* x4 = reinterpret_cast<const uint4*>(x + row * d);
        const uint4* d4 = reinterpret_cast<const uint4*>(dy + row * d);
        uint4 xv[NCH], dv[NCH], gv[NCH];
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            const int c = threadIdx.x + kRowThreads * i;
            xv[i] = c < nc ? __ldg(x4 + c) : make_uint4(0u, 0u, 0u, 0u);
            dv[i] = c < nc ? __ldg(d4 + c) : make_uint4(0u, 0u, 0u, 0u);
            gv[i] = c < nc ? (gamma != nullptr ? __ldg(g4 + c) : make_uint4(kBf16One2, kBf16One2, kBf16One2, kBf16One2))
                           : make_uint4(0u, 0u, 0u, 0u);
        }
        const float r = rstd[row];
        float dot = 0.0f;
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            float f[8], g[8], e[8];
            unpack8(xv[i], f);
            unpack8(gv[i], g);
            unpack8(dv[i], e);
#pragma unroll
            for (int k = 0; k < 8; ++k) dot = fmaf(e[k] * g[k], f[k] * r, dot);
        }
        const float m = block_row_sum(dot, red, parity) / static_cast<float>(d);
        uint4* o4 = reinterpret_cast<uint4*>(dx + row * d);
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            const int c = threadIdx.x + kRowThreads * i;
            if (c < nc) {
                float f[8], g[8], e[8];
                unpack8(xv[i], f);
                unpack8(gv[i], g);
                unpack8(dv[i], e);
#pragma unroll
                for (int k = 0; k < 8; ++k) f[k] = r * (e[k] * g[k] - f[k] * r * m);
                o4[c] = pack8(f);
            }
        }
    }
}

// out[i, j] = bf16_rne(in[i, j] * gamma[j]) for a bf16 [rows, cols] matrix
// (cols a multiple of 8), up to two matrices per launch (blockIdx.y): gamma
// folded into a weight or adapter that multiplies the normalised rows.
struct ScaleCols {
    const __nv_bfloat16* in[2];
    __nv_bfloat16* out[2];
    long long rows[2];
};

__global__ void __launch_bounds__(256) scale_cols_kernel(const ScaleCols a, const __nv_bfloat16* __restrict__ gamma,
                                                         int cols) {
    const int z = blockIdx.y;
    const long long n8 = a.rows[z] * (cols >> 3);
    const uint4* in4 = reinterpret_cast<const uint4*>(a.in[z]);
    uint4* out4 = reinterpret_cast<uint4*>(a.out[z]);
    const uint4* g4 = reinterpret_cast<const uint4*>(gamma);
    const int gc = cols >> 3;
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        float f[8], g[8];
        unpack8(__ldg(in4 + i), f);
        unpack8(__ldg(g4 + i % gc), g);
#pragma unroll
        for (int k = 0; k < 8; ++k) f[k] *= g[k];
        out4[i] = pack8(f);
    }
}

}  // namespace lmlp
