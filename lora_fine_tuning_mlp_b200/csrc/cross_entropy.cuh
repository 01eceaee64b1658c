// Chunked cross-entropy over a large vocabulary (include/lora_ce.h).
//
// Per row z of bf16 logits with label y:  t = s z  (then c tanh(t / c) with
// softcapping),  lse = log sum_j exp(t_j),  loss = lse - t_y.  The vocabulary
// is cut into chunks of kCeChunk logits; one CTA reduces one (row, chunk) to
// its running maximum and sum of exponentials, and a second launch combines a
// row's chunks in chunk order — the separability of logsumexp that the
// chunked kernel of "Unsloth 深度分析报告" (section 创新之处, 分块 Triton
// Cross Entropy Loss) relies on for 256K vocabularies.  The backward is one
// streaming pass: dz = dloss * (exp(t - lse) - [j == y]) * dt/dz.
//
// Both passes are bound by HBM (every logit is read once per pass, and the
// backward writes its gradient once) or, with softcapping, by the special-
// function unit (exp and reciprocal per logit).  A CTA streams its 64K-logit
// chunk in 8K-logit tiles, double buffered in registers, so loads are always
// in flight while the previous tile is reduced.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "f32x2.cuh"

namespace lmlp {

constexpr int kCeThreads = 256;
constexpr int kCeVec = 8;    // bf16 logits per 16-byte load
constexpr int kCeItems = 4;  // 16-byte loads per thread per tile
constexpr long long kCeTile = static_cast<long long>(kCeThreads) * kCeVec * kCeItems;  // 8192 logits
constexpr int kCeTilesPerChunk = 8;
constexpr long long kCeChunk = kCeTile * kCeTilesPerChunk;  // 65536 logits per CTA
// Running maximum before any logit is seen: finite, so that exp(m - M) never
// meets inf - inf, and far below any real logit, so that its weight is 0.
constexpr float kCeNegBig = -3.0e38f;

__device__ int g_ce_status;  // LORA_MLP_ERR_INVALID_ARG after a label outside [0, V)

// Logits, maxima and lse stay in natural units (t = s z is exact for the
// power-of-two scales, so a dominant logit gives p = 1 exactly); each
// exponential is exp2f((t - m) log2(e)) of a small difference.
struct CeArgs {
    const __nv_bfloat16* z;
    long long ld;
    long long V;
    long long N;
    int nchunk;
    const long long* labels;
    long long ignore;
    float scale;  // s
    float cap;    // c (0: none)
    float k2;       // 2 s / c * log2(e): 2^(k2 z) = e^(2 s z / c)
    float inv_cap;  // 1 / c
};

constexpr float kLog2e = 1.4426950408889634f;

// 2^x with the hardware's base-2 exponential (PTX ex2.approx.ftz: relative
// error about 2^-22; results below the normal range flush to 0, which is
// harmless here: such terms do not change a sum that holds a 1).
__device__ __forceinline__ float ce_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// e^x = 2^(x log2(e)), for the (non-positive) differences t - max.
__device__ __forceinline__ float ce_exp(float x) { return ce_exp2(x * kLog2e); }

__device__ __forceinline__ float ce_rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Transformed logit t.  With softcapping,
// c tanh(w) = c - 2c / (1 + e^(2w)), w = s z / c.  Where tanh is +-1 in fp32
// the exponential saturates to inf (reciprocal 0: t = c) or 0 (t = -c).
__device__ __forceinline__ float ce_t(const CeArgs& a, float z) {
    if (a.cap > 0.0f) return fmaf(ce_rcp(1.0f + ce_exp2(a.k2 * z)), -2.0f * a.cap, a.cap);
    return a.scale * z;
}

// The same for the four bf16 pairs of a 16-byte vector, as packed fp32
// pairs {t[2k], t[2k+1]}: the fp32 arithmetic two lanes per instruction,
// each lane rounded as ce_t rounds it.
__device__ __forceinline__ void ce_t8(const CeArgs& a, const uint4& v, uint64_t (&t2)[4]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint64_t z2 = f2_pack(w[k] << 16, w[k] & 0xFFFF0000u);
        if (a.cap > 0.0f) {
            float lo, hi;
            f2_unpack(f2_mul(z2, f2_packf(a.k2, a.k2)), lo, hi);
            f2_unpack(f2_add(f2_packf(ce_exp2(lo), ce_exp2(hi)), f2_packf(1.0f, 1.0f)), lo, hi);
            t2[k] = f2_fma(f2_packf(ce_rcp(lo), ce_rcp(hi)), f2_packf(-2.0f * a.cap, -2.0f * a.cap),
                           f2_packf(a.cap, a.cap));
        } else {
            t2[k] = f2_mul(z2, f2_packf(a.scale, a.scale));
        }
    }
}

// e^(t - m) for four packed pairs: subtract and scale two lanes at a time,
// the exponentials one by one.
__device__ __forceinline__ void ce_exp8(const uint64_t (&t2)[4], float m, uint64_t (&p2)[4]) {
    const uint64_t m2 = f2_packf(m, m), l2e = f2_packf(kLog2e, kLog2e);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        float lo, hi;
        f2_unpack(f2_mul(f2_sub(t2[k], m2), l2e), lo, hi);
        p2[k] = f2_packf(ce_exp2(lo), ce_exp2(hi));
    }
}

// (m, s) := (max, sum of e^(t - max)) of the union of two sets.
__device__ __forceinline__ void ce_merge(float& m, float& s, float m2, float s2) {
    const float M = fmaxf(m, m2);
    s = s * ce_exp(m - M) + s2 * ce_exp(m2 - M);
    m = M;
}

__device__ __forceinline__ uint4 ce_ld16(const __nv_bfloat16* p) {
    return __ldcs(reinterpret_cast<const uint4*>(p));
}

__device__ __forceinline__ void ce_unpack(const uint4& v, float (&x)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        x[2 * e] = __uint_as_float(w[e] << 16);
        x[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
}

// A CTA walks its chunk [c0, c0 + n) of one row in tiles of kCeTile logits;
// each thread holds kCeItems 16-byte vectors of a tile in registers.  Offsets
// are 32-bit and relative to c0.  Tiles are double buffered: the loads of
// tile k+1 are issued before tile k is used.
__device__ __forceinline__ void ce_load_tile(const __nv_bfloat16* zc, int tb, int n, uint4 (&v)[kCeItems]) {
#pragma unroll
    for (int it = 0; it < kCeItems; ++it) {
        const int j = tb + (it * kCeThreads + static_cast<int>(threadIdx.x)) * kCeVec;
        v[it] = j + kCeVec <= n ? ce_ld16(zc + j) : make_uint4(0u, 0u, 0u, 0u);
    }
}

// The transformed logits of the 8-wide vector at offset j < n, as packed
// pairs; past n: -inf.
__device__ __forceinline__ void ce_vector(const CeArgs& a, const __nv_bfloat16* zc, int j, int n, const uint4& v,
                                          uint64_t (&t2)[4]) {
    if (j + kCeVec <= n) {
        ce_t8(a, v, t2);
    } else {
        float t[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
            t[e] = j + e < n ? ce_t(a, __bfloat162float(zc[j + e])) : __int_as_float(0xff800000u);  // -inf
#pragma unroll
        for (int k = 0; k < 4; ++k) t2[k] = f2_packf(t[2 * k], t[2 * k + 1]);
    }
}

struct CeAcc {
    float m = kCeNegBig, s = 0.0f, ty = 0.0f;
    bool has_y = false;
};

__device__ __forceinline__ void ce_fwd_tile(const CeArgs& a, const __nv_bfloat16* zc, int tb, int n, int yr,
                                            const uint4 (&v)[kCeItems], CeAcc& r) {
#pragma unroll
    for (int it = 0; it < kCeItems; ++it) {
        const int j = tb + (it * kCeThreads + static_cast<int>(threadIdx.x)) * kCeVec;
        if (j >= n) break;  // later vectors of this thread lie further right
        uint64_t t2[4];
        ce_vector(a, zc, j, n, v[it], t2);
        float t[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) f2_unpack(t2[k], t[2 * k], t[2 * k + 1]);
        if (static_cast<unsigned>(yr - j) < static_cast<unsigned>(kCeVec)) {  // the label's vector
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (e == yr - j) r.ty = t[e];
            r.has_y = true;
        }
        float m8 = fmaxf(fmaxf(fmaxf(t[0], t[1]), fmaxf(t[2], t[3])), fmaxf(fmaxf(t[4], t[5]), fmaxf(t[6], t[7])));
        if (m8 > r.m) {
            r.s *= ce_exp(r.m - m8);
            r.m = m8;
        }
        uint64_t p2[4];
        ce_exp8(t2, r.m, p2);
        float lo, hi;
        f2_unpack(f2_add(f2_add(p2[0], p2[1]), f2_add(p2[2], p2[3])), lo, hi);
        r.s += lo + hi;
    }
}

// One CTA per (row, chunk): the chunk's (max t, sum e^(t - max t)) ->
// part[blk]; the thread holding the label's logit writes t_y -> ty[row].
__global__ void __launch_bounds__(kCeThreads) ce_fwd_partial_kernel(const CeArgs a, float2* __restrict__ part,
                                                                   float* __restrict__ ty) {
    const long long blk = blockIdx.x;
    const long long row = blk / a.nchunk;
    const long long c0 = (blk - row * a.nchunk) * kCeChunk;
    const int n = static_cast<int>(min(kCeChunk, a.V - c0));
    const int ntiles = (n + static_cast<int>(kCeTile) - 1) / static_cast<int>(kCeTile);
    const __nv_bfloat16* zc = a.z + row * a.ld + c0;
    const long long y = a.labels[row];
    const int yr = (y >= c0 && y < c0 + n) ? static_cast<int>(y - c0) : -kCeVec;

    CeAcc r;
    uint4 va[kCeItems], vb[kCeItems];
    ce_load_tile(zc, 0, n, va);
    for (int k = 0; k < ntiles; k += 2) {
        if (k + 1 < ntiles) ce_load_tile(zc, (k + 1) * static_cast<int>(kCeTile), n, vb);
        ce_fwd_tile(a, zc, k * static_cast<int>(kCeTile), n, yr, va, r);
        if (k + 1 >= ntiles) break;
        if (k + 2 < ntiles) ce_load_tile(zc, (k + 2) * static_cast<int>(kCeTile), n, va);
        ce_fwd_tile(a, zc, (k + 1) * static_cast<int>(kCeTile), n, yr, vb, r);
    }
    if (r.has_y) ty[row] = r.ty;
    float m = r.m, s = r.s;
    // CTA reduction in a fixed order: xor butterfly in each warp, then the
    // warps' results in warp order.
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
        const float s2 = __shfl_xor_sync(0xffffffffu, s, off);
        ce_merge(m, s, m2, s2);
    }
    __shared__ float2 wpart[kCeThreads / 32];
    if ((threadIdx.x & 31) == 0) wpart[threadIdx.x >> 5] = make_float2(m, s);
    __syncthreads();
    if (threadIdx.x == 0) {
        float M = wpart[0].x, S = wpart[0].y;
        for (int w = 1; w < kCeThreads / 32; ++w) ce_merge(M, S, wpart[w].x, wpart[w].y);
        part[blk] = make_float2(M, S);
    }
}

// One thread per row: lse over the row's chunks, combined in chunk order;
// loss = lse - t_y (0 for ignored rows, NaN for a bad label).
__global__ void __launch_bounds__(256) ce_fwd_combine_kernel(const CeArgs a, const float2* __restrict__ part,
                                                             const float* __restrict__ ty, float* __restrict__ loss,
                                                             float* __restrict__ lse) {
    const long long row = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (row >= a.N) return;
    float M = kCeNegBig, S = 0.0f;
    for (int k = 0; k < a.nchunk; ++k) {
        const float2 p = part[row * a.nchunk + k];
        ce_merge(M, S, p.x, p.y);
    }
    const float logS = logf(S);
    lse[row] = M + logS;
    const long long y = a.labels[row];
    if (y == a.ignore) {
        loss[row] = 0.0f;
    } else if (y < 0 || y >= a.V) {
        loss[row] = __int_as_float(0x7fc00000);
        atomicExch(&g_ce_status, -1 /* LORA_MLP_ERR_INVALID_ARG */);
    } else {
        // (M - t_y) + log S rather than lse - t_y: M and t_y are close when
        // the logits are large, and their difference is then exact in fp32,
        // where lse - t_y would cancel two large rounded numbers.
        loss[row] = (M - ty[row]) + logS;
    }
}

__device__ __forceinline__ void ce_bwd_tile(const CeArgs& a, const __nv_bfloat16* zc, __nv_bfloat16* dc, int tb,
                                            int n, int yr, float L, float g, bool ignored,
                                            const uint4 (&v)[kCeItems]) {
#pragma unroll
    for (int it = 0; it < kCeItems; ++it) {
        const int j = tb + (it * kCeThreads + static_cast<int>(threadIdx.x)) * kCeVec;
        if (j >= n) break;
        uint32_t o[4] = {0u, 0u, 0u, 0u};
        if (!ignored) {
            uint64_t t2[4], p2[4];
            ce_vector(a, zc, j, n, v[it], t2);
            ce_exp8(t2, L, p2);
            if (static_cast<unsigned>(yr - j) < static_cast<unsigned>(kCeVec)) {  // the label's vector
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float lo, hi;
                    f2_unpack(p2[k], lo, hi);
                    if (2 * k == yr - j) lo -= 1.0f;
                    if (2 * k + 1 == yr - j) hi -= 1.0f;
                    p2[k] = f2_packf(lo, hi);
                }
            }
            const uint64_t g2 = f2_packf(g, g);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                uint64_t d2 = f2_mul(p2[k], g2);
                if (a.cap > 0.0f) {  // times 1 - (t/c)^2
                    const uint64_t q2 = f2_mul(t2[k], f2_packf(a.inv_cap, a.inv_cap));
                    const uint64_t nq2 = f2_mul(t2[k], f2_packf(-a.inv_cap, -a.inv_cap));
                    d2 = f2_mul(d2, f2_fma(q2, nq2, f2_packf(1.0f, 1.0f)));
                }
                float lo, hi;
                f2_unpack(d2, lo, hi);
                __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
                o[k] = *reinterpret_cast<uint32_t*>(&h);
            }
        }
        if (j + kCeVec <= n) {
            __stcs(reinterpret_cast<uint4*>(dc + j), make_uint4(o[0], o[1], o[2], o[3]));
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (j + e < n) {
                    const uint32_t word = o[e >> 1];
                    dc[j + e] = __ushort_as_bfloat16(static_cast<unsigned short>(e & 1 ? word >> 16 : word & 0xFFFFu));
                }
        }
    }
}

// One CTA per (row, chunk): dz = dloss (exp(t - lse) - [j == y]) dt/dz in
// bf16, tiles double buffered as in the forward; ignored rows get zeros
// (their logits are not read).  dt/dz = s (1 - (t/c)^2) or s: the factor s
// is folded into g.  dz may alias z: every element is read before the same
// thread writes it.
//
// The per-row upstream gradient is dloss[row * dloss_stride], times
// dfactor[1] when dfactor is not null: a reduced loss passes its scalar
// upstream gradient with stride 0 and the forward's d(reduced)/d(row) factor.
__global__ void __launch_bounds__(kCeThreads) ce_bwd_kernel(const CeArgs a, const float* __restrict__ lse,
                                                           const float* __restrict__ dloss, long long dloss_stride,
                                                           const float* __restrict__ dfactor, __nv_bfloat16* dz,
                                                           long long ld_dz) {
    const long long blk = blockIdx.x;
    const long long row = blk / a.nchunk;
    const long long c0 = (blk - row * a.nchunk) * kCeChunk;
    const int n = static_cast<int>(min(kCeChunk, a.V - c0));
    const int ntiles = (n + static_cast<int>(kCeTile) - 1) / static_cast<int>(kCeTile);
    const __nv_bfloat16* zc = a.z + row * a.ld + c0;
    __nv_bfloat16* dc = dz + row * ld_dz + c0;
    const long long y = a.labels[row];
    const bool ignored = y == a.ignore;
    const int yr = (y >= c0 && y < c0 + n) ? static_cast<int>(y - c0) : -kCeVec;
    const float L = lse[row];
    const float gr = dfactor != nullptr ? dloss[row * dloss_stride] * dfactor[1] : dloss[row * dloss_stride];
    const float g = ignored ? 0.0f : gr * a.scale;
    const int ln = ignored ? 0 : n;  // ignored rows: no loads (the zero stores still run)

    uint4 va[kCeItems], vb[kCeItems];
    ce_load_tile(zc, 0, ln, va);
    for (int k = 0; k < ntiles; k += 2) {
        if (k + 1 < ntiles) ce_load_tile(zc, (k + 1) * static_cast<int>(kCeTile), ln, vb);
        ce_bwd_tile(a, zc, dc, k * static_cast<int>(kCeTile), n, yr, L, g, ignored, va);
        if (k + 1 >= ntiles) break;
        if (k + 2 < ntiles) ce_load_tile(zc, (k + 2) * static_cast<int>(kCeTile), ln, va);
        ce_bwd_tile(a, zc, dc, (k + 1) * static_cast<int>(kCeTile), n, yr, L, g, ignored, vb);
    }
}

// The per-row losses reduced to one number by one CTA, in a fixed order (so
// the result is bitwise deterministic): each thread adds its rows
// t, t + T, t + 2T, ... in fp64 and counts those not labelled ignore_index,
// then the threads' totals are added in a fixed tree.  out[0] is the sum
// (mean = false) or the sum over the count (mean = true; a count of 0 counts
// as 1); out[1] is d out[0] / d loss_row for a row that takes part: 1, or
// 1 / count.
constexpr int kCeReduceThreads = 1024;
__global__ void __launch_bounds__(kCeReduceThreads) ce_reduce_kernel(const CeArgs a, const float* __restrict__ loss,
                                                                     bool mean, float* __restrict__ out) {
    __shared__ double ssum[kCeReduceThreads];
    __shared__ long long scnt[kCeReduceThreads];
    double sum = 0.0;
    long long cnt = 0;
    for (long long row = threadIdx.x; row < a.N; row += kCeReduceThreads) {
        sum += static_cast<double>(loss[row]);
        cnt += a.labels[row] != a.ignore ? 1 : 0;
    }
    ssum[threadIdx.x] = sum;
    scnt[threadIdx.x] = cnt;
    __syncthreads();
    for (int h = kCeReduceThreads / 2; h > 0; h >>= 1) {
        if (static_cast<int>(threadIdx.x) < h) {
            ssum[threadIdx.x] += ssum[threadIdx.x + h];
            scnt[threadIdx.x] += scnt[threadIdx.x + h];
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const double n = static_cast<double>(scnt[0] > 0 ? scnt[0] : 1);
        out[0] = static_cast<float>(mean ? ssum[0] / n : ssum[0]);
        out[1] = static_cast<float>(mean ? 1.0 / n : 1.0);
    }
}

}  // namespace lmlp
