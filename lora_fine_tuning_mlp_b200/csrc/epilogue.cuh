// GEMM epilogues: TMEM accumulator tile -> registers -> global memory.
//
// Each epilogue warp owns 32 TMEM lanes (= 32 output rows, one per thread)
// and walks the tile's columns 32 at a time with tcgen05.ld.32x32b.x32.
// The SwiGLU epilogues are where the MLP's elementwise work lives:
//   forward:  g = bf16(G), u = bf16(U), h = bf16(silu(g) * u)
//   backward: with dH the accumulator and g, u read back (bf16),
//             sig = sigmoid(g), silu = g * sig,
//             du = dH * silu, dg = dH * u * sig * (1 + g * (1 - sig)),
//             and h = silu * u recomputed for the down-adapter gradient.
// (The SwiGLU forward and its derivative: the SwiGLU kernel family of
// "Unsloth 深度分析报告", section 关键设计决策.)
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace lmlp {

enum EpiKind : int {
    EPI_BF16 = 0,        // out0[m, n] = bf16(C)
    EPI_F32 = 1,         // fp32 partial tile (split-K): accumulator a -> out_a + split_off
    EPI_SWIGLU_FWD = 2,  // two accumulators G, U: g, u, h
    EPI_SWIGLU_BWD = 3,  // accumulator dH; reads g, u; writes dg, du, h
};

struct EpiOut {
    void* out0;
    void* out1;
    void* out2;
    const void* in0;
    const void* in1;
    long long ld;         // row stride (elements) of every out/in
    long long split_off;  // EPI_F32: element offset of this split's partial
    int M, N;             // valid rows / columns
};

__device__ __forceinline__ float sigmoid_f(float x) { return __frcp_rn(1.0f + __expf(-x)); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// One output tile row per thread: `row` (may be >= M: stores are skipped),
// columns [col_base, col_base + bn).  `tacc` = TMEM address of this warp's
// lane quarter at the tile's accumulator buffer (accumulator a at + a*bn).
template <int NACC, int EPI>
__device__ __forceinline__ void epilogue_tile(const EpiOut& o, int row, int col_base, int bn, uint32_t tacc) {
    const bool row_ok = row < o.M;
    const int nchunks = bn >> 5;
    for (int ch = 0; ch < nchunks; ++ch) {
        const int col0 = col_base + ch * 32;
        if (col0 >= o.N) break;  // warp-uniform
        if constexpr (EPI == EPI_BF16) {
            uint32_t v[32];
            tmem_ld32(tacc + ch * 32, v);
            tmem_ld_wait();
            if (row_ok) {
                __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(o.out0) + row * o.ld + col0;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (col0 + 8 * q < o.N) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
                        w.y = pack_bf16(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
                        w.z = pack_bf16(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
                        w.w = pack_bf16(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
                        *reinterpret_cast<uint4*>(dst + 8 * q) = w;
                    }
                }
            }
        } else if constexpr (EPI == EPI_F32) {
#pragma unroll
            for (int acc = 0; acc < NACC; ++acc) {
                uint32_t v[32];
                tmem_ld32(tacc + acc * bn + ch * 32, v);
                tmem_ld_wait();
                if (row_ok) {
                    float* dst = static_cast<float*>(acc == 0 ? o.out0 : o.out1) + o.split_off + row * o.ld + col0;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if (col0 + 4 * q < o.N) {
                            *reinterpret_cast<uint4*>(dst + 4 * q) =
                                make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                        }
                    }
                }
            }
        } else if constexpr (EPI == EPI_SWIGLU_FWD) {
            uint32_t vg[32], vu[32];
            tmem_ld32(tacc + ch * 32, vg);
            tmem_ld32(tacc + bn + ch * 32, vu);
            tmem_ld_wait();
            if (row_ok) {
                const long long off = row * o.ld + col0;
                __nv_bfloat16* gd = static_cast<__nv_bfloat16*>(o.out0) + off;
                __nv_bfloat16* ud = static_cast<__nv_bfloat16*>(o.out1) + off;
                __nv_bfloat16* hd = static_cast<__nv_bfloat16*>(o.out2) + off;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (col0 + 8 * q < o.N) {
                        uint32_t gw[4], uw[4], hw[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            gw[e] = pack_bf16(__uint_as_float(vg[8 * q + 2 * e]), __uint_as_float(vg[8 * q + 2 * e + 1]));
                            uw[e] = pack_bf16(__uint_as_float(vu[8 * q + 2 * e]), __uint_as_float(vu[8 * q + 2 * e + 1]));
                            const float g0 = bf16_lo(gw[e]), g1 = bf16_hi(gw[e]);
                            const float h0 = g0 * sigmoid_f(g0) * bf16_lo(uw[e]);
                            const float h1 = g1 * sigmoid_f(g1) * bf16_hi(uw[e]);
                            hw[e] = pack_bf16(h0, h1);
                        }
                        *reinterpret_cast<uint4*>(gd + 8 * q) = make_uint4(gw[0], gw[1], gw[2], gw[3]);
                        *reinterpret_cast<uint4*>(ud + 8 * q) = make_uint4(uw[0], uw[1], uw[2], uw[3]);
                        *reinterpret_cast<uint4*>(hd + 8 * q) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    }
                }
            }
        } else {  // EPI_SWIGLU_BWD
            uint4 gv[4], uv[4];
            const long long off = row * o.ld + col0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (row_ok && col0 + 8 * q < o.N) {
                    gv[q] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(o.in0) + off + 8 * q);
                    uv[q] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(o.in1) + off + 8 * q);
                } else {
                    gv[q] = make_uint4(0, 0, 0, 0);
                    uv[q] = make_uint4(0, 0, 0, 0);
                }
            }
            uint32_t v[32];
            tmem_ld32(tacc + ch * 32, v);
            tmem_ld_wait();
            if (row_ok) {
                __nv_bfloat16* dgd = static_cast<__nv_bfloat16*>(o.out0) + off;
                __nv_bfloat16* dud = static_cast<__nv_bfloat16*>(o.out1) + off;
                __nv_bfloat16* hd = static_cast<__nv_bfloat16*>(o.out2) + off;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (col0 + 8 * q < o.N) {
                        const uint32_t gw[4] = {gv[q].x, gv[q].y, gv[q].z, gv[q].w};
                        const uint32_t uw[4] = {uv[q].x, uv[q].y, uv[q].z, uv[q].w};
                        uint32_t dgw[4], duw[4], hw[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            float dg2[2], du2[2], h2[2];
#pragma unroll
                            for (int hsel = 0; hsel < 2; ++hsel) {
                                const float gx = hsel ? bf16_hi(gw[e]) : bf16_lo(gw[e]);
                                const float ux = hsel ? bf16_hi(uw[e]) : bf16_lo(uw[e]);
                                const float dh = __uint_as_float(v[8 * q + 2 * e + hsel]);
                                const float sg = sigmoid_f(gx);
                                const float sl = gx * sg;
                                du2[hsel] = dh * sl;
                                dg2[hsel] = dh * ux * sg * (1.0f + gx * (1.0f - sg));
                                h2[hsel] = sl * ux;
                            }
                            dgw[e] = pack_bf16(dg2[0], dg2[1]);
                            duw[e] = pack_bf16(du2[0], du2[1]);
                            hw[e] = pack_bf16(h2[0], h2[1]);
                        }
                        *reinterpret_cast<uint4*>(dgd + 8 * q) = make_uint4(dgw[0], dgw[1], dgw[2], dgw[3]);
                        *reinterpret_cast<uint4*>(dud + 8 * q) = make_uint4(duw[0], duw[1], duw[2], duw[3]);
                        *reinterpret_cast<uint4*>(hd + 8 * q) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    }
                }
            }
        }
    }
}

}  // namespace lmlp
