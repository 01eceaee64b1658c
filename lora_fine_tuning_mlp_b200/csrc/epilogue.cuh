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
    // EPI_SWIGLU_FWD: optional factor of each row applied to both
    // accumulators before they are rounded (the RMSNorm row scale of the
    // pre-norm block with gamma folded into the gate/up weights)
    const float* row_scale;
};

#ifndef LMLP_FAST_SIGMOID
#define LMLP_FAST_SIGMOID 1
#endif
// sigmoid(x) = 1 / (1 + e^-x) with CUDA's fast exp and fast divide
// intrinsics (for large |x| the result saturates to 0 or 1); the forward and
// the backward epilogues share this one definition, so both form the same h.
__device__ __forceinline__ float sigmoid_f(float x) {
#if LMLP_FAST_SIGMOID
    return __fdividef(1.0f, 1.0f + __expf(-x));
#else
    return __frcp_rn(1.0f + __expf(-x));
#endif
}

#ifndef LMLP_STREAMING_EPILOGUE
#define LMLP_STREAMING_EPILOGUE 1
#endif
// Epilogue traffic (activations written once, g/u read once) is marked
// evict-first so that it does not push the GEMM operands that other tiles are
// still reading out of L2.
__device__ __forceinline__ void st_out(void* p, const uint4& v) {
#if LMLP_STREAMING_EPILOGUE
    __stcs(reinterpret_cast<uint4*>(p), v);
#else
    *reinterpret_cast<uint4*>(p) = v;
#endif
}
__device__ __forceinline__ uint4 ld_in(const void* p) {
#if LMLP_STREAMING_EPILOGUE
    return __ldcs(reinterpret_cast<const uint4*>(p));
#else
    return *reinterpret_cast<const uint4*>(p);
#endif
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Where an epilogue reads its fp32 accumulator row from (32 columns at a time).
// TMEM: `tacc` = TMEM address of this warp's lane quarter at the tile's
// accumulator buffer.  Warp-collective.
struct TmemSrc {
    uint32_t tacc;
    __device__ __forceinline__ void load(int col, uint32_t (&v)[32]) const {
        tmem_ld32(tacc + col, v);
        tmem_ld_wait();
    }
    __device__ __forceinline__ void load2(int c0, uint32_t (&v0)[32], int c1, uint32_t (&v1)[32]) const {
        tmem_ld32(tacc + c0, v0);
        tmem_ld32(tacc + c1, v1);
        tmem_ld_wait();
    }
};

// The sum, in split order, of `splits` fp32 partial rows (split s at
// base + s * split_stride): the accumulator of a tile whose K range was
// divided between CTAs.  Per thread.
struct PartialSrc {
    const float* base;
    long long split_stride;
    int splits;
    __device__ __forceinline__ void load(int col, uint32_t (&v)[32]) const {
        float acc[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] = 0.0f;
        // Two splits' loads are in flight together (the usual case is two).
        for (int sp0 = 0; sp0 < splits; sp0 += 2) {
            float4 x[2][8];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (sp0 + h < splits) {
                    const float4* q = reinterpret_cast<const float4*>(base + (sp0 + h) * split_stride + col);
#pragma unroll
                    for (int i = 0; i < 8; ++i) x[h][i] = __ldcg(q + i);
                }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (sp0 + h < splits) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        acc[4 * i] += x[h][i].x;
                        acc[4 * i + 1] += x[h][i].y;
                        acc[4 * i + 2] += x[h][i].z;
                        acc[4 * i + 3] += x[h][i].w;
                    }
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(acc[i]);
    }
    __device__ __forceinline__ void load2(int c0, uint32_t (&v0)[32], int c1, uint32_t (&v1)[32]) const {
        load(c0, v0);
        load(c1, v1);
    }
};

// SwiGLU backward for 8 consecutive columns: dH (fp32) with g, u (bf16 pairs).
__device__ __forceinline__ void swiglu_bwd8(const uint32_t* dh, const uint4& gq, const uint4& uq, uint4& dgq,
                                            uint4& duq, uint4& hq) {
    const uint32_t gw[4] = {gq.x, gq.y, gq.z, gq.w};
    const uint32_t uw[4] = {uq.x, uq.y, uq.z, uq.w};
    uint32_t dgw[4], duw[4], hw[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float dg2[2], du2[2], h2[2];
#pragma unroll
        for (int hsel = 0; hsel < 2; ++hsel) {
            const float gx = hsel ? bf16_hi(gw[e]) : bf16_lo(gw[e]);
            const float ux = hsel ? bf16_hi(uw[e]) : bf16_lo(uw[e]);
            const float d = __uint_as_float(dh[2 * e + hsel]);
            const float sg = sigmoid_f(gx);
            const float sl = gx * sg;
            du2[hsel] = d * sl;
            dg2[hsel] = d * ux * sg * (1.0f + gx * (1.0f - sg));
            h2[hsel] = sl * ux;
        }
        dgw[e] = pack_bf16(dg2[0], dg2[1]);
        duw[e] = pack_bf16(du2[0], du2[1]);
        hw[e] = pack_bf16(h2[0], h2[1]);
    }
    dgq = make_uint4(dgw[0], dgw[1], dgw[2], dgw[3]);
    duq = make_uint4(duw[0], duw[1], duw[2], duw[3]);
    hq = make_uint4(hw[0], hw[1], hw[2], hw[3]);
}

// Per-warp staging area of the coalesced store: 32 rows of 64 B, padded to
// 80 B so that both the row-per-lane writes and the row-contiguous reads
// touch every bank evenly.
constexpr uint32_t kStageRowBytes = 80;
constexpr uint32_t kStageWarpBytes = 32 * kStageRowBytes;

__device__ __forceinline__ void sts128(uint32_t addr, const uint4& v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ unsigned short lds16(uint32_t addr) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

// Writes one 32-column bf16 chunk of the warp's 32 rows (lane = row; v = this
// row's 32 values) to global memory.  With a staging area (stg != 0) the
// block is transposed through shared memory so that four lanes store 64
// contiguous bytes of one row: every store fills whole 32-byte sectors.
// Warp-collective; rows >= M and columns >= N are not stored.
__device__ __forceinline__ void emit_chunk(__nv_bfloat16* base, long long ld, int row, int col0, int M, int N,
                                           const uint4 (&v)[4], uint32_t stg) {
    const int lane = threadIdx.x & 31;
    if (stg == 0) {
        if (row < M) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (col0 + 8 * q < N) st_out(base + row * ld + col0 + 8 * q, v[q]);
        }
        return;
    }
    __syncwarp();
#pragma unroll
    for (int q = 0; q < 4; ++q) sts128(stg + lane * kStageRowBytes + q * 16, v[q]);
    __syncwarp();
    const int row0 = row - lane;
    const int c = lane & 3;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = i * 8 + (lane >> 2);
        const uint4 w = lds128(stg + r * kStageRowBytes + c * 16);
        if (row0 + r < M && col0 + 8 * c < N) st_out(base + (row0 + r) * ld + col0 + 8 * c, w);
    }
}

// TMA stores of 32 x 32 bf16 output blocks.  Each epilogue warp owns NB
// 2 KB shared-memory buffers (512-byte aligned; rows of 64 bytes in the
// 64-byte swizzle: 16-byte piece q of row r sits at piece q ^ ((r / 2) % 4),
// so the 32 lanes' row writes hit every bank once per quarter-warp) used in
// turn; a buffer is rewritten only once the store issued from it NB stores
// earlier has read it.  The tensor map clips rows and columns outside the
// output.  Warp-uniform state.
constexpr int kTmaBufs = 3;
constexpr uint32_t kTmaBlockBytes = 32 * 64;
constexpr uint32_t kTmaWarpBytes = kTmaBufs * kTmaBlockBytes;
template <int NB>
struct TmaStoreN {
    static_assert(NB >= 1 && NB <= 4, "1 to 4 store buffers a warp");
    const CUtensorMap* map[3];  // out0, out1, out2
    uint32_t buf;               // this warp's NB buffers
    int next;                   // buffer of the next store
    // Warp-collective: output `which`, the warp's 32 rows starting at row y
    // (lane = row; v = its 32 values), columns x .. x + 31.
    __device__ __forceinline__ void emit(int which, int x, int y, const uint4 (&v)[4]) {
        const int lane = threadIdx.x & 31;
        const uint32_t b = buf + static_cast<uint32_t>(next) * kTmaBlockBytes;
        if (++next == NB) next = 0;
        if (lane == 0) bulk_wait_read<NB - 1>();  // this buffer's last store has read it
        __syncwarp();
        const uint32_t rowb = b + static_cast<uint32_t>(lane) * 64u;
        const uint32_t sw = static_cast<uint32_t>(lane >> 1) & 3u;
#pragma unroll
        for (int q = 0; q < 4; ++q) sts128(rowb + ((static_cast<uint32_t>(q) ^ sw) << 4), v[q]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(map[which], b, x, y);
            bulk_commit();
        }
    }
    // Warp-collective: every store issued so far has completed.
    __device__ __forceinline__ void drain() const {
        if ((threadIdx.x & 31) == 0) bulk_wait<0>();
        __syncwarp();
    }
};
using TmaStore = TmaStoreN<kTmaBufs>;

// One output tile row per thread: `row` (may be >= M: stores are skipped),
// columns [col_base, col_base + bn); accumulator a's column c is read from
// `src` at a*acc_stride + c.  `stg`: this warp's staging area (0 = store
// directly); `ts`: TMA stores instead (bf16 outputs).
template <int NACC, int EPI, class Src, bool kPrefetchGU = true>
__device__ __forceinline__ void epilogue_tile(const EpiOut& o, int row, int col_base, int bn, const Src& src,
                                              uint32_t stg = 0, int acc_stride = -1, TmaStore* ts = nullptr) {
    // acc_stride: distance in src columns between the two accumulators
    // (default: bn, when a call covers all of a tile's columns)
    if (acc_stride < 0) acc_stride = bn;
    const bool row_ok = row < o.M;
    const int nchunks = bn >> 5;
    if constexpr (EPI == EPI_SWIGLU_BWD) {
        // g and u of the next 32 columns are loaded while this chunk computes.
        // With a staging area the warp loads its 32 rows x 64 B block
        // coalesced (four lanes per 64-byte row segment, every load filling
        // whole sectors) and transposes it through shared memory into one
        // row per lane; without one, each lane loads its own row.
        const __nv_bfloat16* gbase = static_cast<const __nv_bfloat16*>(o.in0);
        const __nv_bfloat16* ubase = static_cast<const __nv_bfloat16*>(o.in1);
        const int lane = threadIdx.x & 31;
        const int row0 = row - lane;
        uint4 gv[4], uv[4], gn[4], un[4];
        auto load_gu = [&](int c0, uint4(&gq)[4], uint4(&uq)[4]) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                // coalesced: slot q holds row 8q + lane/4, columns c0 + 8 (lane%4) ..
                // per lane:  slot q holds this lane's row, columns c0 + 8q ..
                const int r = stg != 0 ? row0 + 8 * q + (lane >> 2) : row;
                const int c = stg != 0 ? c0 + 8 * (lane & 3) : c0 + 8 * q;
                if (r < o.M && c < o.N) {
                    gq[q] = ld_in(gbase + static_cast<long long>(r) * o.ld + c);
                    uq[q] = ld_in(ubase + static_cast<long long>(r) * o.ld + c);
                } else {
                    gq[q] = make_uint4(0, 0, 0, 0);
                    uq[q] = make_uint4(0, 0, 0, 0);
                }
            }
        };
        // coalesced layout -> one row per lane, through the warp's staging area
        auto to_rows = [&](uint4(&x)[4]) {
            if (stg == 0) return;
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 4; ++q) sts128(stg + (8 * q + (lane >> 2)) * kStageRowBytes + (lane & 3) * 16, x[q]);
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 4; ++q) x[q] = lds128(stg + lane * kStageRowBytes + q * 16);
        };
        if constexpr (kPrefetchGU) load_gu(col_base, gv, uv);
        for (int ch = 0; ch < nchunks; ++ch) {
            const int col0 = col_base + ch * 32;
            if (col0 >= o.N) break;  // warp-uniform
            if constexpr (!kPrefetchGU) load_gu(col0, gv, uv);
            to_rows(gv);
            to_rows(uv);
            if constexpr (kPrefetchGU) {
                if (ch + 1 < nchunks) load_gu(col0 + 32, gn, un);
            }
            uint32_t v[32];
            src.load(ch * 32, v);
            uint4 dgq[4], duq[4], hq[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) swiglu_bwd8(v + 8 * q, gv[q], uv[q], dgq[q], duq[q], hq[q]);
            if (ts != nullptr) {
                ts->emit(0, col0, row0, dgq);
                ts->emit(1, col0, row0, duq);
                ts->emit(2, col0, row0, hq);
            } else {
                emit_chunk(static_cast<__nv_bfloat16*>(o.out0), o.ld, row, col0, o.M, o.N, dgq, stg);
                emit_chunk(static_cast<__nv_bfloat16*>(o.out1), o.ld, row, col0, o.M, o.N, duq, stg);
                emit_chunk(static_cast<__nv_bfloat16*>(o.out2), o.ld, row, col0, o.M, o.N, hq, stg);
            }
            if constexpr (kPrefetchGU) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    gv[q] = gn[q];
                    uv[q] = un[q];
                }
            }
        }
    } else {
        for (int ch = 0; ch < nchunks; ++ch) {
            const int col0 = col_base + ch * 32;
            if (col0 >= o.N) break;  // warp-uniform
            if constexpr (EPI == EPI_BF16) {
                uint32_t v[32];
                src.load(ch * 32, v);
                uint4 w[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    w[q].x = pack_bf16(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
                    w[q].y = pack_bf16(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
                    w[q].z = pack_bf16(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
                    w[q].w = pack_bf16(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
                }
                if (ts != nullptr)
                    ts->emit(0, col0, row - (threadIdx.x & 31), w);
                else
                    emit_chunk(static_cast<__nv_bfloat16*>(o.out0), o.ld, row, col0, o.M, o.N, w, stg);
            } else if constexpr (EPI == EPI_F32) {
#pragma unroll
                for (int acc = 0; acc < NACC; ++acc) {
                    uint32_t v[32];
                    src.load(acc * acc_stride + ch * 32, v);
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
            } else {  // EPI_SWIGLU_FWD
                uint32_t vg[32], vu[32];
                src.load2(ch * 32, vg, acc_stride + ch * 32, vu);
                if (o.row_scale != nullptr) {
                    const float rs = row_ok ? o.row_scale[row] : 0.0f;
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        vg[k] = __float_as_uint(__uint_as_float(vg[k]) * rs);
                        vu[k] = __float_as_uint(__uint_as_float(vu[k]) * rs);
                    }
                }
                uint4 gq[4], uq[4], hq[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
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
                    gq[q] = make_uint4(gw[0], gw[1], gw[2], gw[3]);
                    uq[q] = make_uint4(uw[0], uw[1], uw[2], uw[3]);
                    hq[q] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                }
                if (ts != nullptr) {
                    const int row0 = row - (threadIdx.x & 31);
                    ts->emit(0, col0, row0, gq);
                    ts->emit(1, col0, row0, uq);
                    ts->emit(2, col0, row0, hq);
                } else {
                    emit_chunk(static_cast<__nv_bfloat16*>(o.out0), o.ld, row, col0, o.M, o.N, gq, stg);
                    emit_chunk(static_cast<__nv_bfloat16*>(o.out1), o.ld, row, col0, o.M, o.N, uq, stg);
                    emit_chunk(static_cast<__nv_bfloat16*>(o.out2), o.ld, row, col0, o.M, o.N, hq, stg);
                }
            }
        }
    }
}

}  // namespace lmlp
