// Single-pass adapter-gradient launch of the LoRA MLP backward, for ranks up
// to 32 ("Unsloth 深度分析报告", 创新之处: the fused LoRA MLP backward, whose
// outputs are the six adapter gradients):
//
//   T_g = s dG Bg,  T_u = s dU Bu      row projections, reduced over the d_ff features
//   dBg = dG^T S_g, dBu = dU^T S_u     token reductions
//   dAd^T = H^T T_d                    token reduction
//
// dG, dU and H ([N, d_ff] bf16) are the largest operands of the backward's
// rank-r work, and T and dB reduce them along different axes.  Here each CTA
// owns a 2-D block of them: a range of 128-token blocks, whose T accumulators
// it keeps for the whole launch, and a range of 128-feature blocks, walked one
// by one with the dB accumulators of the current one.  A stage holds one
// 128 x 128 tile of dG, dU or H, brought in once by TMA as two 128-byte-
// swizzled 64-feature boxes, and feeds both kinds of product: read K-major
// (rows = tokens) it is the A operand of T, and the same bytes read MN-major
// (M = features, two 64-feature chunks, K = tokens) are the A operand of dB.
// So every byte of dG, dU and H crosses HBM once.  The B operands are small
// K-major tiles of 32 rows: Bg^T / Bu^T (a transposed copy of the adapter,
// made by the caller), and S_g^T, S_u^T, T_d^T as the forward and the first
// backward launch leave them.  Each CTA writes fp32 partial sums: dB over its
// token range, T over its feature range; dual_finalize_kernel adds them in a
// fixed order, scales and rounds, so the results do not depend on timing.
//
// Warp 0 is the TMA producer, warp 1 allocates TMEM and issues the UMMAs
// (M = 128, N = 32), warps 2-5 drain the accumulators.  TMEM: the T
// accumulators (2 per token block) in columns [0, 64 n_tb), then two buffers
// of the three dB accumulators, so the epilogue of one feature block runs
// under the MMAs of the next.
#pragma once
#include "umma_gemm.cuh"

namespace lmlp {

// T's B operand: 0 = Bg^T / Bu^T (K-major, 32 rows; a transposed copy made
// by the caller), 1 = Bg / Bu themselves, MN-major with N padded to 64 (no
// copy, but 64-column T accumulators and 16 KB of B a stage)
#ifndef LMLP_DUAL_BT_MN
#define LMLP_DUAL_BT_MN 0
#endif
constexpr bool kDualBtMn = LMLP_DUAL_BT_MN != 0;
constexpr int kDualBN = 32;                                // UMMA N of the dB products (ranks <= 32)
constexpr int kDualTN = kDualBtMn ? 64 : 32;               // UMMA N of the T products
constexpr int kDualStages = 4;
constexpr uint32_t kDualA = 2 * kATileBytes;               // 128 tokens x 128 features
constexpr uint32_t kDualBT = 2 * kDualTN * 128;            // T's B for 128 features
constexpr uint32_t kDualBD = 2 * kDualBN * 128;            // S^T / T_d^T rows of 128 tokens
constexpr uint32_t kDualStage = kDualA + kDualBT + kDualBD;  // 48 KB (56 KB with MN-major T B)
constexpr int kDualMaxTb = (512 - 6 * kDualBN) / (2 * kDualTN);  // token blocks a CTA can hold: 5 (2)

struct alignas(64) DualArgs {
    CUtensorMap maps[8];  // 0-2: dG, dU, H; 3-4: Bg^T, Bu^T; 5-7: S_g^T, S_u^T, T_d^T
    int N, dff, r;
    int n_tb;     // token blocks per token range
    int n_tr;     // token ranges
    int fchunks;  // feature ranges per token range (CTAs = n_tr * fchunks)
    int tiles_t, tiles_f;
    float* part_db;  // [n_tr][3][dff][r]: dBg, dBu, dAd^T over one token range
    float* part_t;   // [fchunks][N][2r]: T_g | T_u over one feature range
    long long wait_limit;
    int force_timeout;
    int nmaps;
};

struct DualUnit {
    int tr, fc, tb0, tb1, fb0, fb1;
};

__device__ __forceinline__ DualUnit dual_unit(const DualArgs& a) {
    DualUnit u;
    u.tr = static_cast<int>(blockIdx.x) / a.fchunks;
    u.fc = static_cast<int>(blockIdx.x) - u.tr * a.fchunks;
    u.tb0 = u.tr * a.n_tb;
    u.tb1 = min(a.tiles_t, u.tb0 + a.n_tb);
    u.fb0 = (u.fc * a.tiles_f) / a.fchunks;  // fchunks <= tiles_f: never empty
    u.fb1 = ((u.fc + 1) * a.tiles_f) / a.fchunks;
    return u;
}

// Feature blocks outer, token blocks inner, the three matrices innermost.
__device__ __forceinline__ long long dual_producer(const DualArgs& a, uint32_t base, const SmemCtl& c) {
    const DualUnit u = dual_unit(a);
    long long issued = 0;
    int stage = 0;
    uint32_t phase = 0;
    for (int fb = u.fb0; fb < u.fb1; ++fb) {
        for (int tb = u.tb0; tb < u.tb1; ++tb) {
            for (int m = 0; m < 3; ++m) {
                if (!wait_or_abort(c.empty + 8u * stage, phase ^ 1u, c)) return issued;
                const uint32_t fbar = c.full + 8u * stage;
                mbar_arrive_expect_tx(fbar, kDualA + (m < 2 ? kDualBT : 0u) + kDualBD);
                const uint32_t sA = base + static_cast<uint32_t>(stage) * kDualStage;
                const int x = fb * 128, y = tb * 128;
                tma_load_2d(sA, &a.maps[m], fbar, x, y);
                tma_load_2d(sA + kATileBytes, &a.maps[m], fbar, x + 64, y);
                if (m < 2) {
                    if (kDualBtMn) {  // Bg [dff, r]: box [64 (r, zero-padded) x 64 feature rows]
                        tma_load_2d(sA + kDualA, &a.maps[3 + m], fbar, 0, x);
                        tma_load_2d(sA + kDualA + kDualBT / 2, &a.maps[3 + m], fbar, 0, x + 64);
                    } else {          // Bg^T [r, dff]: box [64 features x 32 rows]
                        tma_load_2d(sA + kDualA, &a.maps[3 + m], fbar, x, 0);
                        tma_load_2d(sA + kDualA + kDualBT / 2, &a.maps[3 + m], fbar, x + 64, 0);
                    }
                }
                tma_load_2d(sA + kDualA + kDualBT, &a.maps[5 + m], fbar, y, 0);
                tma_load_2d(sA + kDualA + kDualBT + kDualBD / 2, &a.maps[5 + m], fbar, y + 64, 0);
                ++issued;
                if (++stage == kDualStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    }
    return issued;
}

// Per stage: T (dG, dU only) with the tile K-major, 8 UMMAs of K = 16 over its
// 128 features; then dB with the tile MN-major, 8 UMMAs of K = 16 over its 128
// tokens.  A T accumulator starts at the range's first feature block, a dB
// accumulator at its first token block.
__device__ __forceinline__ void dual_mma(const DualArgs& a, uint32_t base, uint32_t tmem_base, const SmemCtl& c) {
    const DualUnit u = dual_unit(a);
    const uint32_t id_t = idesc_bf16(kDualTN, false, kDualBtMn);
    const uint32_t id_b = idesc_bf16(kDualBN, true, false);
    const uint64_t a_k0 = sw128_desc(base, 16u, 1024u);           // rows = tokens, 64 features a row
    const uint64_t a_m0 = sw128_desc(base, kATileBytes, 1024u);   // M chunks (64 features) 16 KB apart
    const uint64_t bt0 = sw128_desc(base + kDualA, kDualBtMn ? 8192u : 16u, 1024u);
    const uint64_t bd0 = sw128_desc(base + kDualA + kDualBT, 16u, 1024u);
    constexpr uint32_t kStep = kDualStage >> 4;  // descriptor address units (16 B) per stage
    const uint32_t dcol0 = 2u * static_cast<uint32_t>(a.n_tb) * kDualTN;
    int stage = 0;
    uint32_t phase = 0;
    int dbuf = 0;
    uint32_t dphase = 0;
    for (int fb = u.fb0; fb < u.fb1; ++fb) {
        if (!wait_or_abort(c.acce + 8u * dbuf, dphase ^ 1u, c)) return;
        tc_fence_after();
        const uint32_t dcol = dcol0 + static_cast<uint32_t>(dbuf) * 3u * kDualBN;
        const uint32_t acc_t = fb > u.fb0 ? 1u : 0u;
        for (int tb = u.tb0; tb < u.tb1; ++tb) {
            const uint32_t ti = static_cast<uint32_t>(tb - u.tb0);
            const uint32_t acc_b = tb > u.tb0 ? 1u : 0u;
            for (int m = 0; m < 3; ++m) {
                if (!wait_or_abort(c.full + 8u * stage, phase, c)) return;
                tc_fence_after();
                const uint32_t so = static_cast<uint32_t>(stage) * kStep;
                if (m < 2) {
                    const uint32_t d = tmem_base + (2u * ti + static_cast<uint32_t>(m)) * kDualTN;
#pragma unroll
                    for (uint32_t k = 0; k < 8; ++k) {
                        // K slice k: box k / 4, 32 B further along a row per slice
                        // (MN-major B: 16 K rows of 128 B further down)
                        const uint32_t ao = (k >> 2) * (kATileBytes >> 4) + (k & 3u) * 2u;
                        const uint32_t bo = (k >> 2) * ((kDualBT / 2) >> 4) + (k & 3u) * (kDualBtMn ? (2048u >> 4) : 2u);
                        umma_bf16(d, a_k0 + so + ao, bt0 + so + bo, id_t, (acc_t | k) ? 1u : 0u);
                    }
                }
                const uint32_t d = tmem_base + dcol + static_cast<uint32_t>(m) * kDualBN;
#pragma unroll
                for (uint32_t k = 0; k < 8; ++k) {
                    // K slice k: 16 token rows (2048 B) further down both boxes of A;
                    // the B row for tokens 64 (k / 4) .. in box k / 4
                    const uint32_t ao = k * (2048u >> 4);
                    const uint32_t bo = (k >> 2) * ((kDualBD / 2) >> 4) + (k & 3u) * 2u;
                    umma_bf16(d, a_m0 + so + ao, bd0 + so + bo, id_b, (acc_b | k) ? 1u : 0u);
                }
                umma_commit(c.empty + 8u * stage);
                if (++stage == kDualStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        umma_commit(c.accf + 8u * dbuf);
        if (++dbuf == 2) {
            dbuf = 0;
            dphase ^= 1u;
        }
    }
    umma_commit(c.rawf);  // the T accumulators are complete
}

// r (a multiple of 8, <= 32) fp32 values of one TMEM row to global memory.
__device__ __forceinline__ void dual_store_row(float* dst, const uint32_t (&v)[32], int r) {
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
        if (j < r)
            *reinterpret_cast<float4*>(dst + j) = make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                                                              __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
    }
}

__device__ __forceinline__ void dual_epilogue(const DualArgs& a, uint32_t tmem_base, const SmemCtl& c) {
    const DualUnit u = dual_unit(a);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int quarter = warp & 3;  // TMEM lanes [32 quarter, 32 quarter + 32)
    const uint32_t lanes = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t dcol0 = 2u * static_cast<uint32_t>(a.n_tb) * kDualTN;
    if (a.force_timeout) {
        wait_or_abort(c.never, 0, c);
        return;
    }
    int dbuf = 0;
    uint32_t dphase = 0;
    for (int fb = u.fb0; fb < u.fb1; ++fb) {
        if (!wait_or_abort(c.accf + 8u * dbuf, dphase, c)) return;
        tc_fence_after();
        const int f = fb * 128 + quarter * 32 + lane;  // TMEM lane = feature
#pragma unroll 1
        for (int m = 0; m < 3; ++m) {
            uint32_t v[32];
            tmem_ld32(tmem_base + lanes + dcol0 + static_cast<uint32_t>(dbuf * 3 + m) * kDualBN, v);
            tmem_ld_wait();
            if (f < a.dff)
                dual_store_row(a.part_db + ((static_cast<long long>(u.tr) * 3 + m) * a.dff + f) * a.r, v, a.r);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(c.acce + 8u * dbuf);
        if (++dbuf == 2) {
            dbuf = 0;
            dphase ^= 1u;
        }
    }
    if (!wait_or_abort(c.rawf, 0, c)) return;
    tc_fence_after();
#pragma unroll 1
    for (int tb = u.tb0; tb < u.tb1; ++tb) {
        const int n = tb * 128 + quarter * 32 + lane;  // TMEM lane = token
#pragma unroll 1
        for (int m = 0; m < 2; ++m) {
            uint32_t v[32];
            tmem_ld32(tmem_base + lanes + (2u * static_cast<uint32_t>(tb - u.tb0) + static_cast<uint32_t>(m)) * kDualTN,
                      v);
            tmem_ld_wait();
            if (n < a.N)
                dual_store_row(a.part_t + (static_cast<long long>(u.fc) * a.N + n) * (2 * a.r) + m * a.r, v, a.r);
        }
    }
}

__global__ void __launch_bounds__(kGemmThreads, 1) dual_lowrank_kernel(const __grid_constant__ DualArgs args) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t ctl = base + kDualStages * kDualStage;
    uint8_t* ctl_ptr = smem_raw + (ctl - raw);
    const SmemCtl c = make_ctl(ctl, ctl_ptr, args.wait_limit);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (warp == 0 && lane < args.nmaps) tma_prefetch_desc(&args.maps[lane]);
    if (warp == 0 && lane == 0) {
        for (int s = 0; s < kDualStages; ++s) {
            mbar_init(c.full + 8u * s, 1);
            mbar_init(c.empty + 8u * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(c.accf + 8u * b, 1);  // dB accumulators written
            mbar_init(c.acce + 8u * b, 4);  // ... and drained by the four epilogue warps
        }
        mbar_init(c.rawf, 1);  // T accumulators written
        mbar_init(c.drain, 1);
        mbar_init(c.never, 1);
        *c.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(c.tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(ctl_ptr + (c.tmem_slot - ctl));
#if LMLP_PDL
    grid_dependency_wait();
    grid_launch_dependents();
#endif
    if (warp == 0) {
        if (lane == 0) {
            const long long issued = dual_producer(args, base, c);
            drain_loads(c.full, kDualStages, issued, c.wait_limit);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            dual_mma(args, base, tmem_base, c);
            umma_commit(c.drain);
            const long long t0 = clock64();
            while (!mbar_try_wait(c.drain, 0)) {
                if (clock64() - t0 > c.wait_limit) break;
            }
        }
        __syncwarp();
    } else {
        dual_epilogue(args, tmem_base, c);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, 512);
}

// The sums of the partials, in a fixed order.  One thread per four
// consecutive values (partials read coalesced, eight loads in flight before
// their in-order adds).  Blocks [0, db_blocks): (matrix, feature, 4 ranks) of
// dBg, dBu (row-major [dff, r]) and dAd (written transposed, [r, dff]); the
// rest: (token, 4 of the 2r columns) of T_g | T_u, scaled by s, row-major
// into Tgu [N, 2r] and transposed into TguT [2r, ldN] (there also times the
// token's row scale, when given).
struct DualFin {
    const float* part_db;
    const float* part_t;
    __nv_bfloat16* dBg;
    __nv_bfloat16* dBu;
    __nv_bfloat16* dAd;
    __nv_bfloat16* Tgu;
    __nv_bfloat16* TguT;
    const float* row_scale;
    long long ldN;
    int N, dff, r, n_tr, fchunks, db_blocks;
    float s;
};

constexpr int kDualFinThreads = 256;
constexpr int kDualFinBatch = 8;

// sum over k < n of src[k * stride] (float4), in order of k
__device__ __forceinline__ float4 dual_sum4(const float* src, long long stride, int n) {
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int k0 = 0; k0 < n; k0 += kDualFinBatch) {
        float4 v[kDualFinBatch];
#pragma unroll
        for (int q = 0; q < kDualFinBatch; ++q)
            if (k0 + q < n) v[q] = __ldcg(reinterpret_cast<const float4*>(src + (k0 + q) * stride));
#pragma unroll
        for (int q = 0; q < kDualFinBatch; ++q) {
            if (k0 + q < n) {
                acc.x += v[q].x;
                acc.y += v[q].y;
                acc.z += v[q].z;
                acc.w += v[q].w;
            }
        }
    }
    return acc;
}

__global__ void __launch_bounds__(kDualFinThreads) dual_finalize_kernel(const DualFin p) {
#if LMLP_PDL
    grid_dependency_wait();
    grid_launch_dependents();
#endif
    if (static_cast<int>(blockIdx.x) < p.db_blocks) {
        const int q4 = p.r / 4;
        const long long i = static_cast<long long>(blockIdx.x) * kDualFinThreads + threadIdx.x;
        if (i >= 3ll * p.dff * q4) return;
        const long long mf = i / q4;
        const int j = static_cast<int>(i - mf * q4) * 4;
        const int m = static_cast<int>(mf / p.dff);
        const int f = static_cast<int>(mf - static_cast<long long>(m) * p.dff);
        const float4 v = dual_sum4(p.part_db + mf * p.r + j, 3ll * p.dff * p.r, p.n_tr);
        if (m < 2) {
            __nv_bfloat16* dst = (m == 0 ? p.dBg : p.dBu) + static_cast<long long>(f) * p.r + j;
            *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16(v.x, v.y), pack_bf16(v.z, v.w));
        } else {
            __nv_bfloat16* dst = p.dAd + static_cast<long long>(j) * p.dff + f;
            dst[0] = __float2bfloat16_rn(v.x);
            dst[p.dff] = __float2bfloat16_rn(v.y);
            dst[2ll * p.dff] = __float2bfloat16_rn(v.z);
            dst[3ll * p.dff] = __float2bfloat16_rn(v.w);
        }
        return;
    }
    const int r2 = 2 * p.r, q4 = r2 / 4;
    const long long i = static_cast<long long>(blockIdx.x - p.db_blocks) * kDualFinThreads + threadIdx.x;
    if (i >= static_cast<long long>(p.N) * q4) return;
    const long long n = i / q4;
    const int j = static_cast<int>(i - n * q4) * 4;
    const float4 v = dual_sum4(p.part_t + n * r2 + j, static_cast<long long>(p.N) * r2, p.fchunks);
    const float s = p.s;
    *reinterpret_cast<uint2*>(p.Tgu + n * r2 + j) = make_uint2(pack_bf16(v.x * s, v.y * s), pack_bf16(v.z * s, v.w * s));
    const float rs = p.row_scale != nullptr ? p.row_scale[n] : 1.0f;
    __nv_bfloat16* dst = p.TguT + static_cast<long long>(j) * p.ldN + n;
    dst[0] = __float2bfloat16_rn(v.x * s * rs);
    dst[p.ldN] = __float2bfloat16_rn(v.y * s * rs);
    dst[2 * p.ldN] = __float2bfloat16_rn(v.z * s * rs);
    dst[3 * p.ldN] = __float2bfloat16_rn(v.w * s * rs);
}

}  // namespace lmlp
