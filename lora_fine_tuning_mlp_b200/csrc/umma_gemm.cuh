// Persistent, warp-specialised tcgen05 GEMM for sm_100a.
//
//   C[m, n] = sum_k A[m, k] * B[n, k]      (bf16 in, fp32 accumulate in TMEM)
//
// One CTA per SM walks a list of output tiles ("units").  Warp 0 is the TMA
// producer, warp 1 allocates TMEM and issues tcgen05.mma from one thread,
// warps 2-5 are the epilogue (TMEM -> registers -> global).  Shared-memory
// stages hand operands from TMA to the tensor core through full/empty
// mbarriers; two TMEM accumulator buffers let the epilogue of one tile run
// under the mainloop of the next.
//
// The K dimension of a tile is a list of "segments", each with its own A and
// B tensor maps: this is how the rank-r LoRA path joins a dense projection —
// [X | s·X·A^T] times [W | B]^T is one accumulation, the low-rank segment being
// a K = r extension of the dense one.  With two accumulators (NACC = 2) the
// gate and up projections share the A tiles (X) and each segment says which
// accumulator(s) it feeds.
//
// Tiles are 128 x BN, K blocks are 64 bf16 = 128 B wide, every smem operand
// tile uses the 128-byte swizzle written by TMA.  A is K-major, or MN-major
// (activations [tokens, features] read as the transposed operand of a
// token-reduction); B likewise.  Out-of-range rows/columns of a box are
// zero-filled by TMA, so ragged M, N and K need no special case in the
// mainloop; the epilogue predicates its stores.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#ifndef LMLP_PDL
#define LMLP_PDL 1  // launch the GEMM kernels with programmatic stream serialisation
#endif

#include "epilogue.cuh"
#include "ptx.cuh"

namespace lmlp {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr uint32_t kATileBytes = kBM * kBK * 2;  // 16 KB
constexpr int kMaxMaps = 12;
constexpr int kMaxSegs = 4;
constexpr int kMaxProbs = 5;
constexpr int kMaxStages = 12;
constexpr int kGemmThreads = 192;
constexpr int kMaxPerm = 2048;  // units a launch can reorder (see GemmArgs::perm)

struct Seg {
    int a_map;
    int b_map[2];  // per accumulator; -1 = this segment does not feed it
    int kblocks;
    int k_len;
};

struct Prob {
    int M, N;
    int tiles_m, tiles_n, splits, nkb, nsegs, unit0;
    int a_mn, b_mn;  // operand majorness: 0 = K-major, 1 = MN-major (B MN-major needs bn % 64 == 0)
    Seg seg[kMaxSegs];
    void* out0;
    void* out1;
    void* out2;
    const void* in0;
    const void* in1;
    long long ld;            // row stride (elements) of out*/in*
    long long split_stride;  // elements between split-K partials (EPI_F32)
    // Split-K finalisation (EPI_F32 with counters != nullptr): the last CTA to
    // finish a tile sums the splits' fp32 partials in split order (so results
    // do not depend on timing), scales, and writes bf16 row-major to rm
    // [M, fin_cols] and/or transposed: column j < tr_split to tr0[j][m], the
    // rest to tr1[j - tr_split][m].  A tile covers all columns (tiles_n = 1).
    int* counters;  // one per tile, zero before the launch; reset by the last CTA
    float scale;
    int fin_cols;
    int tr_split;
    void* rm;
    long long ld_rm;
    void* tr0;
    void* tr1;
    long long ld_tr;
    // Optional factor of each accumulator row m for the transposed outputs
    // only (fp32, or bf16), applied after `scale`: the RMSNorm row scale of
    // the pre-norm block with gamma folded into the weights.
    const float* tr_row_scale;
    const __nv_bfloat16* tr_row_scale_bf16;
};

struct alignas(64) GemmArgs {
    CUtensorMap maps[kMaxMaps];
    Prob prob[kMaxProbs];
    int nprobs;
    int total_units;
    int bn;            // tile N (= UMMA N), multiple of 32, <= 256
    int stages;
    int group_m;       // raster: consecutive tiles walk down groups of this many M tiles
    uint32_t b_bytes;  // one B tile: bn rows (or bn/64 MN chunks) x 128 B
    long long wait_limit;  // SM cycles a barrier wait may spin before the kernel gives up
    int force_timeout;     // test hook: the epilogue waits on a barrier nothing signals
    int nmaps;             // maps[0, nmaps) are encoded
    // Optional processing order: with nperm == total_units, the i-th unit
    // taken by the persistent grid is perm[i].  Lets a launch group the units
    // that read the same data into the same round, so the second read hits L2.
    int nperm;
    uint16_t perm[kMaxPerm];
};

struct Unit {
    int p, mb, nb, ks, kb0, kb1;
};

__device__ __forceinline__ Unit decode_unit(const GemmArgs& a, int u) {
    if (a.nperm > 0) u = a.perm[u];
    Unit r;
    r.p = 0;
    for (int i = 1; i < a.nprobs; ++i)
        if (u >= a.prob[i].unit0) r.p = i;
    const Prob& P = a.prob[r.p];
    const int lu = u - P.unit0;
    const int tile = lu / P.splits;
    r.ks = lu - tile * P.splits;
    const int per_group = a.group_m * P.tiles_n;
    const int grp = tile / per_group;
    const int first_m = grp * a.group_m;
    const int gsz = min(a.group_m, P.tiles_m - first_m);
    const int local = tile - grp * per_group;
    r.mb = first_m + local % gsz;
    r.nb = local / gsz;
    r.kb0 = static_cast<int>((static_cast<long long>(r.ks) * P.nkb) / P.splits);
    r.kb1 = static_cast<int>((static_cast<long long>(r.ks + 1) * P.nkb) / P.splits);
    return r;
}

__device__ int g_lmlp_status;  // LORA_MLP_ERR_DEVICE_TIMEOUT once any bounded wait expired

struct SmemCtl {
    uint32_t full, empty, accf, acce, drain, never;  // barrier addresses (shared); `never` is never arrived on
    uint32_t rawf;  // per-stage "codes landed" barriers of the CTA-pair GEMM with int4 B (unused otherwise)
    uint32_t tmem_slot;
    volatile int* abort_flag;
    volatile int* fin_flag;
    long long wait_limit;  // SM cycles a wait may spin before giving up
};

// Bounded wait that also gives up as soon as another role of this CTA gave
// up.  kCluster: acquire at cluster scope (see mbar_try_wait_cluster).
template <bool kCluster = false>
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, const SmemCtl& c) {
    auto ready = [&]() { return kCluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity); };
    if (ready()) return true;
    const long long t0 = clock64();
    while (!ready()) {
        if (*c.abort_flag) return false;
        if (clock64() - t0 > c.wait_limit) {
            *c.abort_flag = 1;
            atomicExch(&g_lmlp_status, -7 /* LORA_MLP_ERR_DEVICE_TIMEOUT */);
            return false;
        }
    }
    return true;
}


// Before a CTA leaves, every TMA load it issued has to have landed: a copy
// still in flight would write into shared memory that the next CTA on the SM
// may own.  On the normal path the MMA issuer has consumed every stage, so
// this returns at once; after a bounded wait gave up it waits, again bounded
// and regardless of the abort flag, for the last phase issued into each
// stage's full barrier (issue i went to stage i % stages with phase parity
// (i / stages) & 1).  One deadline covers all stages.
__device__ __forceinline__ void drain_loads(uint32_t full, int stages, long long issued, long long limit) {
    const long long t0 = clock64();
    for (int s = 0; s < stages && s < issued; ++s) {
        const long long i = s + static_cast<long long>(stages) * ((issued - 1 - s) / stages);
        const uint32_t parity = static_cast<uint32_t>((i / stages) & 1);
        while (!mbar_try_wait(full + 8u * static_cast<uint32_t>(s), parity)) {
            if (clock64() - t0 > limit) return;
        }
    }
}

// ---------------------------------------------------------------------------
// roles

// Loads are issued in bursts of up to kLoadBurst consecutive K blocks: the
// producer first waits until that many stages are free, then issues their
// copies back to back, so the DRAM pages of each A row are requested
// together rather than one 128-byte piece at a time.
#ifndef LMLP_FIN_BATCH
#define LMLP_FIN_BATCH 8  // split-K partials whose loads the finalising CTA issues together
#endif
#ifndef LMLP_MAX_CPS
#define LMLP_MAX_CPS 2  // most CTAs of this kernel that share an SM
#endif
#ifndef LMLP_LOAD_BURST
#define LMLP_LOAD_BURST 4
#endif
constexpr int kLoadBurst = LMLP_LOAD_BURST;

// The producer (one thread).  On the HBM-bound rank-r launches this loop
// bounds the stream, so it is kept as short as the MMA issuer's: segments
// are walked directly, and the per-segment tensor maps and byte count are
// looked up once per segment, not per K block.  A separate wait cursor runs
// up to one burst ahead of the issue cursor.
// Returns the number of stages it filled (issued loads into).
template <int NACC>
__device__ __forceinline__ long long producer_loop(const GemmArgs& a, uint32_t smem_base, uint32_t stage_bytes,
                                                   const SmemCtl& c) {
    long long issued = 0;
    int stage = 0;
    uint32_t phase = 0;
    int wst = 0;  // next stage whose release to wait for
    uint32_t wph = 0;
    int credits = 0;  // stages known free ahead of `stage`
    const int burst = a.stages >= 2 * kLoadBurst ? kLoadBurst : 1;
    for (int u = blockIdx.x; u < a.total_units; u += gridDim.x) {
        const Unit t = decode_unit(a, u);
        const Prob& P = a.prob[t.p];
        const bool a_mn = P.a_mn != 0, b_mn = P.b_mn != 0;
        const int m0 = t.mb * kBM;
        const int n0 = t.nb * a.bn;
        const int nbj = b_mn ? a.bn / 64 : 1;
        int seg_kb0 = 0;
        for (int sg = 0; sg < P.nsegs; ++sg) {
            const Seg& S = P.seg[sg];
            const int lo = max(t.kb0 - seg_kb0, 0), hi = min(t.kb1 - seg_kb0, S.kblocks);
            seg_kb0 += S.kblocks;
            if (lo >= hi) continue;
            const CUtensorMap* am = &a.maps[S.a_map];
            const CUtensorMap* bm[NACC];
            uint32_t bytes = kATileBytes;
#pragma unroll
            for (int acc = 0; acc < NACC; ++acc) {
                bm[acc] = S.b_map[acc] >= 0 ? &a.maps[S.b_map[acc]] : nullptr;
                if (bm[acc] != nullptr) bytes += a.b_bytes;
            }
            for (int kb = lo; kb < hi; ++kb) {
                if (credits == 0) {
                    for (int i = 0; i < burst; ++i) {
                        if (!wait_or_abort(c.empty + 8u * wst, wph ^ 1u, c)) return issued;
                        if (++wst == a.stages) {
                            wst = 0;
                            wph ^= 1u;
                        }
                    }
                    credits = burst;
                }
                --credits;
                const int k0 = kb * kBK;
                const uint32_t fb = c.full + 8u * stage;
                mbar_arrive_expect_tx(fb, bytes);
                const uint32_t sA = smem_base + stage * stage_bytes;
                if (a_mn) {
                    tma_load_2d(sA, am, fb, m0, k0);
                    tma_load_2d(sA + 8192u, am, fb, m0 + 64, k0);
                } else {
                    tma_load_2d(sA, am, fb, k0, m0);
                }
#pragma unroll
                for (int acc = 0; acc < NACC; ++acc) {
                    if (bm[acc] == nullptr) continue;
                    const uint32_t sB = sA + kATileBytes + acc * a.b_bytes;
                    if (b_mn) {
                        for (int j = 0; j < nbj; ++j) tma_load_2d(sB + 8192u * j, bm[acc], fb, n0 + 64 * j, k0);
                    } else {
                        tma_load_2d(sB, bm[acc], fb, k0, n0);
                    }
                }
                ++issued;
                if (++stage == a.stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    }
    return issued;
}

// The MMA issuer (one thread).  The rank-r products are tall and skinny: a
// K block's UMMAs take the tensor core only 16-64 cycles, so this loop, not
// the tensor core, sets how fast a CTA can consume its stages.  It is kept
// short: segments are walked directly (only a segment's last block can be
// partial) and each stage's descriptors are those of stage 0 plus an offset.
template <int NACC>
__device__ __forceinline__ void mma_loop(const GemmArgs& a, uint32_t smem_base, uint32_t stage_bytes,
                                         uint32_t tmem_base, const SmemCtl& c) {
    int stage = 0;
    uint32_t phase = 0;
    int abuf = 0;
    uint32_t aphase = 0;
    const uint32_t acc_cols = NACC * a.bn;
    // bytes >> 4 per stage in the descriptors' 14-bit address field (shared
    // memory is < 256 KB, so adding offsets never carries out of the field)
    const uint32_t sstep = stage_bytes >> 4;
    for (int u = blockIdx.x; u < a.total_units; u += gridDim.x) {
        const Unit t = decode_unit(a, u);
        const Prob& P = a.prob[t.p];
        const bool a_mn = P.a_mn != 0, b_mn = P.b_mn != 0;
        const uint32_t idesc = idesc_bf16(static_cast<uint32_t>(a.bn), a_mn, b_mn);
        // Two accumulators fed by the same segment sit side by side in TMEM and
        // their B tiles side by side in smem, so one UMMA of N = 2*bn does both
        // (A is read from smem once instead of twice).
        const bool pair_ok = NACC == 2 && !b_mn && 2 * a.bn <= 256;
        const uint32_t idesc_pair = idesc_bf16(static_cast<uint32_t>(2 * a.bn), a_mn, b_mn);
        // Stage-0 descriptors; the next 16-wide K slice is 32 B further along
        // a K-major tile and 2048 B (16 rows of 128 B) along an MN-major one.
        const uint64_t a0 = a_mn ? sw128_desc(smem_base, 8192u, 1024u) : sw128_desc(smem_base, 16u, 1024u);
        const uint32_t astep = a_mn ? (2048u >> 4) : (32u >> 4);
        const uint32_t bstep = b_mn ? (2048u >> 4) : (32u >> 4);
        uint64_t b0[NACC];
#pragma unroll
        for (int acc = 0; acc < NACC; ++acc) {
            const uint32_t sB = smem_base + kATileBytes + acc * a.b_bytes;
            b0[acc] = b_mn ? sw128_desc(sB, 8192u, 1024u) : sw128_desc(sB, 16u, 1024u);
        }
        if (!wait_or_abort(c.acce + 8u * abuf, aphase ^ 1u, c)) return;
        tc_fence_after();
        uint32_t started = 0;
        int seg_kb0 = 0;
        for (int sg = 0; sg < P.nsegs; ++sg) {
            const Seg& S = P.seg[sg];
            const int nkb = S.kblocks;
            const int lo = max(t.kb0 - seg_kb0, 0), hi = min(t.kb1 - seg_kb0, nkb);
            seg_kb0 += nkb;
            for (int kb = lo; kb < hi; ++kb) {
                const int nk = kb == nkb - 1 ? ((S.k_len - kb * kBK + 15) >> 4) : 4;
                if (!wait_or_abort(c.full + 8u * stage, phase, c)) return;
                tc_fence_after();
                const uint32_t so = stage * sstep;
                const uint64_t ad = a0 + so;
                if (pair_ok && S.b_map[0] >= 0 && S.b_map[1] >= 0 && (started == 0u || started == 3u)) {
                    const uint64_t bd = b0[0] + so;
                    const uint32_t d = tmem_base + abuf * acc_cols;
                    for (int k = 0; k < nk; ++k)
                        umma_bf16(d, ad + k * astep, bd + k * bstep, idesc_pair, (started & 1u) | (k > 0 ? 1u : 0u));
                    started = 3u;
                } else {
#pragma unroll
                    for (int acc = 0; acc < NACC; ++acc) {
                        if (S.b_map[acc] < 0) continue;
                        const uint64_t bd = b0[acc] + so;
                        const uint32_t d = tmem_base + abuf * acc_cols + acc * a.bn;
                        for (int k = 0; k < nk; ++k)
                            umma_bf16(d, ad + k * astep, bd + k * bstep, idesc,
                                      ((started >> acc) & 1u) | (k > 0 ? 1u : 0u));
                        started |= 1u << acc;
                    }
                }
                umma_commit(c.empty + 8u * stage);
                if (++stage == a.stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        umma_commit(c.accf + 8u * abuf);
        if (++abuf == 2) {
            abuf = 0;
            aphase ^= 1u;
        }
    }
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Called by all four epilogue warps after their rows of a split's partial
// tile are stored.  The CTA that completes a tile last reduces it.
__device__ __forceinline__ void splitk_finalize(const Prob& P, const Unit& t, int row, volatile int* fin_flag) {
    __threadfence();
    epi_bar();
    if (threadIdx.x == 64) {
        int* ctr = P.counters + t.mb * P.tiles_n + t.nb;
        const int old = atomicAdd(ctr, 1);
        const int last = old == P.splits - 1;
        if (last) *ctr = 0;
        *fin_flag = last;
    }
    epi_bar();
    if (!*fin_flag) return;
    __threadfence();
    if (row >= P.M) return;
    const float* src = static_cast<const float*>(P.out0) + row * P.ld;
    __nv_bfloat16* rm = static_cast<__nv_bfloat16*>(P.rm);
    __nv_bfloat16* tr0 = static_cast<__nv_bfloat16*>(P.tr0);
    __nv_bfloat16* tr1 = static_cast<__nv_bfloat16*>(P.tr1);
    for (int j = 0; j < P.fin_cols; j += 8) {
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
        // Loads of up to 8 splits are issued before their (in-order) adds, so a
        // tile with many splits costs a few L2 round trips, not one per split.
        for (int sp0 = 0; sp0 < P.splits; sp0 += LMLP_FIN_BATCH) {
            float4 v[LMLP_FIN_BATCH][2];
#pragma unroll
            for (int q = 0; q < LMLP_FIN_BATCH; ++q) {
                if (sp0 + q < P.splits) {
                    const float4* src4 = reinterpret_cast<const float4*>(src + (sp0 + q) * P.split_stride + j);
                    v[q][0] = __ldcg(src4);
                    v[q][1] = __ldcg(src4 + 1);
                }
            }
#pragma unroll
            for (int q = 0; q < LMLP_FIN_BATCH; ++q) {
                if (sp0 + q < P.splits) {
                    acc[0] += v[q][0].x; acc[1] += v[q][0].y; acc[2] += v[q][0].z; acc[3] += v[q][0].w;
                    acc[4] += v[q][1].x; acc[5] += v[q][1].y; acc[6] += v[q][1].z; acc[7] += v[q][1].w;
                }
            }
        }
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) w[e] = pack_bf16(acc[2 * e] * P.scale, acc[2 * e + 1] * P.scale);
        if (rm != nullptr) *reinterpret_cast<uint4*>(rm + row * P.ld_rm + j) = make_uint4(w[0], w[1], w[2], w[3]);
        if (tr0 != nullptr && (P.tr_row_scale != nullptr || P.tr_row_scale_bf16 != nullptr)) {
            const float rs = P.tr_row_scale != nullptr ? P.tr_row_scale[row] : __bfloat162float(P.tr_row_scale_bf16[row]);
#pragma unroll
            for (int e = 0; e < 4; ++e)
                w[e] = pack_bf16(acc[2 * e] * P.scale * rs, acc[2 * e + 1] * P.scale * rs);
        }
        if (tr0 != nullptr) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int jj = j + e;
                const __nv_bfloat16 v = __ushort_as_bfloat16(static_cast<unsigned short>(e & 1 ? w[e >> 1] >> 16 : w[e >> 1] & 0xFFFFu));
                if (jj < P.tr_split) tr0[jj * P.ld_tr + row] = v;
                else tr1[(jj - P.tr_split) * P.ld_tr + row] = v;
            }
        }
    }
}

template <int NACC, int EPI>
__device__ __forceinline__ void epilogue_loop(const GemmArgs& a, uint32_t tmem_base, const SmemCtl& c) {
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int quarter = warp & 3;  // TMEM lanes this warp may access: [32*quarter, 32*quarter+32)
    int abuf = 0;
    uint32_t aphase = 0;
    const uint32_t acc_cols = NACC * a.bn;
    if (a.force_timeout) {
        wait_or_abort(c.never, 0, c);
        return;
    }
    for (int u = blockIdx.x; u < a.total_units; u += gridDim.x) {
        const Unit t = decode_unit(a, u);
        const Prob& P = a.prob[t.p];
        if (!wait_or_abort(c.accf + 8u * abuf, aphase, c)) return;
        tc_fence_after();
        EpiOut o;
        o.out0 = P.out0;
        o.out1 = P.out1;
        o.out2 = P.out2;
        o.in0 = P.in0;
        o.in1 = P.in1;
        o.ld = P.ld;
        o.split_off = t.ks * P.split_stride;
        o.M = P.M;
        o.N = P.N;
        o.row_scale = nullptr;
        const int row = t.mb * kBM + quarter * 32 + lane;
        const uint32_t tacc = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + abuf * acc_cols;
        epilogue_tile<NACC, EPI>(o, row, t.nb * a.bn, a.bn, TmemSrc{tacc});
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(c.acce + 8u * abuf);
        if (++abuf == 2) {
            abuf = 0;
            aphase ^= 1u;
        }
        if constexpr (EPI == EPI_F32) {
            if (P.counters != nullptr) splitk_finalize(P, t, row, c.fin_flag);
        }
    }
}

// ---------------------------------------------------------------------------
// kernel

__host__ __device__ constexpr uint32_t gemm_ctl_bytes() { return 8u * (2 * kMaxStages + 6) + 16u + 8u * kMaxStages; }

// Barrier/flag block that follows the operand stages in shared memory.
__device__ __forceinline__ SmemCtl make_ctl(uint32_t ctl, uint8_t* ctl_ptr, long long wait_limit) {
    SmemCtl c;
    c.full = ctl;
    c.empty = ctl + 8u * kMaxStages;
    c.accf = ctl + 8u * (2 * kMaxStages);
    c.acce = c.accf + 16u;
    c.drain = c.acce + 16u;
    c.never = c.drain + 8u;
    c.tmem_slot = c.never + 8u;
    c.rawf = c.tmem_slot + 16u;
    c.wait_limit = wait_limit;
    c.abort_flag = reinterpret_cast<volatile int*>(ctl_ptr + (c.tmem_slot + 4u - ctl));
    c.fin_flag = reinterpret_cast<volatile int*>(ctl_ptr + (c.tmem_slot + 8u - ctl));
    return c;
}

__host__ __device__ inline uint32_t gemm_tmem_cols(int nacc, int bn) {
    uint32_t need = 2u * nacc * bn, cols = 32;
    while (cols < need) cols <<= 1;
    return cols;
}

template <int NACC, int EPI>
// Up to two CTAs share an SM (launches with more units than SMs), so the
// register budget is that of two resident CTAs.
__global__ void __launch_bounds__(kGemmThreads, LMLP_MAX_CPS) umma_gemm_kernel(const __grid_constant__ GemmArgs args) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t stage_bytes = kATileBytes + NACC * args.b_bytes;
    const uint32_t ctl = base + args.stages * stage_bytes;
    uint8_t* ctl_ptr = smem_raw + (ctl - raw);

    const SmemCtl c = make_ctl(ctl, ctl_ptr, args.wait_limit);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t tmem_cols = gemm_tmem_cols(NACC, args.bn);

    // The tensor maps are launch parameters, not outputs of an earlier
    // launch: fetching them now overlaps that latency with the previous
    // kernel's tail (programmatic dependent launch).
    if (warp == 0 && lane < args.nmaps) tma_prefetch_desc(&args.maps[lane]);
    if (warp == 0 && lane == 0) {
        for (int s = 0; s < args.stages; ++s) {
            mbar_init(c.full + 8u * s, 1);
            mbar_init(c.empty + 8u * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(c.accf + 8u * b, 1);
            mbar_init(c.acce + 8u * b, 4);
        }
        mbar_init(c.drain, 1);
        mbar_init(c.never, 1);
        *c.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(c.tmem_slot, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(ctl_ptr + (c.tmem_slot - ctl));
#if LMLP_PDL
    // Everything above touched only this CTA's own resources; from here on
    // the kernel reads what the previous launch wrote.
    grid_dependency_wait();
    grid_launch_dependents();
#endif

    if (warp == 0) {
        if (lane == 0) {
            const long long issued = producer_loop<NACC>(args, base, stage_bytes, c);
            drain_loads(c.full, args.stages, issued, c.wait_limit);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            mma_loop<NACC>(args, base, stage_bytes, tmem_base, c);
            // Drain: wait until every MMA issued by this thread has finished
            // before TMEM is released (matters only after an abort).
            umma_commit(c.drain);
            const long long t0 = clock64();
            while (!mbar_try_wait(c.drain, 0)) {
                if (clock64() - t0 > c.wait_limit) break;
            }
        }
        __syncwarp();
    } else {
        epilogue_loop<NACC, EPI>(args, tmem_base, c);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, tmem_cols);
}

}  // namespace lmlp
