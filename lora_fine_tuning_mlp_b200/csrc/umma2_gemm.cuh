// Persistent tcgen05 GEMM on CTA pairs (cta_group::2) for the four large
// projections of the MLP.
//
// A 2-CTA cluster computes a 256 x 256 accumulator: each CTA TMA-loads its
// own 128 rows of A and its own 128-row half of B into its shared memory
// (plain loads, no multicast), the leader CTA issues M = 256 UMMAs that read
// both CTAs' operands, and each CTA's TMEM receives its 128 rows.  Per SM this
// moves half the B bytes of a 1-CTA 128 x 256 tile for the same work, which
// is what lets the TMA keep up with the tensor core.
//
// Synchronisation: both CTAs' loads count on the leader's "full" barrier
// (TMA with .cta_group::2); the leader's tcgen05.commit multicasts to the
// "empty" and "acc-full" barriers of both CTAs; both CTAs' epilogue warps
// arrive on the leader's "acc-empty" barrier.  Every wait is bounded.
//
// The B halves are addressed per segment (map, row offset, K offset), so the
// same kernel serves
//   * single outputs (tile = 256 output columns, halves = rows n0 and n0+128), and
//   * the gate/up pair (tile = 128 output columns; half 0 = Wg rows, half 1 =
//     Wu rows, accumulator columns [0,128) = G and [128,256) = U).  Their
//     rank-r extension is one K = 2r segment: A = [S_g | S_u], half 0 reads
//     Bg at K offset 0 and half 1 reads Bu at K offset -r, the zero fill of
//     out-of-range columns supplying the two zero blocks.
//
// Block-int4 frozen weights (the Q4 instantiation) are dequantised inside
// the kernel: for a segment whose B is int4, each CTA's producer brings the
// packed codes of its B half into a small "raw" slot of the stage by TMA,
// four dequant warps turn them into bf16 in the 128-byte-swizzled layout the
// tensor core reads (the same bytes a TMA load of the bf16 weight would have
// written), and arrive on the leader's full barrier.  The bf16 copy of the
// weight never exists in global memory.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "aux_kernels.cuh"
#include "epilogue.cuh"
#include "ptx.cuh"
#include "umma_gemm.cuh"

namespace lmlp {

constexpr int kPairBM = 256;
constexpr int kPairHalfN = 128;
constexpr uint32_t kPairBBytes = kPairHalfN * kBK * 2;                  // 16 KB per CTA
constexpr uint32_t kPairStageBytes = kATileBytes + kPairBBytes;         // 32 KB per CTA
#ifndef LMLP_PAIR_STAGES
#define LMLP_PAIR_STAGES 6  // 6 x 32 KB: as fast as 7 (measured), leaves room for the store staging
#endif
constexpr int kPairMaxStages = LMLP_PAIR_STAGES;
constexpr uint32_t kPairTmemCols = 512;                                 // 2 buffers x 256 columns

// Epilogue warps of a CTA-pair launch, by epilogue kind: 4 (one per TMEM
// lane quarter) or 8 (two per quarter, each taking half of the tile's
// columns).  Ten warps leave 168 registers a thread (three warps on two of
// the SM's four sub-partitions).  With g and u loaded into registers, 8 warps
// made the dH GEMM 1-2 % faster than 4; with the cp.async ring below, 4 warps
// are faster, since 8 rings leave room for only three operand stages.
#ifndef LMLP_PAIR_EPI_WARPS_BF16
#define LMLP_PAIR_EPI_WARPS_BF16 4
#endif
#ifndef LMLP_PAIR_EPI_WARPS_FWD
#define LMLP_PAIR_EPI_WARPS_FWD 4
#endif
#ifndef LMLP_PAIR_EPI_WARPS_BWD
#define LMLP_PAIR_EPI_WARPS_BWD 4
#endif
static_assert(LMLP_PAIR_EPI_WARPS_BF16 % 4 == 0 && LMLP_PAIR_EPI_WARPS_BF16 <= 8, "4 or 8 epilogue warps");
static_assert(LMLP_PAIR_EPI_WARPS_FWD % 4 == 0 && LMLP_PAIR_EPI_WARPS_FWD <= 8, "4 or 8 epilogue warps");
static_assert(LMLP_PAIR_EPI_WARPS_BWD % 4 == 0 && LMLP_PAIR_EPI_WARPS_BWD <= 8, "4 or 8 epilogue warps");
template <int EPI>
__host__ __device__ constexpr int pair_epi_warps() {
    return EPI == EPI_SWIGLU_BWD ? LMLP_PAIR_EPI_WARPS_BWD
                                 : (EPI == EPI_SWIGLU_FWD ? LMLP_PAIR_EPI_WARPS_FWD : LMLP_PAIR_EPI_WARPS_BF16);
}
// int4 B: the launch runs four warpgroups.  WG0: the producer (warp 0) and
// the MMA issuer (warp 1), warps 2 and 3 idle; WG1 (warps 4-7): the
// epilogue; WG2 and WG3 (warps 8-15): the dequant warps, WG2 converting the
// even stages of the K sequence and WG3 the odd ones, one 64-element line
// (one scale) per thread: the 128 rows of a K-major B half, or the 64 K rows
// x two 64-column chunks of an MN-major one.  The expansion is bound by the
// integer pipe's issue rate: one warp per SM sub-partition took ~640 cycles
// per stage against the tensor core's 512, two ~430 (measured).  So that
// sixteen warps fit, setmaxnreg moves registers from the producer/MMA and
// dequant warpgroups to the epilogue's.
constexpr int kQ4Warps = 4;  // dequant warps of one CTA that arrive per stage (one warpgroup)
constexpr int kQ4Groups = 2;
constexpr int kQ4RegsCtl = 80, kQ4RegsEpi = 232, kQ4RegsDq = 88;
static_assert(128 * (kQ4RegsCtl + kQ4RegsEpi) + 256 * kQ4RegsDq <= 512 * 128,
              "the warpgroups' register counts must fit the 128 a thread of a 512-thread block launches with");
// Frozen-weight formats of the B operand: bf16 (TMA straight into the
// stage), block-int4 or block-FP8 (codes and scales into a raw slot of the
// stage, expanded by the dequant warps).
enum : int { QF_NONE = 0, QF_INT4 = 1, QF_FP8 = 2 };
// Per CTA and stage: codes of the 128 x 64 B half (4 KB of nibbles, 8 KB of
// E4M3 bytes), its 128 scales (fp16 or fp32), and the raw slot they share,
// rounded so that stages stay 1 KB aligned.
template <int QF>
__host__ __device__ constexpr uint32_t q_code_bytes() {
    return QF == QF_FP8 ? kPairHalfN * kBK : kPairHalfN * kBK / 2;
}
template <int QF>
__host__ __device__ constexpr uint32_t q_scale_bytes() {
    return QF == QF_FP8 ? kPairHalfN * 4 : kPairHalfN * 2;
}
template <int QF>
__host__ __device__ constexpr uint32_t q_raw_bytes() {
    return QF == QF_NONE ? 0u : (q_code_bytes<QF>() + q_scale_bytes<QF>() + 1023u) & ~1023u;
}
template <int QF>
__host__ __device__ constexpr uint32_t pair_stage_bytes() {
    return kPairStageBytes + q_raw_bytes<QF>();
}
template <int EPI, bool Q4 = false>
__host__ __device__ constexpr int pair_threads() {
    return Q4 ? 16 * 32 : (2 + pair_epi_warps<EPI>()) * 32;
}
// First epilogue warp: 2, or 4 (warpgroup 1) in an int4 launch.
template <bool Q4>
__host__ __device__ constexpr int pair_epi_first() {
    return Q4 ? 4 : 2;
}
// The dH epilogue's g and u stream through a per-warp ring of shared-memory
// slots filled by cp.async, LMLP_BWD_GU_RING chunks deep: the next chunk (at
// a tile's end, the next tile's first) is in flight while one computes, no
// registers hold it, and it lands row-major with no transpose.  0 loads g and
// u into registers instead.  Measured interleaved on the dH GEMM against the
// register path: TinyLlama-1.1B shapes 1027 -> 812 us, Qwen2-7B 1047 -> 1010
// us, Llama-3-8B within noise (476 -> 468 us).  Deeper rings (3, 4 chunks)
// cost an operand stage and measured slower on two of the three shapes.
#ifndef LMLP_BWD_GU_RING
#define LMLP_BWD_GU_RING 2
#endif
constexpr int kGuRing = LMLP_BWD_GU_RING;
static_assert(kGuRing == 0 || kGuRing >= 2, "a ring holds at least two chunks");
// Ring slot layout: 1 = 64-byte rows in the 64-byte swizzle (16-byte piece q
// of row R at piece q ^ ((R / 2) mod 4)), so that both the coalesced
// cp.async writes (two rows per quarter-warp) and the per-row reads (eight
// rows per quarter-warp) touch every bank once; 0 = 80-byte padded rows,
// whose cp.async writes conflict.  Measured interleaved (medians, identical
// bits): Llama-3-8B 456 -> 453 us, TinyLlama-1.1B 802 -> 796 us, Qwen2-7B
// 1009 -> 985 us.  A three-deep ring with two TMA-store buffers a warp (same
// shared memory, five stages) measured within noise of it; every layout
// that left four operand stages was 3-8 % slower.
#ifndef LMLP_BWD_GU_SWZ
#define LMLP_BWD_GU_SWZ 1
#endif
constexpr bool kGuSwz = LMLP_BWD_GU_SWZ != 0;
constexpr uint32_t kGuHalfBytes = kGuSwz ? 32u * 64u : kStageWarpBytes;  // g (then u) of one 32 x 32 chunk
constexpr uint32_t kGuSlotBytes = 2 * kGuHalfBytes;
template <int EPI>
__host__ __device__ constexpr uint32_t pair_ring_bytes() {
    return (EPI == EPI_SWIGLU_BWD && kGuRing > 0) ? pair_epi_warps<EPI>() * kGuRing * kGuSlotBytes : 0u;
}
// TMA-store buffers a warp of the dH epilogue cycles through (the others use
// kTmaBufs).
#ifndef LMLP_BWD_TMA_BUFS
#define LMLP_BWD_TMA_BUFS 3
#endif
constexpr int kBwdTmaBufs = LMLP_BWD_TMA_BUFS;
// bf16 outputs leave through TMA stores (32 x 32 blocks staged in shared
// memory) instead of per-lane stores, by epilogue kind.  Measured
// interleaved against the transposing per-lane stores: the SwiGLU epilogues
// (three outputs per chunk) 1.5-3 % faster on the Llama-3-8B and
// TinyLlama-1.1B shapes, within noise on Qwen2-7B; the single bf16 output
// (stored directly, no transpose) no faster, so it keeps per-lane stores.
#ifndef LMLP_PAIR_TMA_STORE_BF16
#define LMLP_PAIR_TMA_STORE_BF16 0
#endif
#ifndef LMLP_PAIR_TMA_STORE_FWD
#define LMLP_PAIR_TMA_STORE_FWD 1
#endif
#ifndef LMLP_PAIR_TMA_STORE_BWD
#define LMLP_PAIR_TMA_STORE_BWD 1
#endif
template <int EPI>
__host__ __device__ constexpr bool pair_tma_store() {
    return EPI == EPI_SWIGLU_BWD ? LMLP_PAIR_TMA_STORE_BWD != 0
                                 : (EPI == EPI_SWIGLU_FWD ? LMLP_PAIR_TMA_STORE_FWD != 0 : LMLP_PAIR_TMA_STORE_BF16 != 0);
}
// Shared memory after the barrier block, per epilogue warp: store staging
// (transposes or TMA-store buffers; none for direct bf16 stores).
template <int EPI>
__host__ __device__ constexpr uint32_t pair_stage_warp_bytes() {
    return pair_tma_store<EPI>()
               ? (EPI == EPI_SWIGLU_BWD && kGuRing > 0 ? kBwdTmaBufs * kTmaBlockBytes : kTmaWarpBytes)
               : (EPI == EPI_BF16 ? 0u : kStageWarpBytes);
}
// Start of the epilogue's shared memory: 512-byte aligned, as the TMA-store
// buffers' swizzle requires.
__device__ __forceinline__ uint32_t pair_epi_area(const SmemCtl& c) {
    return (c.full + gemm_ctl_bytes() + 511u) & ~511u;
}
// Named barrier 1 over the epilogue warps.
template <int EPI>
__device__ __forceinline__ void pair_epi_bar() {
    asm volatile("bar.sync 1, %0;" ::"n"(pair_epi_warps<EPI>() * 32) : "memory");
}

struct PairSeg {
    int a_map;
    int b_map[2];  // B half 0 / half 1
    int b_row[2];  // N-row offset of each half from the tile's first B row
    int b_k[2];    // K-coordinate offset of each half
    int kblocks;
    int k_len;
    // int4 B (Q4 launches): the codes come through the uint8 maps qmap
    // (K-major: [rows, K/2], box 32 B x 128 rows; MN-major: [K, cols/2], box
    // 32 B x 64 rows) and the scales through smap, maps of their transpose
    // [cols/64, rows] (K-major: box 128 x 1; MN-major: box 64 x 1), both into
    // the stage's raw slot.  Outside the weight both read as TMA's zero fill,
    // so those lines dequantise to zeros.
    int q4;
    int qmap[2];
    int smap[2];
};

struct PairProb {
    int M, N;    // output rows / columns
    int tile_n;  // output columns per tile (256, or 128 for the gate/up pair)
    int tiles_m, tiles_n, nkb, nsegs;
    PairSeg seg[kMaxSegs];
    void* out0;
    void* out1;
    void* out2;
    const void* in0;
    const void* in1;
    long long ld;
    int omap[3];  // tensor maps of out0..out2 for TMA stores (when the kind uses them)
    const float* row_scale;  // EPI_SWIGLU_FWD: optional factor of each output row (see EpiOut)
};

// Tail split (stream-K for the last partial wave): the first `full_units`
// tiles run whole; each of the remaining tiles is cut into `tail_splits`
// K ranges run by different clusters, so the last round takes a fraction of
// a tile's time instead of a whole one.  Each CTA of such a unit stores its
// fp32 accumulator rows in `tail_part`; the CTA that finishes a (tile, rank)
// last (counter in `tail_ctr`) adds the partials in split order and runs the
// real epilogue on the sum.
struct alignas(64) PairArgs {
    CUtensorMap maps[kMaxMaps];
    PairProb prob;
    int total_units;
    int full_units;
    int tail_splits;
    int stages;
    int group_m;
    float* tail_part;  // [tail tile][split][rank][128 rows][256 columns]
    int* tail_ctr;     // [tail tile][rank], zero before the launch
    long long wait_limit;  // SM cycles a barrier wait may spin before the kernel gives up
    int force_timeout;     // test hook: the epilogue waits on a barrier nothing signals
    int nmaps;             // maps[0, nmaps) are encoded
};

struct PairUnit {
    int mb, nb, kb0, kb1;
    int tail;  // -1 for a whole tile, else the tail tile index
    int ks;
};

__device__ __forceinline__ PairUnit pair_decode(const PairArgs& a, int u) {
    const PairProb& P = a.prob;
    PairUnit r;
    int tile;
    if (u < a.full_units) {
        tile = u;
        r.tail = -1;
        r.ks = 0;
        r.kb0 = 0;
        r.kb1 = P.nkb;
    } else {
        const int v = u - a.full_units;
        r.tail = v / a.tail_splits;
        r.ks = v - r.tail * a.tail_splits;
        tile = a.full_units + r.tail;
        r.kb0 = static_cast<int>((static_cast<long long>(r.ks) * P.nkb) / a.tail_splits);
        r.kb1 = static_cast<int>((static_cast<long long>(r.ks + 1) * P.nkb) / a.tail_splits);
    }
    const int per_group = a.group_m * P.tiles_n;
    const int grp = tile / per_group;
    const int first_m = grp * a.group_m;
    const int gsz = min(a.group_m, P.tiles_m - first_m);
    const int local = tile - grp * per_group;
    r.mb = first_m + local % gsz;
    r.nb = local / gsz;
    return r;
}

// Returns the number of stages it filled.  Both CTAs' loads of a stage
// count on the leader's full barrier, so the leader's count is what
// drain_loads needs.
template <bool B_MN, int QF>
__device__ __forceinline__ long long pair_producer(const PairArgs& a, uint32_t base, uint32_t rank, bool leader,
                                                   const SmemCtl& c) {
    constexpr bool Q4 = QF != QF_NONE;
    constexpr uint32_t kSB = pair_stage_bytes<QF>();
    constexpr uint32_t kCode = q_code_bytes<QF>(), kScale = q_scale_bytes<QF>();
    const PairProb& P = a.prob;
    long long issued = 0;
    const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
    int stage = 0;
    uint32_t phase = 0;
    for (int u = cid; u < a.total_units; u += ncl) {
        const PairUnit t = pair_decode(a, u);
        const int mb = t.mb, nb = t.nb;
        int seg = 0, seg_kb0 = 0;
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
            while (kb >= seg_kb0 + P.seg[seg].kblocks) {
                seg_kb0 += P.seg[seg].kblocks;
                ++seg;
            }
            const PairSeg& S = P.seg[seg];
            const int k0 = (kb - seg_kb0) * kBK;
            if (!wait_or_abort(c.empty + 8u * stage, phase ^ 1u, c)) return issued;
            const bool q4 = Q4 && S.q4 != 0;
            const uint32_t fb_local = c.full + 8u * stage;
            // int4 B reaches the stage through the dequant warps, whose
            // arrivals (not bytes) the full barrier counts
            if (leader) mbar_arrive_expect_tx(fb_local, q4 ? 2u * kATileBytes : 2u * kPairStageBytes);
            const uint32_t fb = mapa_shared(fb_local, 0);
            const uint32_t sA = base + stage * kSB;
            const uint32_t sB = sA + kATileBytes;
            tma_load_2d_pair(sA, &a.maps[S.a_map], fb, k0, mb * kPairBM + static_cast<int>(rank) * kBM);
            const int brow = nb * P.tile_n + S.b_row[rank];
            const int bk = k0 + S.b_k[rank];
            if (q4) {
                // the codes of this CTA's B half into the raw slot, counted on
                // this CTA's own raw barrier (x in bytes: brow and bk are
                // multiples of 64, so x is 16-byte aligned)
                const uint32_t rf = c.rawf + 8u * stage;
                const uint32_t raw = sA + kPairStageBytes;
                const CUtensorMap* qm = &a.maps[S.qmap[rank]];
                const CUtensorMap* sm = &a.maps[S.smap[rank]];
                // x of a code box in bytes: half an element per nibble, one per E4M3 byte
                constexpr int kSh = QF == QF_FP8 ? 0 : 1;
                mbar_arrive_expect_tx(rf, kCode + kScale);
                if (B_MN) {
                    tma_load_2d(raw, qm, rf, brow >> kSh, bk);
                    tma_load_2d(raw + kCode / 2, qm, rf, (brow + 64) >> kSh, bk);
                    tma_load_2d(raw + kCode, sm, rf, bk, brow >> 6);
                    tma_load_2d(raw + kCode + kScale / 2, sm, rf, bk, (brow >> 6) + 1);
                } else {
                    tma_load_2d(raw, qm, rf, bk >> kSh, brow);
                    tma_load_2d(raw + kCode, sm, rf, brow, bk >> 6);
                }
            } else {
                const CUtensorMap* bm = &a.maps[S.b_map[rank]];
                if (B_MN) {
                    tma_load_2d_pair(sB, bm, fb, brow, bk);
                    tma_load_2d_pair(sB + 8192u, bm, fb, brow + 64, bk);
                } else {
                    tma_load_2d_pair(sB, bm, fb, bk, brow);
                }
                if (Q4) mbar_arrive(c.rawf + 8u * stage);  // nothing to convert: release the dequant warps
            }
            ++issued;
            if (++stage == a.stages) {
                stage = 0;
                phase ^= 1u;
            }
        }
    }
    return issued;
}

// The MMA issuer.  One thread feeds the tensor core, and on the projection
// shapes it is the bottleneck unless its loop is short: the tensor core takes
// 512 cycles per 64-wide K block of a 256 x 256 pair tile, and every
// instruction of this loop is a dependent step of a single thread.  So the
// loop walks the segments directly (only the last block of a segment can be
// partial) and forms each stage's descriptors by adding offsets to those of
// stage 0 instead of re-encoding them.  Measured on the Llama-3-8B MLP
// shapes: 725-811 -> 574-681 SM cycles per K block.
template <bool B_MN, int QF>
__device__ __forceinline__ void pair_mma(const PairArgs& a, uint32_t base, uint32_t tmem_base, const SmemCtl& c) {
    constexpr bool Q4 = QF != QF_NONE;
    const PairProb& P = a.prob;
    const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
    const uint32_t idesc = idesc_bf16(256u, false, B_MN, 256u);
    // Stage s adds s * kPairStageBytes to both start addresses (the 14-bit
    // address field holds bytes >> 4 and cannot carry: shared memory < 256 KB).
    const uint64_t a0 = sw128_desc(base, 16u, 1024u);
    const uint64_t b0 = B_MN ? sw128_desc(base + kATileBytes, 8192u, 1024u)
                             : sw128_desc(base + kATileBytes, 16u, 1024u);
    constexpr uint32_t kStageStep = pair_stage_bytes<QF>() >> 4;
    constexpr uint32_t kAStep = 32u >> 4;                        // next 16-wide K slice of A
    constexpr uint32_t kBStep = B_MN ? (2048u >> 4) : (32u >> 4);  // ... of B
    int stage = 0;
    uint32_t phase = 0;
    int abuf = 0;
    uint32_t aphase = 0;
    for (int u = cid; u < a.total_units; u += ncl) {
        const PairUnit t = pair_decode(a, u);
        if (!wait_or_abort(c.acce + 8u * abuf, aphase ^ 1u, c)) return;
        tc_fence_after();
        const uint32_t d = tmem_base + abuf * 256u;
        uint32_t acc = 0;
        int seg_kb0 = 0;
        for (int sg = 0; sg < P.nsegs; ++sg) {
            const int nkb = P.seg[sg].kblocks;
            const int lo = max(t.kb0 - seg_kb0, 0), hi = min(t.kb1 - seg_kb0, nkb);
            const int k_len = P.seg[sg].k_len;
            seg_kb0 += nkb;
            for (int kb = lo; kb < hi; ++kb) {
                // int4: the other CTA's dequant warps wrote its B half
                if (!wait_or_abort<Q4>(c.full + 8u * stage, phase, c)) return;
                tc_fence_after();
                const uint64_t ad = a0 + static_cast<uint64_t>(stage * kStageStep);
                const uint64_t bd = b0 + static_cast<uint64_t>(stage * kStageStep);
                const int nk = kb == nkb - 1 ? ((k_len - kb * kBK + 15) >> 4) : 4;
                if (nk == 4) {
                    umma_bf16_pair(d, ad, bd, idesc, acc);
                    umma_bf16_pair(d, ad + kAStep, bd + kBStep, idesc, 1u);
                    umma_bf16_pair(d, ad + 2u * kAStep, bd + 2u * kBStep, idesc, 1u);
                    umma_bf16_pair(d, ad + 3u * kAStep, bd + 3u * kBStep, idesc, 1u);
                } else {
                    for (int k = 0; k < nk; ++k)
                        umma_bf16_pair(d, ad + k * kAStep, bd + k * kBStep, idesc, (acc | k) ? 1u : 0u);
                }
                acc = 1u;
                umma_commit_pair(c.empty + 8u * stage, 3);
                if (++stage == a.stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        umma_commit_pair(c.accf + 8u * abuf, 3);
        if (++abuf == 2) {
            abuf = 0;
            aphase ^= 1u;
        }
    }
}

// The dequant warps of an int4 launch, one warpgroup per parity of the
// position in the (unit, K block) sequence the producer walks.  For each of
// its stages a warpgroup waits for the stage's raw barrier; if the stage's B
// is int4, each thread reads its line's 32 code bytes and its scale from the
// raw slot, expands them (int4_line) and writes the 128 bytes into the
// stage's B tile at the 128-byte swizzle (16-byte piece w of tile row R at
// piece w ^ (R mod 8)), then fences its writes to the async proxy.  Each warp
// then arrives once on the leader's full barrier.  Every input arrives by
// TMA: the warps hold no outstanding global loads that their arrive would
// wait for.
// A stage is always converted by the same warpgroup (stage index mod 2), so
// successive uses of a stage's barriers come from one warpgroup working in
// order, never more than one phase behind them; with an odd stage count the
// warpgroups' shares differ by one stage in S.  (Splitting by the position's
// parity instead lets, with an odd count, one warpgroup run two phases ahead
// of the other on a stage, and the barrier's phase parity aliases: seen as a
// few stale lines per launch on the Llama-3-8B int4 shapes.)
template <bool B_MN, int QF>
__device__ __forceinline__ void pair_dequant(const PairArgs& a, uint32_t base, const SmemCtl& c, int group, int t) {
    const PairProb& P = a.prob;
    const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
    const int lane = threadIdx.x & 31;
    constexpr uint32_t kSB = pair_stage_bytes<QF>();
    constexpr uint32_t kCode = q_code_bytes<QF>();
    constexpr uint32_t kLineBytes = QF == QF_FP8 ? 64u : 32u;  // code bytes of one 64-element line
    const int lrow = B_MN ? (t & 63) : t;  // tile row: N row (K-major) or K row (MN-major)
    const int lj = B_MN ? (t >> 6) : 0;    // 64-column chunk (MN-major)
    const uint32_t raw_off = kPairStageBytes + static_cast<uint32_t>(lj) * (kCode / 2) +
                             static_cast<uint32_t>(lrow) * kLineBytes;
    // the scales: one 128-entry run (K-major), or one 64-entry run per chunk
    const uint32_t sc_off = kPairStageBytes + kCode + static_cast<uint32_t>(t) * (QF == QF_FP8 ? 4u : 2u);
    const uint32_t out_off = kATileBytes + static_cast<uint32_t>(lj) * 8192u + static_cast<uint32_t>(lrow) * 128u;
    const uint32_t swz = static_cast<uint32_t>(lrow & 7);
    // read order of the two 16-byte halves: alternating every four rows puts
    // the eight rows of a quarter-warp on distinct bank groups
    const uint32_t h0 = static_cast<uint32_t>((lrow >> 2) & 1) * 16u;
    int stage = 0;
    uint32_t phase = 0;
    for (int u = cid; u < a.total_units; u += ncl) {
        const PairUnit tu = pair_decode(a, u);
        int seg = 0, seg_kb0 = 0;
        for (int kb = tu.kb0; kb < tu.kb1; ++kb) {
            while (kb >= seg_kb0 + P.seg[seg].kblocks) {
                seg_kb0 += P.seg[seg].kblocks;
                ++seg;
            }
            if ((stage & 1) == group) {
                if (!wait_or_abort(c.rawf + 8u * stage, phase, c)) return;
                if (P.seg[seg].q4) {
                    const uint32_t sb = base + static_cast<uint32_t>(stage) * kSB;
                    uint4 o[8];
                    if constexpr (QF == QF_FP8) {
                        // 64-byte code rows land in TMA's 64-byte swizzle: 16-byte
                        // piece q of row R at piece q ^ ((R / 2) mod 4), so the
                        // eight rows of a quarter-warp hit distinct bank groups
                        const uint32_t sw = static_cast<uint32_t>((lrow >> 1) & 3);
                        uint4 x[4];
#pragma unroll
                        for (uint32_t q = 0; q < 4; ++q) x[q] = lds128(sb + raw_off + ((q ^ sw) << 4));
                        fp8_line(x, __uint_as_float(lds32(sb + sc_off)), o);
                    } else {
                        const uint4 x0 = lds128(sb + raw_off + h0);
                        const uint4 x1 = lds128(sb + raw_off + (h0 ^ 16u));
                        const float sc = __half2float(__ushort_as_half(lds16(sb + sc_off)));
                        int4_line(h0 ? x1 : x0, h0 ? x0 : x1, sc, o);
                    }
#pragma unroll
                    for (uint32_t w = 0; w < 8; ++w) sts128(sb + out_off + ((w ^ swz) << 4), o[w]);
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(mapa_shared(c.full + 8u * stage, 0));
            }
            if (++stage == a.stages) {
                stage = 0;
                phase ^= 1u;
            }
        }
    }
}

// The dH + SwiGLU-backward epilogue with g and u streamed through the
// warp's cp.async ring.  The warp walks the same (unit, chunk) sequence twice:
// an issue cursor kGuRing - 1 chunks ahead fills ring slots (zeros outside
// the matrix), and the consumer reads its row of each chunk back from shared
// memory.  Each chunk is one cp.async group, so waiting until kGuRing - 1
// groups remain in flight means the oldest chunk has landed.
template <int EPI, int kFirst>
__device__ __forceinline__ void pair_epilogue_bwd_ring(const PairArgs& a, uint32_t tmem_base, uint32_t rank,
                                                       const SmemCtl& c) {
    const PairProb& P = a.prob;
    const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int quarter = warp & 3;
    constexpr int kGroups = pair_epi_warps<EPI>() / 4;
    const int group = (warp - kFirst) >> 2;
    const int gcols = 256 / kGroups;
    const int gcol0 = group * gcols;
    const int nch = gcols >> 5;
    const uint32_t area = pair_epi_area(c);
    const uint32_t stg = area + static_cast<uint32_t>(warp - kFirst) * pair_stage_warp_bytes<EPI>();
    const uint32_t ring = area + pair_epi_warps<EPI>() * pair_stage_warp_bytes<EPI>() +
                          static_cast<uint32_t>(warp - kFirst) * (kGuRing * kGuSlotBytes);
    TmaStoreN<kBwdTmaBufs> ts;
    ts.map[0] = &a.maps[P.omap[0]];
    ts.map[1] = &a.maps[P.omap[1]];
    ts.map[2] = &a.maps[P.omap[2]];
    ts.buf = stg;
    ts.next = 0;
    const __nv_bfloat16* gbase = static_cast<const __nv_bfloat16*>(P.in0);
    const __nv_bfloat16* ubase = static_cast<const __nv_bfloat16*>(P.in1);
    if (a.force_timeout) {
        wait_or_abort(c.never, 0, c);
        return;
    }
    // issue cursor: unit iu, chunk ich, its first row and column, next slot
    int iu = cid, ich = 0, irow0 = 0, icol0 = 0;
    uint32_t islot = 0;
    auto set_unit = [&]() {
        if (iu < a.total_units) {
            const PairUnit ti = pair_decode(a, iu);
            irow0 = ti.mb * kPairBM + static_cast<int>(rank) * kBM + quarter * 32;
            icol0 = ti.nb * P.tile_n + gcol0;
        }
    };
    // 16-byte piece (row 8q + lane/4, columns 8 (lane%4) ..) of a chunk, as in
    // a coalesced load: four lanes cover one row's 64 bytes.  With the
    // swizzled slots, rows 8q + lane/4 have (row / 2) mod 4 = (lane / 8) mod 4.
    const int prow = lane >> 2, pcol = 8 * (lane & 3);
    constexpr uint32_t kRowB = kGuSwz ? 64u : kStageRowBytes;
    const uint32_t ppiece = kGuSwz ? ((static_cast<uint32_t>(lane & 3) ^ (static_cast<uint32_t>(lane >> 3) & 3u)) << 4)
                                   : static_cast<uint32_t>(lane & 3) * 16u;
    const uint32_t poff = static_cast<uint32_t>(prow) * kRowB + ppiece;
    auto issue = [&]() {
        if (iu < a.total_units) {
            const uint32_t sb = ring + islot * kGuSlotBytes + poff;
            const int cc = icol0 + ich * 32 + pcol;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int r = irow0 + 8 * q + prow;
                const bool ok = r < P.M && cc < P.N;
                const long long off = ok ? static_cast<long long>(r) * P.ld + cc : 0;
                cp_async16(sb + q * 8 * kRowB, gbase + off, ok ? 16u : 0u);
                cp_async16(sb + kGuHalfBytes + q * 8 * kRowB, ubase + off, ok ? 16u : 0u);
            }
            if (++ich == nch) {
                ich = 0;
                iu += ncl;
                set_unit();
            }
        }
        cp_async_commit();
        if (++islot == static_cast<uint32_t>(kGuRing)) islot = 0;
    };
    set_unit();
#pragma unroll 1
    for (int k = 0; k < kGuRing - 1; ++k) issue();

    int abuf = 0;
    uint32_t aphase = 0;
    uint32_t cslot = 0;
    for (int u = cid; u < a.total_units; u += ncl) {
        const PairUnit t = pair_decode(a, u);
        if (!wait_or_abort(c.accf + 8u * abuf, aphase, c)) {
            cp_async_wait_all();
            if constexpr (pair_tma_store<EPI>()) ts.drain();
            return;
        }
        tc_fence_after();
        const int row = t.mb * kPairBM + static_cast<int>(rank) * kBM + quarter * 32 + lane;
        const uint32_t tacc =
            tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + abuf * 256u + static_cast<uint32_t>(gcol0);
        for (int ch = 0; ch < nch; ++ch) {
            issue();
            cp_async_wait<(kGuRing > 0 ? kGuRing - 1 : 0)>();
            __syncwarp();
            const int col0 = t.nb * P.tile_n + gcol0 + ch * 32;
            if (col0 < P.N) {  // warp-uniform
                uint32_t v[32];
                tmem_ld32(tacc + ch * 32, v);
                const uint32_t rb = ring + cslot * kGuSlotBytes + static_cast<uint32_t>(lane) * kRowB;
                const uint32_t rsw = kGuSwz ? (static_cast<uint32_t>(lane >> 1) & 3u) : 0u;
                uint4 gv[4], uv[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t pq = (static_cast<uint32_t>(q) ^ rsw) << 4;
                    gv[q] = lds128(rb + pq);
                    uv[q] = lds128(rb + kGuHalfBytes + pq);
                }
                tmem_ld_wait();
                uint4 dgq[4], duq[4], hq[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) swiglu_bwd8(v + 8 * q, gv[q], uv[q], dgq[q], duq[q], hq[q]);
                if constexpr (pair_tma_store<EPI>()) {
                    ts.emit(0, col0, row - lane, dgq);
                    ts.emit(1, col0, row - lane, duq);
                    ts.emit(2, col0, row - lane, hq);
                } else {
                    emit_chunk(static_cast<__nv_bfloat16*>(P.out0), P.ld, row, col0, P.M, P.N, dgq, stg);
                    emit_chunk(static_cast<__nv_bfloat16*>(P.out1), P.ld, row, col0, P.M, P.N, duq, stg);
                    emit_chunk(static_cast<__nv_bfloat16*>(P.out2), P.ld, row, col0, P.M, P.N, hq, stg);
                }
            }
            __syncwarp();
            if (++cslot == static_cast<uint32_t>(kGuRing)) cslot = 0;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(c.acce + 8u * abuf, 0));
        if (++abuf == 2) {
            abuf = 0;
            aphase ^= 1u;
        }
    }
    cp_async_wait_all();
    if constexpr (pair_tma_store<EPI>()) ts.drain();
}

template <int EPI, int kFirst>
__device__ __forceinline__ void pair_epilogue(const PairArgs& a, uint32_t tmem_base, uint32_t rank,
                                              const SmemCtl& c) {
    if constexpr (EPI == EPI_SWIGLU_BWD && kGuRing > 0) {
        pair_epilogue_bwd_ring<EPI, kFirst>(a, tmem_base, rank, c);
        return;
    }
    constexpr int NACC = EPI == EPI_SWIGLU_FWD ? 2 : 1;
    const PairProb& P = a.prob;
    const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int quarter = warp & 3;
    // With 8 epilogue warps, warps 2-5 and 6-9 take the two column halves.
    constexpr int kGroups = pair_epi_warps<EPI>() / 4;
    // Two groups hold half the registers per thread: they load g and u chunk
    // by chunk instead of one chunk ahead.
    constexpr bool kPrefetch = kGroups == 1;
    const int group = (warp - kFirst) >> 2;
    EpiOut o;
    o.out0 = P.out0;
    o.out1 = P.out1;
    o.out2 = P.out2;
    o.in0 = P.in0;
    o.in1 = P.in1;
    o.ld = P.ld;
    o.split_off = 0;
    o.M = P.M;
    o.N = P.N;
    o.row_scale = P.row_scale;
    const int bn = 256 / NACC;               // columns of each accumulator
    const int gcols = bn / kGroups;          // of which this warp's group takes
    const int gcol0 = group * gcols;
    // This warp's staging area for coalesced stores, after the barrier block.
    // Used by the SwiGLU epilogues (three outputs per chunk); the single bf16
    // output stores directly (measured interleaved: staging helps the former
    // by 1-2% and costs the latter about as much).
    const uint32_t stg = pair_stage_warp_bytes<EPI>() == 0u
                             ? 0u
                             : pair_epi_area(c) + static_cast<uint32_t>(warp - kFirst) * pair_stage_warp_bytes<EPI>();
    TmaStore tsv;
    TmaStore* ts = nullptr;
    if constexpr (pair_tma_store<EPI>()) {
        tsv.map[0] = &a.maps[P.omap[0]];
        tsv.map[1] = &a.maps[P.omap[1]];
        tsv.map[2] = &a.maps[P.omap[2]];
        tsv.buf = stg;
        tsv.next = 0;
        ts = &tsv;
    }
    int abuf = 0;
    uint32_t aphase = 0;
    if (a.force_timeout) {
        wait_or_abort(c.never, 0, c);
        return;
    }
    for (int u = cid; u < a.total_units; u += ncl) {
        const PairUnit t = pair_decode(a, u);
        if (!wait_or_abort(c.accf + 8u * abuf, aphase, c)) {
            if (ts != nullptr) ts->drain();
            return;
        }
        tc_fence_after();
        const int lrow = quarter * 32 + lane;  // row within this CTA's 128
        const int row = t.mb * kPairBM + static_cast<int>(rank) * kBM + lrow;
        const uint32_t tacc = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + abuf * 256u;
        float* part = nullptr;
        if (t.tail < 0) {
            epilogue_tile<NACC, EPI, TmemSrc, kPrefetch>(o, row, t.nb * P.tile_n + gcol0, gcols,
                                                         TmemSrc{tacc + static_cast<uint32_t>(gcol0)}, stg, bn, ts);
        } else {
            // this split's accumulator rows (this group's columns) -> fp32 partial
            part = a.tail_part + ((static_cast<long long>(t.tail) * a.tail_splits + t.ks) * 2 + rank) * (kBM * 256ll) +
                   lrow * 256ll;
            for (int ch = group * (8 / kGroups); ch < (group + 1) * (8 / kGroups); ++ch) {
                uint32_t v[32];
                tmem_ld32(tacc + ch * 32, v);
                tmem_ld_wait();
                uint4* dst = reinterpret_cast<uint4*>(part + ch * 32);
#pragma unroll
                for (int q = 0; q < 8; ++q) dst[q] = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(c.acce + 8u * abuf, 0));
        if (++abuf == 2) {
            abuf = 0;
            aphase ^= 1u;
        }
        if (t.tail >= 0) {
            __threadfence();
            pair_epi_bar<EPI>();
            if (threadIdx.x == kFirst * 32) {
                int* ctr = a.tail_ctr + t.tail * 2 + rank;
                const int old = atomicAdd(ctr, 1);
                const int last = old == a.tail_splits - 1;
                if (last) *ctr = 0;
                *c.fin_flag = last;
            }
            pair_epi_bar<EPI>();
            if (*c.fin_flag) {
                __threadfence();
                const long long split_stride = 2ll * kBM * 256;
                PartialSrc src{part - static_cast<long long>(t.ks) * split_stride + gcol0, split_stride,
                               a.tail_splits};
                epilogue_tile<NACC, EPI, PartialSrc, kPrefetch>(o, row, t.nb * P.tile_n + gcol0, gcols, src, stg, bn,
                                                                ts);
            }
        }
    }
    if (ts != nullptr) ts->drain();
}

// Per-warpgroup register budgets (all four warps of a warpgroup execute the
// same instruction).  .dec gives registers back to the block's pool; .inc
// waits until the pool holds enough.
template <int N>
__device__ __forceinline__ void regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

template <bool B_MN, int EPI, int QF = QF_NONE>
__global__ void __launch_bounds__(pair_threads<EPI, QF != QF_NONE>(), 1)
    umma2_gemm_kernel(const __grid_constant__ PairArgs args) {
    constexpr bool Q4 = QF != QF_NONE;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t ctl = base + args.stages * pair_stage_bytes<QF>();
    uint8_t* ctl_ptr = smem_raw + (ctl - raw);

    const SmemCtl c = make_ctl(ctl, ctl_ptr, args.wait_limit);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    // Tensor maps are launch parameters: prefetch them under the previous
    // kernel's tail (programmatic dependent launch).
    if (warp == 0 && lane < args.nmaps) tma_prefetch_desc(&args.maps[lane]);
    if (warp == 0 && lane == 0) {
        for (int s = 0; s < args.stages; ++s) {
            // int4: the leader's arrive.expect_tx plus one arrival per dequant warp of both CTAs
            mbar_init(c.full + 8u * s, Q4 ? 1 + 2 * kQ4Warps : 1);
            mbar_init(c.empty + 8u * s, 1);
            if (Q4) mbar_init(c.rawf + 8u * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(c.accf + 8u * b, 1);
            mbar_init(c.acce + 8u * b, 2 * pair_epi_warps<EPI>());  // every epilogue warp of both CTAs
        }
        mbar_init(c.drain, 1);
        mbar_init(c.never, 1);
        *c.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(c.tmem_slot, kPairTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(ctl_ptr + (c.tmem_slot - ctl));
#if LMLP_PDL
    // Everything above touched only this CTA's own resources; from here on
    // the kernel reads what the previous launch wrote.
    grid_dependency_wait();
    grid_launch_dependents();
#endif

    static_assert(!Q4 || pair_epi_warps<EPI>() == 4, "an int4 launch runs one epilogue warpgroup");
    constexpr int kFirst = pair_epi_first<Q4>();
    auto producer_role = [&]() {
        if (lane == 0) {
            // The leader waits for both CTAs' loads (they count on its full
            // barriers); the other CTA cannot leave before it, since the
            // cluster barrier below holds it until the leader arrives.
            const long long issued = pair_producer<B_MN, QF>(args, base, rank, leader, c);
            if (leader) drain_loads(c.full, args.stages, issued, c.wait_limit);
            if (Q4) drain_loads(c.rawf, args.stages, issued, c.wait_limit);  // this CTA's code loads
        }
        __syncwarp();
    };
    auto mma_role = [&]() {
        if (lane == 0 && leader) {
            pair_mma<B_MN, QF>(args, base, tmem_base, c);
            umma_commit_pair(c.drain, 1);
            const long long t0 = clock64();
            while (!mbar_try_wait(c.drain, 0)) {
                if (clock64() - t0 > c.wait_limit) break;
            }
        }
        __syncwarp();
    };
    if constexpr (Q4) {
        // each warpgroup's role runs inside the branch that sets its register
        // budget, so that the compiler allocates for it accordingly
        if (warp < 4) {
            regs_dec<kQ4RegsCtl>();
            if (warp == 0) producer_role();
            else if (warp == 1) mma_role();
            // warps 2 and 3: idle
        } else if (warp < 8) {
            regs_inc<kQ4RegsEpi>();
            pair_epilogue<EPI, kFirst>(args, tmem_base, rank, c);
        } else {
            regs_dec<kQ4RegsDq>();
            const int dq = static_cast<int>(threadIdx.x) - 8 * 32;  // 0 .. 255
            pair_dequant<B_MN, QF>(args, base, c, dq >> 7, dq & 127);
        }
    } else {
        if (warp == 0) producer_role();
        else if (warp == 1) mma_role();
        else pair_epilogue<EPI, kFirst>(args, tmem_base, rank, c);
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, kPairTmemCols);
}

}  // namespace lmlp
