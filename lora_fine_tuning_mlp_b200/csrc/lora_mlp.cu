// C ABI of the fused LoRA + SwiGLU MLP (include/lora_mlp.h): argument
// validation, workspace layout, tensor-map encoding and the stream-ordered
// launch sequence of forward and backward.
//
// Forward  (s = alpha / r; S_x denotes an s-scaled rank-r projection):
//   F0  [S_g | S_u] = s X [Ag; Au]^T          tcgen05, two accumulators, split-K
//   F1  G = X Wg^T + S_g Bg^T, U likewise;   tcgen05, two accumulators,
//       epilogue writes g, u and h = silu(g) u (bf16)
//   F2  S_d = s h Ad^T                        tcgen05, split-K
//   F3  out = h Wd^T + S_d Bd^T               tcgen05
// Backward:
//   B0  T_d = s dOut Bd;  dBd = dOut^T S_d    tcgen05 (token-reduction for dBd)
//   B1  dH = dOut Wd + T_d Ad; epilogue recomputes sigmoid/silu from g, u and
//       writes dg, du (and h for B2)          tcgen05, MN-major weights
//   B2  dAd = T_d^T h                          tcgen05 token-reduction
//   B3  T_g = s dg Bg, T_u = s du Bu;  dBg = dg^T S_g, dBu = du^T S_u
//   B4  dX = dg Wg + du Wu + T_g Ag + T_u Au   tcgen05, K = 2 d_ff + 2r
//   B5  dAg = T_g^T X, dAu = T_u^T X           tcgen05 token-reduction
// (The chain rule of the LoRA SwiGLU MLP; "Unsloth 深度分析报告", 创新之处:
// hand-derived fused LoRA MLP backward that stores no autograd intermediates.)
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "lora_mlp.h"
#include "lora_linear.h"
#include "lora_rmsnorm.h"
#include "lora_ce.h"
#include "aux_kernels.cuh"
#include "cross_entropy.cuh"
#include "rmsnorm.cuh"
#include "ptx.cuh"
#include "umma_gemm.cuh"
#include "umma2_gemm.cuh"
#include "lowrank_dual.cuh"

using namespace lmlp;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kTargetCtas = 148;  // split-K sizing target (B200 SM count); a layout constant
constexpr int kMaxSplits = 32;
constexpr size_t kAlign = 256;
constexpr uint32_t kSmemLimit = 232448;  // max dynamic shared memory per block on sm_100
// Compile-time tuning knobs (defaults are the measured best on B200).
#ifndef LMLP_PAIR_GROUP_M
#define LMLP_PAIR_GROUP_M 16  // CTA-pair raster: tiles walk down groups of this many 256-row M tiles
#endif
#ifndef LMLP_TAIL_SPLIT
#define LMLP_TAIL_SPLIT 1  // split the last partial round of CTA-pair tiles in two K halves
#endif
// The tail split pays off for launches with a plain bf16 store epilogue (the
// down and dX GEMMs: -55 us and -15 us per step on the Llama-3-8B shapes,
// measured interleaved) but not for the SwiGLU epilogues (+31 us, +39 us;
// the gate/up GEMM again +2 % and +3 % on the Llama-3-8B and TinyLlama-1.1B
// shapes with its TMA-store epilogue, in two or four K ranges), so those
// launches run without it.
#ifndef LMLP_TAIL_SPLIT_SWIGLU
#define LMLP_TAIL_SPLIT_SWIGLU 0
#endif
constexpr int kTailMaxUnits = 74;        // tail-split units of one CTA-pair launch (one per cluster)
constexpr size_t kTailPartFloats = static_cast<size_t>(kTailMaxUnits) * 2 * kBM * 256;

std::atomic<int64_t> g_launches{0};
std::atomic<int> g_force_timeout{0};
std::atomic<long long> g_wait_limit{kWaitLimitCycles};

// ----------------------------------------------------------------------------- device info
struct DevInfo {
    int checked;
    int ok;
    int sms;
    void* status_addr;
};
DevInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int device_info(DevInfo* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LORA_MLP_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DevInfo& di = g_dev[dev];
    if (!di.checked) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return LORA_MLP_ERR_CUDA;
        di.ok = (major == 10 && minor == 0);
        di.sms = sms;
        void* addr = nullptr;
        if (di.ok && cudaGetSymbolAddress(&addr, g_lmlp_status) != cudaSuccess) return LORA_MLP_ERR_CUDA;
        di.status_addr = addr;
        di.checked = 1;
    }
    *out = di;
    return di.ok ? LORA_MLP_OK : LORA_MLP_ERR_UNSUPPORTED_ARCH;
}

// ----------------------------------------------------------------------------- timing
struct TimingRec {
    const char* name;
    cudaEvent_t beg, end;
};
std::mutex g_time_mu;
std::atomic<int> g_timing{0};
std::vector<TimingRec> g_recs;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t pool_event() {
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

struct LaunchScope {
    const char* name;
    cudaStream_t st;
    cudaEvent_t beg = nullptr, end = nullptr;
    LaunchScope(const char* n, cudaStream_t s) : name(n), st(s) {
        g_launches.fetch_add(1, std::memory_order_relaxed);
        if (g_timing.load(std::memory_order_relaxed)) {
            std::lock_guard<std::mutex> lk(g_time_mu);
            beg = pool_event();
            end = pool_event();
            cudaEventRecord(beg, st);
        }
    }
    ~LaunchScope() {
        if (beg != nullptr) {
            cudaEventRecord(end, st);
            std::lock_guard<std::mutex> lk(g_time_mu);
            g_recs.push_back({name, beg, end});
        }
    }
};

int last_launch_error() { return cudaGetLastError() == cudaSuccess ? LORA_MLP_OK : LORA_MLP_ERR_CUDA; }

// ----------------------------------------------------------------------------- tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Tiled, 128-byte-swizzled TMA descriptor of a bf16 matrix [outer, inner]
// (row stride ld elements) with a box_inner x box_outer box.  Out-of-range
// elements of a box read as zero.
bool encode_map(CUtensorMap* m, const void* ptr, int64_t inner, int64_t outer, int64_t ld, uint32_t box_inner,
                uint32_t box_outer, CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tiled, unswizzled TMA descriptor of a byte matrix [outer, inner] (row
// stride ld bytes, a multiple of 16) with a box_inner x box_outer box: the
// codes of an int4 or FP8 weight.  Out-of-range bytes read as zero.
// (elem = 2 or 4: a 16- or 32-bit matrix, the transposed block scales; ld
// then in elements.)
bool encode_map_u8(CUtensorMap* m, const void* ptr, int64_t inner, int64_t outer, int64_t ld, uint32_t box_inner,
                   uint32_t box_outer, int elem = 1, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_NONE) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * static_cast<cuuint64_t>(elem)};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t es[2] = {1, 1};
    const CUtensorMapDataType ty = elem == 4   ? CU_TENSOR_MAP_DATA_TYPE_UINT32
                                   : elem == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16
                                               : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    return fn(m, ty, 2, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }
int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

// Builds the argument block of one GEMM launch.
struct GemmBuilder {
    GemmArgs a;
    int nmaps = 0;
    bool ok = true;
    int units = 0;

    explicit GemmBuilder(int bn) {
        std::memset(&a, 0, sizeof(a));
        a.bn = bn;
        a.group_m = 16;
    }
    // bf16 matrix [outer, inner] with row stride ld elements; box inner x outer.
    int map(const void* ptr, int64_t inner, int64_t outer, int64_t ld, uint32_t box_inner, uint32_t box_outer) {
        if (nmaps >= kMaxMaps) {
            ok = false;
            return 0;
        }
        if (!encode_map(&a.maps[nmaps], ptr, inner, outer, ld, box_inner, box_outer)) ok = false;
        return nmaps++;
    }
    // A operand, K-major: matrix [rows, K] (K contiguous).
    int a_k(const void* p, int64_t rows, int64_t K, int64_t ld) { return map(p, K, rows, ld, kBK, kBM); }
    // A operand, MN-major: matrix [K, M] (M contiguous), read as A[m, k].
    int a_mn(const void* p, int64_t K, int64_t M, int64_t ld) { return map(p, M, K, ld, 64, kBK); }
    // B operand, K-major: matrix [Nn, K].
    int b_k(const void* p, int64_t Nn, int64_t K, int64_t ld) {
        return map(p, K, Nn, ld, kBK, static_cast<uint32_t>(a.bn));
    }
    // B operand, MN-major: matrix [K, Nn] (Nn contiguous), read as B[n, k]; needs bn % 64 == 0.
    int b_mn(const void* p, int64_t K, int64_t Nn, int64_t ld) {
        if (a.bn % 64) ok = false;
        return map(p, Nn, K, ld, 64, kBK);
    }
    Prob* prob(int64_t M, int64_t N, int splits, bool a_mn = false, bool b_mn = false) {
        if (a.nprobs >= kMaxProbs) {
            ok = false;
            return &a.prob[0];
        }
        Prob& p = a.prob[a.nprobs++];
        p.M = static_cast<int>(M);
        p.N = static_cast<int>(N);
        p.tiles_m = ceil_div(M, kBM);
        p.tiles_n = ceil_div(N, a.bn);
        p.splits = splits;
        p.a_mn = a_mn ? 1 : 0;
        p.b_mn = b_mn ? 1 : 0;
        return &p;
    }
    void seg(Prob* p, int amap, int b0, int b1, int64_t k_len) {
        if (p->nsegs >= kMaxSegs) {
            ok = false;
            return;
        }
        Seg& s = p->seg[p->nsegs++];
        s.a_map = amap;
        s.b_map[0] = b0;
        s.b_map[1] = b1;
        s.k_len = static_cast<int>(k_len);
        s.kblocks = ceil_div(k_len, kBK);
        p->nkb += s.kblocks;
    }
    // Finalise problem p in-kernel (see Prob): scale, bf16 row-major and/or transposed outputs.
    void fin(Prob* p, float scale, int fin_cols, void* rm, long long ld_rm, void* tr0, void* tr1, long long ld_tr,
             int tr_split) {
        p->scale = scale;
        p->fin_cols = fin_cols;
        p->rm = rm;
        p->ld_rm = ld_rm;
        p->tr0 = tr0;
        p->tr1 = tr1;
        p->ld_tr = ld_tr;
        p->tr_split = tr_split;
        p->counters = reinterpret_cast<int*>(1);  // placeholder: assigned in finish()
    }
    // Processing order by feature band: unit u of problem p gets the key
    // feat_of(p, tile, kb0, kb1) (the feature coordinate of the data it reads);
    // units are taken in increasing key order (ties: launch order).  Called
    // after finish().  Only for launches whose problems all have tiles_n == 1.
    template <class KeyFn>
    void order_units(KeyFn feat_of) {
        if (units > kMaxPerm || units > 65535) return;
        std::vector<std::pair<long long, int>> key(static_cast<size_t>(units));
        for (int i = 0; i < a.nprobs; ++i) {
            const Prob& p = a.prob[i];
            if (p.tiles_n != 1) return;
            const int n = p.tiles_m * p.splits;
            for (int lu = 0; lu < n; ++lu) {
                const int tile = lu / p.splits, ks = lu - tile * p.splits;
                const int kb0 = static_cast<int>((static_cast<long long>(ks) * p.nkb) / p.splits);
                const int kb1 = static_cast<int>((static_cast<long long>(ks + 1) * p.nkb) / p.splits);
                key[static_cast<size_t>(p.unit0 + lu)] = {feat_of(i, tile, kb0, kb1), p.unit0 + lu};
            }
        }
        std::stable_sort(key.begin(), key.end(),
                         [](const std::pair<long long, int>& x, const std::pair<long long, int>& y) {
                             return x.first < y.first;
                         });
        for (int i = 0; i < units; ++i) a.perm[i] = static_cast<uint16_t>(key[static_cast<size_t>(i)].second);
        a.nperm = units;
    }
    void finish(int* counters) {
        int u = 0, c = 0;
        for (int i = 0; i < a.nprobs; ++i) {
            Prob& p = a.prob[i];
            if (p.splits > p.nkb) p.splits = p.nkb;
            if (p.splits < 1) p.splits = 1;
            p.unit0 = u;
            u += p.tiles_m * p.tiles_n * p.splits;
            if (p.counters != nullptr) {
                if (counters == nullptr || p.tiles_n != 1) ok = false;
                p.counters = counters + c;
                c += p.tiles_m * p.tiles_n;
            }
        }
        a.total_units = u;
        units = u;
    }
};

template <int NACC, int EPI>
int launch_gemm(GemmBuilder& b, int sms, cudaStream_t st, const char* name, int* counters = nullptr) {
    b.finish(counters);
    if (!b.ok) return LORA_MLP_ERR_CUDA;
    GemmArgs& a = b.a;
    a.nmaps = b.nmaps;
    a.b_bytes = static_cast<uint32_t>(a.bn * 128);  // K-major: bn rows x 128 B; MN-major: bn/64 chunks x 8 KB
    const uint32_t stage_bytes = kATileBytes + NACC * a.b_bytes;
    // A launch with more units than SMs runs two CTAs per SM, each with half
    // the shared memory: a CTA's single TMA-issuing thread, not the stage
    // count, limits how fast these HBM-bound products stream (measured on the
    // adapter-gradient launch of the Llama-3-8B shapes: 164 -> 107 us).
    // Launches with at most one unit per SM keep one CTA and the deeper
    // pipeline, which measured faster for them.
    // Two CTAs also need their accumulators to fit the SM's 512 TMEM columns
    // together and at least three stages each.
    const uint32_t budget1 = kSmemLimit - 1024 - gemm_ctl_bytes();
    const uint32_t budgetN = kSmemLimit / LMLP_MAX_CPS - 2048 - gemm_ctl_bytes();
    const int cps = (b.units > sms && gemm_tmem_cols(NACC, a.bn) <= 512 / LMLP_MAX_CPS &&
                     budgetN / stage_bytes >= 3) ? LMLP_MAX_CPS : 1;
    int stages = static_cast<int>((cps > 1 ? budgetN : budget1) / stage_bytes);
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 2) return LORA_MLP_ERR_UNSUPPORTED_SHAPE;
    a.stages = stages;
    const size_t smem = 1024 + static_cast<size_t>(stages) * stage_bytes + gemm_ctl_bytes();
    auto kern = umma_gemm_kernel<NACC, EPI>;
    static bool attr_set[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) != cudaSuccess)
            return LORA_MLP_ERR_CUDA;
        attr_set[dev] = true;
    }
    a.wait_limit = g_wait_limit.load();
    a.force_timeout = g_force_timeout.load();
    const int ctas = sms * cps;
    const int grid = b.units < ctas ? b.units : ctas;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = LMLP_PDL ? 1 : 0;
    cudaError_t err;
    {
        LaunchScope scope(name, st);
        err = cudaLaunchKernelEx(&cfg, kern, a);
    }
    if (err != cudaSuccess) return LORA_MLP_ERR_CUDA;
    return last_launch_error();
}

// Builds the argument block of one CTA-pair GEMM launch (256-row tiles).
struct PairBuilder {
    PairArgs a;
    int nmaps = 0;
    bool ok = true;

    PairBuilder(int64_t M, int64_t N, int tile_n) {
        std::memset(&a, 0, sizeof(a));
        a.group_m = LMLP_PAIR_GROUP_M;
        a.prob.M = static_cast<int>(M);
        a.prob.N = static_cast<int>(N);
        a.prob.tile_n = tile_n;
        a.prob.tiles_m = ceil_div(M, kPairBM);
        a.prob.tiles_n = ceil_div(N, tile_n);
    }
    int map(const void* ptr, int64_t inner, int64_t outer, int64_t ld, uint32_t bi, uint32_t bo) {
        if (nmaps >= kMaxMaps) {
            ok = false;
            return 0;
        }
        if (!encode_map(&a.maps[nmaps], ptr, inner, outer, ld, bi, bo)) ok = false;
        return nmaps++;
    }
    int a_k(const void* p, int64_t rows, int64_t K, int64_t ld) { return map(p, K, rows, ld, kBK, kBM); }
    int b_k(const void* p, int64_t Nn, int64_t K, int64_t ld) { return map(p, K, Nn, ld, kBK, kPairHalfN); }
    // bf16 output [M, N] (row stride prob.ld) as 32 x 32 blocks in the 64-byte
    // swizzle, for the epilogue's TMA stores.
    int out_map(const void* p) {
        if (nmaps >= kMaxMaps) {
            ok = false;
            return 0;
        }
        if (!encode_map(&a.maps[nmaps], p, a.prob.N, a.prob.M, a.prob.ld, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
            ok = false;
        return nmaps++;
    }
    int b_mn(const void* p, int64_t K, int64_t Nn, int64_t ld) { return map(p, Nn, K, ld, 64, kBK); }
    // The codes of a quantised weight [rows, cols]: int4 (uint8 [rows,
    // cols/2], 32-byte line rows) or FP8 (uint8 [rows, cols], 64-byte line
    // rows in TMA's 64-byte swizzle), read K-major (K = cols, 128 rows per
    // box) or MN-major (K = rows, 64 rows per box).
    int q_map(const void* codes, int64_t rows, int64_t cols, bool mn, int qf) {
        if (nmaps >= kMaxMaps) {
            ok = false;
            return 0;
        }
        const bool f8 = qf == QF_FP8;
        const int64_t inner = f8 ? cols : cols / 2;
        if (!encode_map_u8(&a.maps[nmaps], codes, inner, rows, inner, f8 ? 64 : 32, mn ? 64 : kPairHalfN, 1,
                           f8 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE))
            ok = false;
        return nmaps++;
    }
    // The transposed scales [cols/64, rows] of a weight [rows, cols]: one
    // box holds the scales of 128 consecutive rows (K-major B) or 64 (MN-major).
    int s_map(const void* st, int64_t rows, int64_t cols, bool mn, int qf) {
        if (nmaps >= kMaxMaps) {
            ok = false;
            return 0;
        }
        if (!encode_map_u8(&a.maps[nmaps], st, rows, cols / 64, rows, mn ? 64 : kPairHalfN, 1, qf == QF_FP8 ? 4 : 2))
            ok = false;
        return nmaps++;
    }
    // Marks segment `sg` as reading int4 B: code and scale maps of halves 0 / 1.
    void quant(int sg, int q0, int q1, int s0, int s1) {
        PairSeg& S = a.prob.seg[sg];
        S.q4 = 1;
        S.qmap[0] = q0;
        S.qmap[1] = q1;
        S.smap[0] = s0;
        S.smap[1] = s1;
    }
    void seg(int amap, int b0, int b1, int row0, int row1, int k0, int k1, int64_t k_len) {
        PairProb& p = a.prob;
        if (p.nsegs >= kMaxSegs) {
            ok = false;
            return;
        }
        PairSeg& s = p.seg[p.nsegs++];
        s.a_map = amap;
        s.b_map[0] = b0;
        s.b_map[1] = b1;
        s.b_row[0] = row0;
        s.b_row[1] = row1;
        s.b_k[0] = k0;
        s.b_k[1] = k1;
        s.k_len = static_cast<int>(k_len);
        s.kblocks = ceil_div(k_len, kBK);
        p.nkb += s.kblocks;
    }
};

// Tail split of a CTA-pair launch: with `clusters` clusters and `tiles`
// tiles, the tiles of the last, partial round are each cut into two K
// halves when enough clusters are free, so that round takes half a tile's
// time.  More pieces would shorten it further but the CTA that finishes a
// tile then has to add more partials, which costs more than it saves.
// Returns the number of pieces (1 = no split).
int pair_tail_splits(int tiles, int clusters, int nkb) {
    if (clusters < 1 || tiles < 1 || nkb < 4) return 1;
    const int tail = tiles % clusters;
    if (tail == 0 || 2 * tail > clusters) return 1;
    return 2;
}

template <bool B_MN, int EPI, int QF = QF_NONE>
int launch_pair(PairBuilder& b, int sms, cudaStream_t st, const char* name, float* tail_part, int* tail_ctr) {
    constexpr bool Q4 = QF != QF_NONE;
    if constexpr (pair_tma_store<EPI>()) {
        b.a.prob.omap[0] = b.out_map(b.a.prob.out0);
        if (EPI != EPI_BF16) {
            b.a.prob.omap[1] = b.out_map(b.a.prob.out1);
            b.a.prob.omap[2] = b.out_map(b.a.prob.out2);
        }
    }
    if (!b.ok) return LORA_MLP_ERR_CUDA;
    PairArgs& a = b.a;
    a.nmaps = b.nmaps;
    const int tiles = a.prob.tiles_m * a.prob.tiles_n;
    a.total_units = tiles;
    a.full_units = tiles;
    a.tail_splits = 1;
    a.tail_part = tail_part;
    a.tail_ctr = tail_ctr;
    // (512-byte alignment) epilogue store staging per warp, then the dH epilogue's g/u rings
    const uint32_t staging = 512 + pair_epi_warps<EPI>() * pair_stage_warp_bytes<EPI>() + pair_ring_bytes<EPI>();
    constexpr uint32_t kSB = pair_stage_bytes<QF>();
    const uint32_t budget = kSmemLimit - 1024 - gemm_ctl_bytes() - staging;
    int stages = static_cast<int>(budget / kSB);
    if (stages > kPairMaxStages) stages = kPairMaxStages;
    if (stages < 2) return LORA_MLP_ERR_UNSUPPORTED_SHAPE;
    a.stages = stages;
    const size_t smem = 1024 + static_cast<size_t>(stages) * kSB + gemm_ctl_bytes() + staging;
    auto kern = umma2_gemm_kernel<B_MN, EPI, QF>;
    static int max_clusters[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(pair_threads<EPI, Q4>(), 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (max_clusters[dev] == 0) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) != cudaSuccess)
            return LORA_MLP_ERR_CUDA;
        cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) n = sms / 2;
        max_clusters[dev] = n;
    }
    const int avail = std::min(max_clusters[dev], kTailMaxUnits);
    const bool tail_ok = EPI == EPI_BF16 ? LMLP_TAIL_SPLIT != 0 : LMLP_TAIL_SPLIT_SWIGLU != 0;
    if (tail_ok && tail_part != nullptr && tail_ctr != nullptr) {
        const int S = pair_tail_splits(tiles, avail, a.prob.nkb);
        if (S > 1) {
            const int tail = tiles % avail;
            a.full_units = tiles - tail;
            a.tail_splits = S;
            a.total_units = a.full_units + tail * S;
        }
    }
    a.wait_limit = g_wait_limit.load();
    a.force_timeout = g_force_timeout.load();
    int clusters = a.total_units < max_clusters[dev] ? a.total_units : max_clusters[dev];
    cfg.gridDim = dim3(2 * clusters, 1, 1);
    cfg.numAttrs = LMLP_PDL ? 2 : 1;
    cudaError_t err;
    {
        LaunchScope scope(name, st);
        err = cudaLaunchKernelEx(&cfg, kern, a);
    }
    if (err != cudaSuccess) return LORA_MLP_ERR_CUDA;
    return last_launch_error();
}

// launch_pair with the weight format chosen at run time.
template <bool B_MN, int EPI>
int launch_pair_q(PairBuilder& b, int qf, int sms, cudaStream_t st, const char* name, float* tail_part,
                  int* tail_ctr) {
    if (qf == QF_INT4) return launch_pair<B_MN, EPI, QF_INT4>(b, sms, st, name, tail_part, tail_ctr);
    if (qf == QF_FP8) return launch_pair<B_MN, EPI, QF_FP8>(b, sms, st, name, tail_part, tail_ctr);
    return launch_pair<B_MN, EPI, QF_NONE>(b, sms, st, name, tail_part, tail_ctr);
}

int launch_dequant(const void* packed, const void* scales, int64_t rows, int64_t cols, void* w, int sms,
                   cudaStream_t st) {
    const long long nlines = rows * (cols / 64);  // one scale and 64 elements per line
    long long blocks = (nlines + kDqThreads - 1) / kDqThreads;
    const long long cap = static_cast<long long>(sms) * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    {
        LaunchScope scope("dequant_int4", st);
        dequant_int4_kernel<<<static_cast<int>(blocks), kDqThreads, 0, st>>>(
            static_cast<const uint4*>(packed), static_cast<const __half*>(scales), nlines, static_cast<uint4*>(w));
    }
    return last_launch_error();
}

int launch_dequant_fp8(const void* codes, const void* scales, int64_t rows, int64_t cols, void* w, int sms,
                       cudaStream_t st) {
    const long long nlines = rows * (cols / 64);
    long long blocks = (nlines + kDqThreads - 1) / kDqThreads;
    const long long cap = static_cast<long long>(sms) * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    {
        LaunchScope scope("dequant_fp8", st);
        dequant_fp8_kernel<<<static_cast<int>(blocks), kDqThreads, 0, st>>>(
            static_cast<const uint4*>(codes), static_cast<const float*>(scales), nlines, static_cast<uint4*>(w));
    }
    return last_launch_error();
}

// Transposes up to three block-scale matrices [rows, cols/64] into
// [cols/64, rows] (scale_transpose_kernel), one launch; elements of 2 bytes
// (int4's fp16 scales) or 4 (FP8's fp32 scales).
template <class T>
int launch_scale_t_typed(int n, const void* const* src, void* const* dst, const int64_t* rows,
                         const int64_t* cols, cudaStream_t st) {
    ScaleT<T> a{};
    unsigned gx = 1;
    for (int i = 0; i < n; ++i) {
        a.src[i] = static_cast<const T*>(src[i]);
        a.dst[i] = static_cast<T*>(dst[i]);
        a.rows[i] = static_cast<int>(rows[i]);
        a.nb[i] = static_cast<int>(cols[i] / 64);
        gx = std::max(gx, static_cast<unsigned>((rows[i] + 31) / 32));
    }
    {
        LaunchScope scope("scales_t", st);
        scale_transpose_kernel<T><<<dim3(gx, n), 256, 0, st>>>(a);
    }
    return last_launch_error();
}
int launch_scale_t(int qf, int n, const void* const* src, void* const* dst, const int64_t* rows,
                   const int64_t* cols, cudaStream_t st) {
    return qf == QF_FP8 ? launch_scale_t_typed<unsigned int>(n, src, dst, rows, cols, st)
                        : launch_scale_t_typed<unsigned short>(n, src, dst, rows, cols, st);
}

// Bg, Bu [dff, r] -> Bg^T, Bu^T [r, dff] (the K-major B operands of the
// single-pass adapter-gradient launch), one launch.
int launch_adapter_t(const void* Bg, const void* Bu, void* BgT, void* BuT, int64_t dff, int64_t r, cudaStream_t st) {
    ScaleT<unsigned short> a{};
    a.src[0] = static_cast<const unsigned short*>(Bg);
    a.src[1] = static_cast<const unsigned short*>(Bu);
    a.dst[0] = static_cast<unsigned short*>(BgT);
    a.dst[1] = static_cast<unsigned short*>(BuT);
    a.rows[0] = a.rows[1] = static_cast<int>(dff);
    a.nb[0] = a.nb[1] = static_cast<int>(r);
    {
        LaunchScope scope("B_mid_adapter_t", st);
        scale_transpose_kernel<unsigned short><<<dim3(static_cast<unsigned>((dff + 31) / 32), 2), 256, 0, st>>>(a);
    }
    return last_launch_error();
}

// ----------------------------------------------------------------------------- layout
// Split-K factors for the skinny problems of one launch.  All problems of a
// launch are cut into units of about T K blocks (problem p gets
// ceil(nkb_p / T) splits); T is chosen to minimise the estimated makespan of
// the persistent grid, rounds(T) * (T + kUnitCost), where a round is one
// unit per SM and kUnitCost (in K blocks) stands for a unit's epilogue and
// split-K bookkeeping.  Depends only on the shape (a fixed 148-CTA grid), so
// workspace sizes do not depend on the device.
#ifndef LMLP_UNIT_COST
#define LMLP_UNIT_COST 6
#endif
constexpr int64_t kUnitCost = LMLP_UNIT_COST;

struct SkinnySpec {
    int64_t M;      // output rows
    int64_t ncols;  // partial columns (the valid N of the problem)
    int64_t nkb;    // K blocks
};

void plan_splits(const SkinnySpec* sp, int n, int* out, int slots = kTargetCtas) {
    int64_t max_kb = 1;
    for (int i = 0; i < n; ++i) max_kb = std::max(max_kb, sp[i].nkb);
    double best = 1e300;
    int64_t best_T = max_kb;
    for (int64_t T = 4; T <= max_kb + 4; T += (T < 64 ? 4 : 16)) {
        int64_t units = 0, longest = 0;
        for (int i = 0; i < n; ++i) {
            const int64_t s = std::min<int64_t>(std::max<int64_t>((sp[i].nkb + T - 1) / T, 1), kMaxSplits);
            units += ceil_div(sp[i].M, kBM) * s;
            longest = std::max(longest, (sp[i].nkb + s - 1) / s);
        }
        const int64_t rounds = (units + slots - 1) / slots;
        const double cost = static_cast<double>(rounds) * static_cast<double>(longest + kUnitCost);
        if (cost < best - 1e-9) {
            best = cost;
            best_T = T;
        }
    }
    for (int i = 0; i < n; ++i) {
        const int64_t s = std::min<int64_t>(std::max<int64_t>((sp[i].nkb + best_T - 1) / best_T, 1), kMaxSplits);
        out[i] = static_cast<int>(std::min<int64_t>(s, std::max<int64_t>(sp[i].nkb, 1)));
    }
}

int64_t launch_tiles(const SkinnySpec* sp, int n) {
    int64_t t = 0;
    for (int i = 0; i < n; ++i) t += ceil_div(sp[i].M, kBM);
    return t;
}

// The skinny launches of one forward + backward, in launch order.
enum { SK_F0, SK_F2, SK_B0, SK_BMID, SK_B5, SK_COUNT };
constexpr int kSkinnyProbs[SK_COUNT] = {1, 1, 2, 5, 1};
// Units per round that plan_splits sizes each launch for: one per SM, or two
// for the row projections that then run two CTAs per SM (launch_gemm), which
// measured faster for them on the Llama-3-8B shapes (F2 50 -> 44 us, B0
// 37 -> 29 us) and slower for F0 and B5, whose finalising CTAs write the
// transposed tiles.
constexpr int kSkinnySlots[SK_COUNT] = {kTargetCtas, 2 * kTargetCtas, 2 * kTargetCtas, kTargetCtas, kTargetCtas};

struct Plan {
    int64_t N, d, d_ff, r, ldN;
    float s;
    int qf;  // frozen-weight format: QF_NONE (bf16), QF_INT4, QF_FP8
    int bn_r, bn_r64, bn_2r;
    SkinnySpec spec[SK_COUNT][kMaxProbs];
    int splits[SK_COUNT][kMaxProbs];
    size_t part_off[SK_COUNT][kMaxProbs];  // float offset of each problem's partials
    // forward workspace
    size_t f_h, f_sgu, f_sd, f_part, f_ctr, f_tail, f_st[3], f_total;  // f_st: block scales, transposed
    // backward workspace
    size_t b_dg, b_du, b_h, b_td, b_tdT, b_tgu, b_tguT, b_part, b_ctr, b_tail, b_st[3], b_total;
    // single-pass adapter-gradient launch (ranks <= 32): its partition and
    // buffers (Bg^T | Bu^T, the dB and T partial sums)
    bool dual;
    int dual_ntb, dual_ntr, dual_fchunks;
    size_t b_bT, b_pdb, b_pt;
    size_t ctr_bytes;  // per-tile split-K counters (zeroed at the start of each call)
    // saved
    size_t s_sgT, s_suT, s_sdT, s_total;
};

struct Carver {
    size_t off = 0;
    size_t take(size_t bytes) {
        const size_t o = off;
        off += (bytes + kAlign - 1) / kAlign * kAlign;
        return o;
    }
};

// Partition of the single-pass adapter-gradient launch (lowrank_dual.cuh):
// n_tb token blocks per token range (at most kDualMaxTb, for TMEM), as many
// feature ranges per token range as fill 148 SMs.  Chosen by an estimate of
// its time: the busiest CTA's bytes at one SM's share of HBM, or all of them
// at HBM's rate, whichever is longer, plus the partial sums written and read
// back.  Depends only on the shape.
#ifndef LMLP_DUAL
#define LMLP_DUAL 1  // 0: the adapter-gradient launch as five split-K problems (two reads of dg, du)
#endif
void dual_plan(Plan& p) {
    p.dual = false;
    if (!LMLP_DUAL || p.r > kDualBN) return;
    const int64_t tiles_t = ceil_div(p.N, 128), tiles_f = ceil_div(p.d_ff, 128);
    const double kSmRate = 45e9, kHbmRate = 6.5e12;
    const double tile_bytes = 3.0 * kDualA + 2.0 * kDualBT + 3.0 * kDualBD;  // one (token, feature) block, 3 matrices
    double best = 1e300;
    for (int ntb = 1; ntb <= kDualMaxTb; ++ntb) {
        const int64_t ntr = ceil_div(tiles_t, ntb);
        if (ntr > kTargetCtas) continue;
        const int64_t fch = std::min<int64_t>(tiles_f, kTargetCtas / ntr);
        if (fch < 1) continue;
        const int64_t per_cta = std::min<int64_t>(ntb, tiles_t) * ceil_div(tiles_f, fch);
        const double stream = std::max(per_cta * tile_bytes / kSmRate, tiles_t * tiles_f * tile_bytes / kHbmRate);
        const double partial = 4.0 * (ntr * 3.0 * p.d_ff * p.r + fch * 2.0 * p.N * p.r);
        const double est = stream + 2.0 * partial / kHbmRate;
        if (est < best) {
            best = est;
            p.dual = true;
            p.dual_ntb = ntb;
            p.dual_ntr = static_cast<int>(ntr);
            p.dual_fchunks = static_cast<int>(fch);
        }
    }
}

Plan make_plan(const lora_mlp_shape& sh) {
    Plan p{};
    p.N = sh.N;
    p.d = sh.d;
    p.d_ff = sh.d_ff;
    p.r = sh.r;
    p.ldN = round_up(sh.N, 8);
    p.s = static_cast<float>(static_cast<double>(sh.alpha) / static_cast<double>(sh.r));
    p.qf = sh.weight_format == LORA_MLP_WEIGHTS_INT4_B64  ? QF_INT4
           : sh.weight_format == LORA_MLP_WEIGHTS_FP8_B64 ? QF_FP8
                                                           : QF_NONE;
    p.bn_r = static_cast<int>(round_up(sh.r, 32));
    p.bn_r64 = static_cast<int>(round_up(sh.r, 64));
    p.bn_2r = static_cast<int>(round_up(2 * sh.r, 32));
    const int64_t N = p.N, d = p.d, dff = p.d_ff, r = p.r;
    const int64_t kb_d = ceil_div(d, kBK), kb_f = ceil_div(dff, kBK), kb_n = ceil_div(N, kBK);
    // F0: [S_g|S_u] (two accumulators, 2r partial columns); F2: S_d
    p.spec[SK_F0][0] = {N, 2 * r, kb_d};
    p.spec[SK_F2][0] = {N, r, kb_f};
    // B0: T_d (rows = tokens) and dBd (rows = d)
    p.spec[SK_B0][0] = {N, r, kb_d};
    p.spec[SK_B0][1] = {d, r, kb_n};
    // B-mid: T_g, T_u (longest units first), dAd, dBg, dBu
    p.spec[SK_BMID][0] = {N, r, kb_f};
    p.spec[SK_BMID][1] = {N, r, kb_f};
    p.spec[SK_BMID][2] = {dff, r, kb_n};
    p.spec[SK_BMID][3] = {dff, r, kb_n};
    p.spec[SK_BMID][4] = {dff, r, kb_n};
    // B5: [dAg; dAu]^T (2r partial columns)
    p.spec[SK_B5][0] = {d, 2 * r, kb_n};
    size_t part_f = 0, part_b = 0;
    int64_t max_tiles = 0;
    for (int l = 0; l < SK_COUNT; ++l) {
        plan_splits(p.spec[l], kSkinnyProbs[l], p.splits[l], kSkinnySlots[l]);
        size_t off = 0;
        for (int i = 0; i < kSkinnyProbs[l]; ++i) {
            p.part_off[l][i] = off;
            off += static_cast<size_t>(p.splits[l][i]) * p.spec[l][i].M * p.spec[l][i].ncols;
        }
        if (l <= SK_F2) part_f = std::max(part_f, off);
        else part_b = std::max(part_b, off);
        max_tiles = std::max(max_tiles, launch_tiles(p.spec[l], kSkinnyProbs[l]));
    }
    p.ctr_bytes = static_cast<size_t>(std::max<int64_t>(max_tiles, 2 * kTailMaxUnits) + 8) * sizeof(int);

    const size_t bf = 2, f32 = 4;
    const size_t Nz = N, fz = dff, rz = r, ldN = p.ldN;

    Carver f;
    p.f_h = f.take(Nz * fz * bf);
    p.f_sgu = f.take(Nz * 2 * rz * bf);
    p.f_sd = f.take(Nz * rz * bf);
    p.f_part = f.take(part_f * f32);
    p.f_ctr = f.take(p.ctr_bytes);
    p.f_tail = f.take(kTailPartFloats * f32);
    // one weight's block scales (fp16 for int4, fp32 for FP8)
    const size_t stsz = static_cast<size_t>(d) * static_cast<size_t>(dff) / 64 * (p.qf == QF_FP8 ? 4 : 2);
    for (int i = 0; i < 3; ++i) p.f_st[i] = p.qf ? f.take(stsz) : 0;
    p.f_total = f.off;

    Carver b;
    p.b_dg = b.take(Nz * fz * bf);
    p.b_du = b.take(Nz * fz * bf);
    p.b_h = b.take(Nz * fz * bf);
    p.b_td = b.take(Nz * rz * bf);
    p.b_tdT = b.take(rz * ldN * bf);
    p.b_tgu = b.take(Nz * 2 * rz * bf);
    p.b_tguT = b.take(2 * rz * ldN * bf);
    p.b_part = b.take(part_b * f32);
    p.b_ctr = b.take(p.ctr_bytes);
    p.b_tail = b.take(kTailPartFloats * f32);
    for (int i = 0; i < 3; ++i) p.b_st[i] = p.qf ? b.take(stsz) : 0;
    dual_plan(p);
    if (p.dual) {
        p.b_bT = kDualBtMn ? 0 : b.take(2 * rz * fz * bf);
        p.b_pdb = b.take(static_cast<size_t>(p.dual_ntr) * 3 * fz * rz * f32);
        p.b_pt = b.take(static_cast<size_t>(p.dual_fchunks) * Nz * 2 * rz * f32);
    }
    p.b_total = b.off;

    Carver sv;
    p.s_sgT = sv.take(rz * ldN * bf);
    p.s_suT = p.s_sgT + rz * ldN * bf;  // contiguous with S_g^T: [S_g^T; S_u^T] is one [2r, ldN] matrix
    sv.take(rz * ldN * bf);
    p.s_sdT = sv.take(rz * ldN * bf);
    p.s_total = sv.off;
    return p;
}

// ----------------------------------------------------------------------------- validation
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The single-pass adapter-gradient launch and the launch that sums its
// partials (lowrank_dual.cuh).  row_scale: optional factor per token of the
// transposed T outputs.
int launch_dual(const Plan& pl, const void* dg, const void* du, const void* h, const void* BgT, const void* BuT,
                const void* SgT, const void* SuT, const void* TdT, uint8_t* ws, const lora_mlp_grads* grads,
                void* Tgu, void* TguT, const float* row_scale, cudaStream_t st) {
    DualArgs a;
    std::memset(&a, 0, sizeof(a));
    const int64_t N = pl.N, dff = pl.d_ff, r = pl.r, ldN = pl.ldN;
    bool ok = true;
    const void* mats[3] = {dg, du, h};
    for (int m = 0; m < 3; ++m) ok = ok && encode_map(&a.maps[m], mats[m], dff, N, dff, 64, 128);
    if (kDualBtMn) {
        ok = ok && encode_map(&a.maps[3], BgT, r, dff, r, 64, 64);
        ok = ok && encode_map(&a.maps[4], BuT, r, dff, r, 64, 64);
    } else {
        ok = ok && encode_map(&a.maps[3], BgT, dff, r, dff, 64, kDualBN);
        ok = ok && encode_map(&a.maps[4], BuT, dff, r, dff, 64, kDualBN);
    }
    const void* bd[3] = {SgT, SuT, TdT};
    for (int m = 0; m < 3; ++m) ok = ok && encode_map(&a.maps[5 + m], bd[m], N, r, ldN, 64, kDualBN);
    if (!ok) return LORA_MLP_ERR_CUDA;
    a.nmaps = 8;
    a.N = static_cast<int>(N);
    a.dff = static_cast<int>(dff);
    a.r = static_cast<int>(r);
    a.n_tb = pl.dual_ntb;
    a.n_tr = pl.dual_ntr;
    a.fchunks = pl.dual_fchunks;
    a.tiles_t = ceil_div(N, 128);
    a.tiles_f = ceil_div(dff, 128);
    a.part_db = reinterpret_cast<float*>(ws + pl.b_pdb);
    a.part_t = reinterpret_cast<float*>(ws + pl.b_pt);
    a.wait_limit = g_wait_limit.load();
    a.force_timeout = g_force_timeout.load();
    const size_t smem = 1024 + static_cast<size_t>(kDualStages) * kDualStage + gemm_ctl_bytes();
    static bool attr_set[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(dual_lowrank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) !=
            cudaSuccess)
            return LORA_MLP_ERR_CUDA;
        attr_set[dev] = true;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(a.n_tr * a.fchunks), 1, 1);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = LMLP_PDL ? 1 : 0;
    cudaError_t err;
    {
        LaunchScope scope("B_mid_lowrank_grads", st);
        err = cudaLaunchKernelEx(&cfg, dual_lowrank_kernel, a);
    }
    if (err != cudaSuccess || last_launch_error() != LORA_MLP_OK) return LORA_MLP_ERR_CUDA;
    DualFin f{};
    f.part_db = a.part_db;
    f.part_t = a.part_t;
    f.dBg = static_cast<__nv_bfloat16*>(grads->dBg);
    f.dBu = static_cast<__nv_bfloat16*>(grads->dBu);
    f.dAd = static_cast<__nv_bfloat16*>(grads->dAd);
    f.Tgu = static_cast<__nv_bfloat16*>(Tgu);
    f.TguT = static_cast<__nv_bfloat16*>(TguT);
    f.row_scale = row_scale;
    f.ldN = ldN;
    f.N = a.N;
    f.dff = a.dff;
    f.r = a.r;
    f.n_tr = a.n_tr;
    f.fchunks = a.fchunks;
    f.s = pl.s;
    f.db_blocks = ceil_div(3 * dff * (r / 4), kDualFinThreads);
    cfg.gridDim = dim3(static_cast<unsigned>(f.db_blocks + ceil_div(N * (r / 2), kDualFinThreads)), 1, 1);
    cfg.blockDim = dim3(kDualFinThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    {
        LaunchScope scope("B_mid_finalize", st);
        err = cudaLaunchKernelEx(&cfg, dual_finalize_kernel, f);
    }
    if (err != cudaSuccess) return LORA_MLP_ERR_CUDA;
    return last_launch_error();
}

int validate_shape(const lora_mlp_shape* sh) {
    if (sh == nullptr) return LORA_MLP_ERR_INVALID_ARG;
    if (sh->N < 1 || sh->d < 1 || sh->d_ff < 1 || sh->r < 1) return LORA_MLP_ERR_INVALID_ARG;
    if (!std::isfinite(sh->alpha)) return LORA_MLP_ERR_INVALID_ARG;
    if (sh->weight_format != LORA_MLP_WEIGHTS_BF16 && sh->weight_format != LORA_MLP_WEIGHTS_INT4_B64 &&
        sh->weight_format != LORA_MLP_WEIGHTS_FP8_B64)
        return LORA_MLP_ERR_INVALID_ARG;
    if (sh->d % 8 || sh->d_ff % 8 || sh->r % 8) return LORA_MLP_ERR_UNSUPPORTED_SHAPE;
    if (sh->r > 128) return LORA_MLP_ERR_UNSUPPORTED_SHAPE;
    if (sh->weight_format != LORA_MLP_WEIGHTS_BF16 && (sh->d % 64 || sh->d_ff % 64))
        return LORA_MLP_ERR_UNSUPPORTED_SHAPE;
    const int64_t lim = (int64_t{1} << 31) - 1;
    if (sh->N > lim || sh->d > lim || sh->d_ff > lim) return LORA_MLP_ERR_UNSUPPORTED_SHAPE;
    return LORA_MLP_OK;
}

int check_ptrs(std::initializer_list<const void*> ps) {
    for (const void* p : ps) {
        if (p == nullptr) return LORA_MLP_ERR_INVALID_ARG;
    }
    for (const void* p : ps) {
        if (!aligned16(p)) return LORA_MLP_ERR_MISALIGNED;
    }
    return LORA_MLP_OK;
}

int check_weights(const lora_mlp_shape* sh, const lora_mlp_weights* w) {
    if (w == nullptr) return LORA_MLP_ERR_INVALID_ARG;
    int rc = check_ptrs({w->Wg, w->Wu, w->Wd, w->Ag, w->Bg, w->Au, w->Bu, w->Ad, w->Bd});
    if (rc) return rc;
    if (sh->weight_format != LORA_MLP_WEIGHTS_BF16) return check_ptrs({w->Sg, w->Su, w->Sd});
    return LORA_MLP_OK;
}

// Memory the kernels may touch: device or managed memory of the current
// device, as CUDA reports it.  Ordinary or page-locked host memory, another
// device's memory and addresses CUDA does not know are refused on the host,
// after the other argument checks and before anything is enqueued.
bool device_memory(const void* p) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    cudaPointerAttributes at{};
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (at.type == cudaMemoryTypeManaged) return true;
    return at.type == cudaMemoryTypeDevice && at.device == dev;
}
int check_memory(std::initializer_list<const void*> ps) {
    for (const void* p : ps)
        if (!device_memory(p)) return LORA_MLP_ERR_INVALID_ARG;
    return LORA_MLP_OK;
}
int check_weight_memory(const lora_mlp_shape* sh, const lora_mlp_weights* w) {
    const int rc = check_memory({w->Wg, w->Wu, w->Wd, w->Ag, w->Bg, w->Au, w->Bu, w->Ad, w->Bd});
    if (rc != LORA_MLP_OK) return rc;
    if (sh->weight_format != LORA_MLP_WEIGHTS_BF16) return check_memory({w->Sg, w->Su, w->Sd});
    return LORA_MLP_OK;
}

#define LMLP_TRY(expr)              \
    do {                            \
        const int rc_ = (expr);     \
        if (rc_ != LORA_MLP_OK) return rc_; \
    } while (0)

// int4 / FP8: the three weights' scales, transposed into the workspace at off[0..2]
// (Wg, Wu, Wd) for the GEMMs' scale maps.
int mlp_scales_t(const Plan& pl, const lora_mlp_weights* w, uint8_t* ws, const size_t* off, cudaStream_t st) {
    const void* src[3] = {w->Sg, w->Su, w->Sd};
    void* dst[3] = {ws + off[0], ws + off[1], ws + off[2]};
    const int64_t rows[3] = {pl.d_ff, pl.d_ff, pl.d};
    const int64_t cols[3] = {pl.d, pl.d, pl.d_ff};
    return launch_scale_t(pl.qf, 3, src, dst, rows, cols, st);
}

// The pre-norm block with gamma folded into the gate/up weights runs the
// MLP on the raw rows X with these hooks (X_hat = diag(rstd) X diag(gamma)):
// F0 uses A diag(gamma) and writes the saved rank-r copy scaled by rstd; the
// gate/up epilogue scales its accumulators by rstd; B-mid scales the copy of
// T that B5 reads by rstd; B4 uses A diag(gamma), so dX comes out as
// dX_hat * gamma; B5 scales dA by gamma.
struct Fold {
    const float* rstd;         // [N]
    const void* Ag;            // Ag diag(gamma), bf16 [r, d]
    const void* Au;            // Au diag(gamma)
    const void* gamma;         // bf16 [d]
};

}  // namespace

// ============================================================================= C ABI

extern "C" {

int lora_mlp_sizes(const lora_mlp_shape* shape, size_t* fwd_workspace_bytes, size_t* bwd_workspace_bytes,
                   size_t* saved_bytes) {
    LMLP_TRY(validate_shape(shape));
    const Plan pl = make_plan(*shape);
    if (fwd_workspace_bytes) *fwd_workspace_bytes = pl.f_total;
    if (bwd_workspace_bytes) *bwd_workspace_bytes = pl.b_total;
    if (saved_bytes) *saved_bytes = pl.s_total;
    return LORA_MLP_OK;
}

int lora_mlp_workspace_size(const lora_mlp_shape* shape, size_t* fwd_bytes, size_t* bwd_bytes) {
    return lora_mlp_sizes(shape, fwd_bytes, bwd_bytes, nullptr);
}

static int mlp_forward_impl(const lora_mlp_shape* shape, const lora_mlp_weights* w, const void* X, void* out,
                            void* g, void* u, void* saved, void* workspace, size_t workspace_bytes, void* stream,
                            const Fold* fold) {
    LMLP_TRY(validate_shape(shape));
    LMLP_TRY(check_weights(shape, w));
    LMLP_TRY(check_ptrs({X, out, g, u, saved, workspace}));
    const Plan pl = make_plan(*shape);
    if (workspace_bytes < pl.f_total) return LORA_MLP_ERR_WORKSPACE_TOO_SMALL;
    LMLP_TRY(check_weight_memory(shape, w));
    LMLP_TRY(check_memory({X, out, g, u, saved, workspace}));
    DevInfo di;
    LMLP_TRY(device_info(&di));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint8_t* sv = static_cast<uint8_t*>(saved);
    const int64_t N = pl.N, d = pl.d, dff = pl.d_ff, r = pl.r;
    __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(ws + pl.f_h);
    __nv_bfloat16* Sgu = reinterpret_cast<__nv_bfloat16*>(ws + pl.f_sgu);
    __nv_bfloat16* Sd = reinterpret_cast<__nv_bfloat16*>(ws + pl.f_sd);
    float* part = reinterpret_cast<float*>(ws + pl.f_part);
    int* ctr = reinterpret_cast<int*>(ws + pl.f_ctr);
    float* tailp = reinterpret_cast<float*>(ws + pl.f_tail);
    if (cudaMemsetAsync(ctr, 0, pl.ctr_bytes, st) != cudaSuccess) return LORA_MLP_ERR_CUDA;
    if (pl.qf) LMLP_TRY(mlp_scales_t(pl, w, ws, pl.f_st, st));
    {  // F0: [S_g | S_u] = s X [Ag; Au]^T  -> Sgu [N, 2r] and saved [S_g^T; S_u^T] [2r, ldN]
        GemmBuilder b(pl.bn_r);
        const int ax = b.a_k(X, N, d, d);
        const int bg = b.b_k(fold != nullptr ? fold->Ag : w->Ag, r, d, d);
        const int bu = b.b_k(fold != nullptr ? fold->Au : w->Au, r, d, d);
        Prob* p = b.prob(N, r, pl.splits[SK_F0][0]);
        b.seg(p, ax, bg, bu, d);
        p->out0 = part;
        p->out1 = part + r;
        p->ld = 2 * r;
        p->split_stride = N * 2 * r;
        b.fin(p, pl.s, static_cast<int>(2 * r), Sgu, 2 * r, sv + pl.s_sgT, nullptr, pl.ldN, static_cast<int>(2 * r));
        if (fold != nullptr) p->tr_row_scale = fold->rstd;
        LMLP_TRY((launch_gemm<2, EPI_F32>(b, di.sms, st, "F0_lowrank_in", ctr)));
    }
    {  // F1: G = X Wg^T + S_g Bg^T, U = X Wu^T + S_u Bu^T; g, u, h  (CTA pairs: half 0 = gate, half 1 = up)
        PairBuilder b(N, dff, 128);
        const int ax = b.a_k(X, N, d, d);
        const int asgu = b.a_k(Sgu, N, 2 * r, 2 * r);
        const int bwg = pl.qf ? b.q_map(w->Wg, dff, d, false, pl.qf) : b.b_k(w->Wg, dff, d, d);
        const int bwu = pl.qf ? b.q_map(w->Wu, dff, d, false, pl.qf) : b.b_k(w->Wu, dff, d, d);
        const int bbg = b.b_k(w->Bg, dff, r, r);
        const int bbu = b.b_k(w->Bu, dff, r, r);
        b.seg(ax, bwg, bwu, 0, 0, 0, 0, d);
        b.seg(asgu, bbg, bbu, 0, 0, 0, static_cast<int>(-r), 2 * r);
        b.a.prob.out0 = g;
        b.a.prob.out1 = u;
        b.a.prob.out2 = h;
        b.a.prob.ld = dff;
        if (fold != nullptr) b.a.prob.row_scale = fold->rstd;
        if (pl.qf) {
            const int sg = b.s_map(ws + pl.f_st[0], dff, d, false, pl.qf);
            const int su = b.s_map(ws + pl.f_st[1], dff, d, false, pl.qf);
            b.quant(0, bwg, bwu, sg, su);
        }
        LMLP_TRY((launch_pair_q<false, EPI_SWIGLU_FWD>(b, pl.qf, di.sms, st, "F1_gate_up_swiglu", tailp, ctr)));
    }
    {  // F2: S_d = s h Ad^T  -> Sd [N, r] and saved S_d^T [r, ldN]
        GemmBuilder b(pl.bn_r);
        const int ah = b.a_k(h, N, dff, dff);
        const int bad = b.b_k(w->Ad, r, dff, dff);
        Prob* p = b.prob(N, r, pl.splits[SK_F2][0]);
        b.seg(p, ah, bad, -1, dff);
        p->out0 = part;
        p->ld = r;
        p->split_stride = N * r;
        b.fin(p, pl.s, static_cast<int>(r), Sd, r, sv + pl.s_sdT, nullptr, pl.ldN, static_cast<int>(r));
        LMLP_TRY((launch_gemm<1, EPI_F32>(b, di.sms, st, "F2_lowrank_mid", ctr)));
    }
    {  // F3: out = h Wd^T + S_d Bd^T
        PairBuilder b(N, d, 256);
        const int ah = b.a_k(h, N, dff, dff);
        const int asd = b.a_k(Sd, N, r, r);
        const int bwd = pl.qf ? b.q_map(w->Wd, d, dff, false, pl.qf) : b.b_k(w->Wd, d, dff, dff);
        const int bbd = b.b_k(w->Bd, d, r, r);
        b.seg(ah, bwd, bwd, 0, kPairHalfN, 0, 0, dff);
        b.seg(asd, bbd, bbd, 0, kPairHalfN, 0, 0, r);
        b.a.prob.out0 = out;
        b.a.prob.ld = d;
        if (pl.qf) {
            const int sd = b.s_map(ws + pl.f_st[2], d, dff, false, pl.qf);
            b.quant(0, bwd, bwd, sd, sd);
        }
        LMLP_TRY((launch_pair_q<false, EPI_BF16>(b, pl.qf, di.sms, st, "F3_down", tailp, ctr)));
    }
    return LORA_MLP_OK;
}

static int mlp_backward_impl(const lora_mlp_shape* shape, const lora_mlp_weights* w, const void* X, const void* g,
                             const void* u, const void* saved, const void* dOut, void* dX,
                             const lora_mlp_grads* grads, void* workspace, size_t workspace_bytes, void* stream,
                             const Fold* fold) {
    LMLP_TRY(validate_shape(shape));
    LMLP_TRY(check_weights(shape, w));
    if (grads == nullptr) return LORA_MLP_ERR_INVALID_ARG;
    LMLP_TRY(check_ptrs({X, g, u, saved, dOut, dX, workspace, grads->dAg, grads->dBg, grads->dAu, grads->dBu,
                         grads->dAd, grads->dBd}));
    const Plan pl = make_plan(*shape);
    if (workspace_bytes < pl.b_total) return LORA_MLP_ERR_WORKSPACE_TOO_SMALL;
    LMLP_TRY(check_weight_memory(shape, w));
    LMLP_TRY(check_memory({X, g, u, saved, dOut, dX, workspace, grads->dAg, grads->dBg, grads->dAu, grads->dBu,
                           grads->dAd, grads->dBd}));
    DevInfo di;
    LMLP_TRY(device_info(&di));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const uint8_t* sv = static_cast<const uint8_t*>(saved);
    const int64_t N = pl.N, d = pl.d, dff = pl.d_ff, r = pl.r, ldN = pl.ldN;
    __nv_bfloat16* dg = reinterpret_cast<__nv_bfloat16*>(ws + pl.b_dg);
    __nv_bfloat16* du = reinterpret_cast<__nv_bfloat16*>(ws + pl.b_du);
    __nv_bfloat16* hb = reinterpret_cast<__nv_bfloat16*>(ws + pl.b_h);
    __nv_bfloat16* Td = reinterpret_cast<__nv_bfloat16*>(ws + pl.b_td);
    __nv_bfloat16* TdT = reinterpret_cast<__nv_bfloat16*>(ws + pl.b_tdT);
    __nv_bfloat16* Tgu = reinterpret_cast<__nv_bfloat16*>(ws + pl.b_tgu);
    __nv_bfloat16* TguT = reinterpret_cast<__nv_bfloat16*>(ws + pl.b_tguT);
    float* part = reinterpret_cast<float*>(ws + pl.b_part);
    int* ctr = reinterpret_cast<int*>(ws + pl.b_ctr);
    float* tailp = reinterpret_cast<float*>(ws + pl.b_tail);
    if (cudaMemsetAsync(ctr, 0, pl.ctr_bytes, st) != cudaSuccess) return LORA_MLP_ERR_CUDA;
    if (pl.qf) LMLP_TRY(mlp_scales_t(pl, w, ws, pl.b_st, st));
    const void* SgT = sv + pl.s_sgT;
    const void* SuT = sv + pl.s_suT;
    const void* SdT = sv + pl.s_sdT;
    if (pl.dual && !kDualBtMn) {
        // Bg^T, Bu^T for the single-pass adapter-gradient launch: they depend
        // on the weights only, so this runs first, off the chain of launches
        // that depend on each other's outputs
        __nv_bfloat16* BgT = reinterpret_cast<__nv_bfloat16*>(ws + pl.b_bT);
        LMLP_TRY(launch_adapter_t(w->Bg, w->Bu, BgT, BgT + r * dff, dff, r, st));
    }
    // adapter B matrices as K-major operands of the rank-r projections
    {  // B0: T_d = s dOut Bd -> Td [N, r], Td^T [r, ldN];  dBd = dOut^T S_d
        const int* sp = pl.splits[SK_B0];
        GemmBuilder b(pl.bn_r64);
        const int a0 = b.a_k(dOut, N, d, d);
        const int b0 = b.b_mn(w->Bd, d, r, r);
        const int a1 = b.a_mn(dOut, N, d, d);
        const int b1 = b.b_k(SdT, r, N, ldN);
        Prob* p0 = b.prob(N, r, sp[0], false, true);
        b.seg(p0, a0, b0, -1, d);
        p0->out0 = part + pl.part_off[SK_B0][0];
        p0->ld = r;
        p0->split_stride = N * r;
        b.fin(p0, pl.s, static_cast<int>(r), Td, r, TdT, nullptr, ldN, static_cast<int>(r));
        Prob* p1 = b.prob(d, r, sp[1], true, false);
        b.seg(p1, a1, b1, -1, N);
        p1->out0 = part + pl.part_off[SK_B0][1];
        p1->ld = r;
        p1->split_stride = d * r;
        b.fin(p1, 1.0f, static_cast<int>(r), grads->dBd, r, nullptr, nullptr, 0, static_cast<int>(r));
        LMLP_TRY((launch_gemm<1, EPI_F32>(b, di.sms, st, "B0_lowrank_out_dBd", ctr)));
    }
    {  // B1: dH = dOut Wd + T_d Ad, SwiGLU backward in the epilogue
        PairBuilder b(N, dff, 256);
        const int a = b.a_k(dOut, N, d, d);
        const int atd = b.a_k(Td, N, r, r);
        const int bwd = pl.qf ? b.q_map(w->Wd, d, dff, true, pl.qf) : b.b_mn(w->Wd, d, dff, dff);
        const int bad = b.b_mn(w->Ad, r, dff, dff);
        b.seg(a, bwd, bwd, 0, kPairHalfN, 0, 0, d);
        b.seg(atd, bad, bad, 0, kPairHalfN, 0, 0, r);
        PairProb& p = b.a.prob;
        p.in0 = g;
        p.in1 = u;
        p.out0 = dg;
        p.out1 = du;
        p.out2 = hb;
        p.ld = dff;
        if (pl.qf) {
            const int sd = b.s_map(ws + pl.b_st[2], d, dff, true, pl.qf);
            b.quant(0, bwd, bwd, sd, sd);
        }
        LMLP_TRY((launch_pair_q<true, EPI_SWIGLU_BWD>(b, pl.qf, di.sms, st, "B1_dh_swiglu_bwd", tailp, ctr)));
    }
    if (pl.dual) {  // B-mid in one pass over dg, du and h (ranks <= 32)
        const __nv_bfloat16* BgT = reinterpret_cast<const __nv_bfloat16*>(ws + pl.b_bT);
        LMLP_TRY(launch_dual(pl, dg, du, hb, kDualBtMn ? w->Bg : BgT, kDualBtMn ? w->Bu : BgT + r * dff, SgT, SuT,
                             TdT, ws, grads, Tgu, TguT, fold != nullptr ? fold->rstd : nullptr, st));
    } else {  // B-mid: T_g = s dg Bg, T_u = s du Bu -> Tgu [N, 2r], Tgu^T [2r, ldN];
       //        dAd = T_d^T h (written transposed);  dBg = dg^T S_g, dBu = du^T S_u
        const int* sp = pl.splits[SK_BMID];
        const size_t* po = pl.part_off[SK_BMID];
        GemmBuilder b(pl.bn_r64);
        const int adg_k = b.a_k(dg, N, dff, dff);
        const int adu_k = b.a_k(du, N, dff, dff);
        const int bbg = b.b_mn(w->Bg, dff, r, r);
        const int bbu = b.b_mn(w->Bu, dff, r, r);
        const int ah = b.a_mn(hb, N, dff, dff);
        const int btd = b.b_k(TdT, r, N, ldN);
        const int adg_m = b.a_mn(dg, N, dff, dff);
        const int adu_m = b.a_mn(du, N, dff, dff);
        const int bsg = b.b_k(SgT, r, N, ldN);
        const int bsu = b.b_k(SuT, r, N, ldN);
        Prob* tg = b.prob(N, r, sp[0], false, true);
        b.seg(tg, adg_k, bbg, -1, dff);
        tg->out0 = part + po[0];
        tg->ld = r;
        tg->split_stride = N * r;
        b.fin(tg, pl.s, static_cast<int>(r), Tgu, 2 * r, TguT, nullptr, ldN, static_cast<int>(r));
        if (fold != nullptr) tg->tr_row_scale = fold->rstd;
        Prob* tu = b.prob(N, r, sp[1], false, true);
        b.seg(tu, adu_k, bbu, -1, dff);
        tu->out0 = part + po[1];
        tu->ld = r;
        tu->split_stride = N * r;
        b.fin(tu, pl.s, static_cast<int>(r), Tgu + r, 2 * r, TguT + r * ldN, nullptr, ldN, static_cast<int>(r));
        if (fold != nullptr) tu->tr_row_scale = fold->rstd;
        Prob* pad = b.prob(dff, r, sp[2], true, false);
        b.seg(pad, ah, btd, -1, N);
        pad->out0 = part + po[2];
        pad->ld = r;
        pad->split_stride = dff * r;
        b.fin(pad, 1.0f, static_cast<int>(r), nullptr, 0, grads->dAd, nullptr, dff, static_cast<int>(r));
        Prob* pbg = b.prob(dff, r, sp[3], true, false);
        b.seg(pbg, adg_m, bsg, -1, N);
        pbg->out0 = part + po[3];
        pbg->ld = r;
        pbg->split_stride = dff * r;
        b.fin(pbg, 1.0f, static_cast<int>(r), grads->dBg, r, nullptr, nullptr, 0, static_cast<int>(r));
        Prob* pbu = b.prob(dff, r, sp[4], true, false);
        b.seg(pbu, adu_m, bsu, -1, N);
        pbu->out0 = part + po[4];
        pbu->ld = r;
        pbu->split_stride = dff * r;
        b.fin(pbu, 1.0f, static_cast<int>(r), grads->dBu, r, nullptr, nullptr, 0, static_cast<int>(r));
        // dg and du are read twice here (K-major for T, MN-major for dB) and
        // are larger than L2 together.  Taking the units in order of the
        // hidden features they read puts both reads of each feature band in
        // the same round, so the second one is served from L2.
        b.finish(ctr);
        b.order_units([](int prob, int tile, int kb0, int kb1) -> long long {
            return prob < 2 ? static_cast<long long>(kb0 + kb1) * (kBK / 2)    // T: K runs over features
                            : static_cast<long long>(tile) * kBM + kBM / 2;   // dAd, dB: M runs over features
        });
        LMLP_TRY((launch_gemm<1, EPI_F32>(b, di.sms, st, "B_mid_lowrank_grads", ctr)));
    }
    {  // B4: dX = dg Wg + du Wu + T_g Ag + T_u Au
        PairBuilder b(N, d, 256);
        const int adg = b.a_k(dg, N, dff, dff);
        const int adu = b.a_k(du, N, dff, dff);
        const int atg = b.a_k(Tgu, N, r, 2 * r);
        const int atu = b.a_k(Tgu + r, N, r, 2 * r);
        const int bwg = pl.qf ? b.q_map(w->Wg, dff, d, true, pl.qf) : b.b_mn(w->Wg, dff, d, d);
        const int bwu = pl.qf ? b.q_map(w->Wu, dff, d, true, pl.qf) : b.b_mn(w->Wu, dff, d, d);
        const int bag = b.b_mn(fold != nullptr ? fold->Ag : w->Ag, r, d, d);
        const int bau = b.b_mn(fold != nullptr ? fold->Au : w->Au, r, d, d);
        b.seg(adg, bwg, bwg, 0, kPairHalfN, 0, 0, dff);
        b.seg(adu, bwu, bwu, 0, kPairHalfN, 0, 0, dff);
        b.seg(atg, bag, bag, 0, kPairHalfN, 0, 0, r);
        b.seg(atu, bau, bau, 0, kPairHalfN, 0, 0, r);
        b.a.prob.out0 = dX;
        b.a.prob.ld = d;
        if (pl.qf) {
            const int sg = b.s_map(ws + pl.b_st[0], dff, d, true, pl.qf);
            const int su = b.s_map(ws + pl.b_st[1], dff, d, true, pl.qf);
            b.quant(0, bwg, bwg, sg, sg);
            b.quant(1, bwu, bwu, su, su);
        }
        LMLP_TRY((launch_pair_q<true, EPI_BF16>(b, pl.qf, di.sms, st, "B4_dX", tailp, ctr)));
    }
    {  // B5: [dAg; dAu]^T = X^T [T_g | T_u]  (written transposed: dAg, dAu [r, d])
        GemmBuilder b(pl.bn_2r);
        const int a = b.a_mn(X, N, d, d);
        const int bb = b.b_k(TguT, 2 * r, N, ldN);
        Prob* p = b.prob(d, 2 * r, pl.splits[SK_B5][0], true, false);
        b.seg(p, a, bb, -1, N);
        p->out0 = part;
        p->ld = 2 * r;
        p->split_stride = d * 2 * r;
        b.fin(p, 1.0f, static_cast<int>(2 * r), nullptr, 0, grads->dAg, grads->dAu, d, static_cast<int>(r));
        if (fold != nullptr) p->tr_row_scale_bf16 = static_cast<const __nv_bfloat16*>(fold->gamma);
        LMLP_TRY((launch_gemm<1, EPI_F32>(b, di.sms, st, "B5_dA_in", ctr)));
    }
    return LORA_MLP_OK;
}

int lora_mlp_forward(const lora_mlp_shape* shape, const lora_mlp_weights* w, const void* X, void* out, void* g,
                     void* u, void* saved, void* workspace, size_t workspace_bytes, void* stream) {
    return mlp_forward_impl(shape, w, X, out, g, u, saved, workspace, workspace_bytes, stream, nullptr);
}

int lora_mlp_backward(const lora_mlp_shape* shape, const lora_mlp_weights* w, const void* X, const void* g,
                      const void* u, const void* saved, const void* dOut, void* dX, const lora_mlp_grads* grads,
                      void* workspace, size_t workspace_bytes, void* stream) {
    return mlp_backward_impl(shape, w, X, g, u, saved, dOut, dX, grads, workspace, workspace_bytes, stream,
                             nullptr);
}

int lora_mlp_dequant_int4(const void* packed, const void* scales, int64_t rows, int64_t cols, void* w_bf16,
                          void* stream) {
    if (rows < 1 || cols < 1) return LORA_MLP_ERR_INVALID_ARG;
    if (cols % 64) return LORA_MLP_ERR_UNSUPPORTED_SHAPE;
    LMLP_TRY(check_ptrs({packed, scales, w_bf16}));
    LMLP_TRY(check_memory({packed, scales, w_bf16}));
    DevInfo di;
    LMLP_TRY(device_info(&di));
    return launch_dequant(packed, scales, rows, cols, w_bf16, di.sms, static_cast<cudaStream_t>(stream));
}

int lora_mlp_dequant_fp8(const void* codes, const void* scales, int64_t rows, int64_t cols, void* w_bf16,
                         void* stream) {
    if (rows < 1 || cols < 1) return LORA_MLP_ERR_INVALID_ARG;
    if (cols % 64) return LORA_MLP_ERR_UNSUPPORTED_SHAPE;
    LMLP_TRY(check_ptrs({codes, scales, w_bf16}));
    LMLP_TRY(check_memory({codes, scales, w_bf16}));
    DevInfo di;
    LMLP_TRY(device_info(&di));
    return launch_dequant_fp8(codes, scales, rows, cols, w_bf16, di.sms, static_cast<cudaStream_t>(stream));
}

int lora_mlp_check_pointer(const void* p, size_t alignment) {
    if (p == nullptr) return LORA_MLP_ERR_INVALID_ARG;
    if (alignment > 1 && reinterpret_cast<uintptr_t>(p) % alignment) return LORA_MLP_ERR_MISALIGNED;
    return device_memory(p) ? LORA_MLP_OK : LORA_MLP_ERR_INVALID_ARG;
}

int lora_mlp_device_status(void* stream, int* status) {
    if (status == nullptr) return LORA_MLP_ERR_INVALID_ARG;
    DevInfo di;
    LMLP_TRY(device_info(&di));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int v = 0;
    const int zero = 0;
    if (cudaMemcpyAsync(&v, di.status_addr, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaMemcpyAsync(di.status_addr, &zero, sizeof(int), cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return LORA_MLP_ERR_CUDA;
    *status = v;
    return LORA_MLP_OK;
}

const char* lora_mlp_strerror(int code) {
    switch (code) {
        case LORA_MLP_OK: return "ok";
        case LORA_MLP_ERR_INVALID_ARG: return "invalid argument";
        case LORA_MLP_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case LORA_MLP_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case LORA_MLP_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case LORA_MLP_ERR_UNSUPPORTED_ARCH: return "device is not compute capability 10.0 (B200)";
        case LORA_MLP_ERR_CUDA: return "CUDA error";
        case LORA_MLP_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait expired";
        default: return "unknown error";
    }
}

int lora_mlp_timing_enable(int enable) {
    g_timing.store(enable ? 1 : 0);
    return LORA_MLP_OK;
}

int lora_mlp_timing_collect(lora_mlp_kernel_time* out, int max, int* count) {
    std::lock_guard<std::mutex> lk(g_time_mu);
    int n = 0;
    int rc = LORA_MLP_OK;
    for (const TimingRec& rec : g_recs) {
        float ms = 0.0f;
        if (cudaEventSynchronize(rec.end) != cudaSuccess || cudaEventElapsedTime(&ms, rec.beg, rec.end) != cudaSuccess)
            rc = LORA_MLP_ERR_CUDA;
        if (out != nullptr && n < max) {
            out[n].name = rec.name;
            out[n].ms = ms;
        }
        ++n;
        g_event_pool.push_back(rec.beg);
        g_event_pool.push_back(rec.end);
    }
    g_recs.clear();
    if (count) *count = n;
    return rc;
}

int64_t lora_mlp_launch_count(void) { return g_launches.load(); }

int lora_mlp_debug_force_timeout(int enable, int64_t wait_cycles) {
    if (enable && wait_cycles < 1) return LORA_MLP_ERR_INVALID_ARG;
    g_wait_limit.store(enable ? static_cast<long long>(wait_cycles) : kWaitLimitCycles);
    g_force_timeout.store(enable ? 1 : 0);
    return LORA_MLP_OK;
}

}  // extern "C"

// ============================================================================= LoRA linear
//
// One LoRA-adapted projection (include/lora_linear.h), on the same engines:
//   L0  R  = s X A^T   -> R [N, r] and saved R^T [r, ldN]      split-K, finalised in kernel
//   L1  Y  = X W^T + R B^T                                     CTA pairs, K = d_in + r
//   L2  T  = s dY B    -> T [N, r], T^T [r, ldN];  dB = dY^T R  split-K, two problems
//   L3  dX = dY W + T A                                        CTA pairs, MN-major W and A
//   L4  dA = T^T X     (written [r, d_in])                     split-K token reduction

namespace {

enum { LK_R, LK_TDB, LK_DA, LK_COUNT };
constexpr int kLinProbs[LK_COUNT] = {1, 2, 1};

struct LinPlan {
    int64_t N, din, dout, r, ldN;
    float s;
    int qf;  // frozen-weight format
    int bn_r, bn_r64;
    SkinnySpec spec[LK_COUNT][kMaxProbs];
    int splits[LK_COUNT][kMaxProbs];
    size_t part_off[LK_COUNT][kMaxProbs];
    size_t ctr_bytes;
    size_t f_r, f_part, f_ctr, f_tail, f_st, f_total;  // f_st, b_st: block scales, transposed
    size_t b_t, b_tT, b_part, b_ctr, b_tail, b_st, b_total;
    size_t s_rT, s_total;
};

LinPlan make_lin_plan(const lora_linear_shape& sh) {
    LinPlan p{};
    p.N = sh.N;
    p.din = sh.d_in;
    p.dout = sh.d_out;
    p.r = sh.r;
    p.ldN = round_up(sh.N, 8);
    p.s = static_cast<float>(static_cast<double>(sh.alpha) / static_cast<double>(sh.r));
    p.qf = sh.weight_format == LORA_MLP_WEIGHTS_INT4_B64  ? QF_INT4
           : sh.weight_format == LORA_MLP_WEIGHTS_FP8_B64 ? QF_FP8
                                                           : QF_NONE;
    p.bn_r = static_cast<int>(round_up(sh.r, 32));
    p.bn_r64 = static_cast<int>(round_up(sh.r, 64));
    const int64_t N = p.N, di = p.din, dout = p.dout, r = p.r;
    const int64_t kb_in = ceil_div(di, kBK), kb_out = ceil_div(dout, kBK), kb_n = ceil_div(N, kBK);
    p.spec[LK_R][0] = {N, r, kb_in};
    p.spec[LK_TDB][0] = {N, r, kb_out};
    p.spec[LK_TDB][1] = {dout, r, kb_n};
    p.spec[LK_DA][0] = {di, r, kb_n};
    size_t part_f = 0, part_b = 0;
    int64_t max_tiles = 0;
    for (int l = 0; l < LK_COUNT; ++l) {
        plan_splits(p.spec[l], kLinProbs[l], p.splits[l]);
        size_t off = 0;
        for (int i = 0; i < kLinProbs[l]; ++i) {
            p.part_off[l][i] = off;
            off += static_cast<size_t>(p.splits[l][i]) * p.spec[l][i].M * p.spec[l][i].ncols;
        }
        if (l == LK_R) part_f = off;
        else part_b = std::max(part_b, off);
        max_tiles = std::max(max_tiles, launch_tiles(p.spec[l], kLinProbs[l]));
    }
    p.ctr_bytes = static_cast<size_t>(std::max<int64_t>(max_tiles, 2 * kTailMaxUnits) + 8) * sizeof(int);
    const size_t bf = 2, f32 = 4, rz = r, ldN = p.ldN;
    Carver f;
    p.f_r = f.take(static_cast<size_t>(N) * rz * bf);
    p.f_part = f.take(part_f * f32);
    p.f_ctr = f.take(p.ctr_bytes);
    p.f_tail = f.take(kTailPartFloats * f32);
    const size_t stsz = static_cast<size_t>(dout) * static_cast<size_t>(di) / 64 * (p.qf == QF_FP8 ? 4 : 2);
    p.f_st = p.qf ? f.take(stsz) : 0;
    p.f_total = f.off;
    Carver b;
    p.b_t = b.take(static_cast<size_t>(N) * rz * bf);
    p.b_tT = b.take(rz * ldN * bf);
    p.b_part = b.take(part_b * f32);
    p.b_ctr = b.take(p.ctr_bytes);
    p.b_tail = b.take(kTailPartFloats * f32);
    p.b_st = p.qf ? b.take(stsz) : 0;
    p.b_total = b.off;
    Carver sv;
    p.s_rT = sv.take(rz * ldN * bf);
    p.s_total = sv.off;
    return p;
}

int validate_lin_shape(const lora_linear_shape* sh) {
    if (sh == nullptr) return LORA_MLP_ERR_INVALID_ARG;
    if (sh->N < 1 || sh->d_in < 1 || sh->d_out < 1 || sh->r < 1) return LORA_MLP_ERR_INVALID_ARG;
    if (!std::isfinite(sh->alpha)) return LORA_MLP_ERR_INVALID_ARG;
    if (sh->weight_format != LORA_MLP_WEIGHTS_BF16 && sh->weight_format != LORA_MLP_WEIGHTS_INT4_B64 &&
        sh->weight_format != LORA_MLP_WEIGHTS_FP8_B64)
        return LORA_MLP_ERR_INVALID_ARG;
    if (sh->d_in % 8 || sh->d_out % 8 || sh->r % 8 || sh->r > 128) return LORA_MLP_ERR_UNSUPPORTED_SHAPE;
    if (sh->weight_format != LORA_MLP_WEIGHTS_BF16 && sh->d_in % 64) return LORA_MLP_ERR_UNSUPPORTED_SHAPE;
    const int64_t lim = (int64_t{1} << 31) - 1;
    if (sh->N > lim || sh->d_in > lim || sh->d_out > lim) return LORA_MLP_ERR_UNSUPPORTED_SHAPE;
    return LORA_MLP_OK;
}

int check_lin_weights(const lora_linear_shape* sh, const lora_linear_weights* w) {
    if (w == nullptr) return LORA_MLP_ERR_INVALID_ARG;
    LMLP_TRY(check_ptrs({w->W, w->A, w->B}));
    if (sh->weight_format != LORA_MLP_WEIGHTS_BF16) return check_ptrs({w->S});
    return LORA_MLP_OK;
}
int check_lin_weight_memory(const lora_linear_shape* sh, const lora_linear_weights* w) {
    LMLP_TRY(check_memory({w->W, w->A, w->B}));
    if (sh->weight_format != LORA_MLP_WEIGHTS_BF16) return check_memory({w->S});
    return LORA_MLP_OK;
}

}  // namespace

extern "C" {

int lora_linear_sizes(const lora_linear_shape* shape, size_t* fwd_workspace_bytes, size_t* bwd_workspace_bytes,
                      size_t* saved_bytes) {
    LMLP_TRY(validate_lin_shape(shape));
    const LinPlan pl = make_lin_plan(*shape);
    if (fwd_workspace_bytes) *fwd_workspace_bytes = pl.f_total;
    if (bwd_workspace_bytes) *bwd_workspace_bytes = pl.b_total;
    if (saved_bytes) *saved_bytes = pl.s_total;
    return LORA_MLP_OK;
}

int lora_linear_forward(const lora_linear_shape* shape, const lora_linear_weights* w, const void* X, void* Y,
                        void* saved, void* workspace, size_t workspace_bytes, void* stream) {
    LMLP_TRY(validate_lin_shape(shape));
    LMLP_TRY(check_lin_weights(shape, w));
    LMLP_TRY(check_ptrs({X, Y, saved, workspace}));
    const LinPlan pl = make_lin_plan(*shape);
    if (workspace_bytes < pl.f_total) return LORA_MLP_ERR_WORKSPACE_TOO_SMALL;
    LMLP_TRY(check_lin_weight_memory(shape, w));
    LMLP_TRY(check_memory({X, Y, saved, workspace}));
    DevInfo di;
    LMLP_TRY(device_info(&di));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint8_t* sv = static_cast<uint8_t*>(saved);
    const int64_t N = pl.N, din = pl.din, dout = pl.dout, r = pl.r;
    __nv_bfloat16* R = reinterpret_cast<__nv_bfloat16*>(ws + pl.f_r);
    float* part = reinterpret_cast<float*>(ws + pl.f_part);
    int* ctr = reinterpret_cast<int*>(ws + pl.f_ctr);
    float* tailp = reinterpret_cast<float*>(ws + pl.f_tail);
    if (cudaMemsetAsync(ctr, 0, pl.ctr_bytes, st) != cudaSuccess) return LORA_MLP_ERR_CUDA;
    if (pl.qf) {
        const void* src = w->S;
        void* dst = ws + pl.f_st;
        LMLP_TRY(launch_scale_t(pl.qf, 1, &src, &dst, &pl.dout, &pl.din, st));
    }
    {  // L0: R = s X A^T -> R [N, r], saved R^T [r, ldN]
        GemmBuilder b(pl.bn_r);
        const int ax = b.a_k(X, N, din, din);
        const int ba = b.b_k(w->A, r, din, din);
        Prob* p = b.prob(N, r, pl.splits[LK_R][0]);
        b.seg(p, ax, ba, -1, din);
        p->out0 = part;
        p->ld = r;
        p->split_stride = N * r;
        b.fin(p, pl.s, static_cast<int>(r), R, r, sv + pl.s_rT, nullptr, pl.ldN, static_cast<int>(r));
        LMLP_TRY((launch_gemm<1, EPI_F32>(b, di.sms, st, "L0_lowrank_in", ctr)));
    }
    {  // L1: Y = X W^T + R B^T
        PairBuilder b(N, dout, 256);
        const int ax = b.a_k(X, N, din, din);
        const int ar = b.a_k(R, N, r, r);
        const int bw = pl.qf ? b.q_map(w->W, dout, din, false, pl.qf) : b.b_k(w->W, dout, din, din);
        const int bb = b.b_k(w->B, dout, r, r);
        b.seg(ax, bw, bw, 0, kPairHalfN, 0, 0, din);
        b.seg(ar, bb, bb, 0, kPairHalfN, 0, 0, r);
        b.a.prob.out0 = Y;
        b.a.prob.ld = dout;
        if (pl.qf) {
            const int sm = b.s_map(ws + pl.f_st, dout, din, false, pl.qf);
            b.quant(0, bw, bw, sm, sm);
        }
        LMLP_TRY((launch_pair_q<false, EPI_BF16>(b, pl.qf, di.sms, st, "L1_linear_fwd", tailp, ctr)));
    }
    return LORA_MLP_OK;
}

int lora_linear_backward(const lora_linear_shape* shape, const lora_linear_weights* w, const void* X,
                         const void* saved, const void* dY, void* dX, void* dA, void* dB, void* workspace,
                         size_t workspace_bytes, void* stream) {
    LMLP_TRY(validate_lin_shape(shape));
    LMLP_TRY(check_lin_weights(shape, w));
    LMLP_TRY(check_ptrs({X, saved, dY, dX, dA, dB, workspace}));
    const LinPlan pl = make_lin_plan(*shape);
    if (workspace_bytes < pl.b_total) return LORA_MLP_ERR_WORKSPACE_TOO_SMALL;
    LMLP_TRY(check_lin_weight_memory(shape, w));
    LMLP_TRY(check_memory({X, saved, dY, dX, dA, dB, workspace}));
    DevInfo di;
    LMLP_TRY(device_info(&di));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const uint8_t* sv = static_cast<const uint8_t*>(saved);
    const int64_t N = pl.N, din = pl.din, dout = pl.dout, r = pl.r, ldN = pl.ldN;
    __nv_bfloat16* T = reinterpret_cast<__nv_bfloat16*>(ws + pl.b_t);
    __nv_bfloat16* TT = reinterpret_cast<__nv_bfloat16*>(ws + pl.b_tT);
    float* part = reinterpret_cast<float*>(ws + pl.b_part);
    int* ctr = reinterpret_cast<int*>(ws + pl.b_ctr);
    float* tailp = reinterpret_cast<float*>(ws + pl.b_tail);
    if (cudaMemsetAsync(ctr, 0, pl.ctr_bytes, st) != cudaSuccess) return LORA_MLP_ERR_CUDA;
    if (pl.qf) {
        const void* src = w->S;
        void* dst = ws + pl.b_st;
        LMLP_TRY(launch_scale_t(pl.qf, 1, &src, &dst, &pl.dout, &pl.din, st));
    }
    {  // L2: T = s dY B -> T [N, r], T^T [r, ldN];  dB = dY^T R (R from saved, already s-scaled)
        const int* sp = pl.splits[LK_TDB];
        GemmBuilder b(pl.bn_r64);
        const int a0 = b.a_k(dY, N, dout, dout);
        const int b0 = b.b_mn(w->B, dout, r, r);
        const int a1 = b.a_mn(dY, N, dout, dout);
        const int b1 = b.b_k(sv + pl.s_rT, r, N, ldN);
        Prob* p0 = b.prob(N, r, sp[0], false, true);
        b.seg(p0, a0, b0, -1, dout);
        p0->out0 = part + pl.part_off[LK_TDB][0];
        p0->ld = r;
        p0->split_stride = N * r;
        b.fin(p0, pl.s, static_cast<int>(r), T, r, TT, nullptr, ldN, static_cast<int>(r));
        Prob* p1 = b.prob(dout, r, sp[1], true, false);
        b.seg(p1, a1, b1, -1, N);
        p1->out0 = part + pl.part_off[LK_TDB][1];
        p1->ld = r;
        p1->split_stride = dout * r;
        b.fin(p1, 1.0f, static_cast<int>(r), dB, r, nullptr, nullptr, 0, static_cast<int>(r));
        LMLP_TRY((launch_gemm<1, EPI_F32>(b, di.sms, st, "L2_lowrank_out_dB", ctr)));
    }
    {  // L3: dX = dY W + T A
        PairBuilder b(N, din, 256);
        const int ady = b.a_k(dY, N, dout, dout);
        const int at = b.a_k(T, N, r, r);
        const int bw = pl.qf ? b.q_map(w->W, dout, din, true, pl.qf) : b.b_mn(w->W, dout, din, din);
        const int ba = b.b_mn(w->A, r, din, din);
        b.seg(ady, bw, bw, 0, kPairHalfN, 0, 0, dout);
        b.seg(at, ba, ba, 0, kPairHalfN, 0, 0, r);
        b.a.prob.out0 = dX;
        b.a.prob.ld = din;
        if (pl.qf) {
            const int sm = b.s_map(ws + pl.b_st, dout, din, true, pl.qf);
            b.quant(0, bw, bw, sm, sm);
        }
        LMLP_TRY((launch_pair_q<true, EPI_BF16>(b, pl.qf, di.sms, st, "L3_linear_dX", tailp, ctr)));
    }
    {  // L4: dA^T = X^T T  (written transposed: dA [r, d_in])
        GemmBuilder b(pl.bn_r);
        const int a = b.a_mn(X, N, din, din);
        const int bt = b.b_k(TT, r, N, ldN);
        Prob* p = b.prob(din, r, pl.splits[LK_DA][0], true, false);
        b.seg(p, a, bt, -1, N);
        p->out0 = part;
        p->ld = r;
        p->split_stride = din * r;
        b.fin(p, 1.0f, static_cast<int>(r), nullptr, 0, dA, nullptr, din, static_cast<int>(r));
        LMLP_TRY((launch_gemm<1, EPI_F32>(b, di.sms, st, "L4_dA", ctr)));
    }
    return LORA_MLP_OK;
}

}  // extern "C"

// ============================================================================= pre-norm block
//
// out = MLP(RMSNorm(X)): one norm launch, then the MLP's launches on the
// normalised rows.  Backward: the normalised rows are recomputed from X and
// the saved rstd (the same kernel and arithmetic as the forward, so the same
// bits), the MLP backward runs on them, and one launch maps its dX through
// the norm's backward.

namespace {

// Rows of up to 16384 (forward) / 8192 (backward) elements run one row per
// 128-thread CTA with the row in registers; wider rows fall back to the
// warp-per-row loop kernels.
int launch_rmsnorm_fwd(int64_t N, int64_t d, float eps, const void* x, const void* gamma, const float* rstd_in,
                       float* rstd_out, void* y, int sms, cudaStream_t st) {
    const auto* xb = static_cast<const __nv_bfloat16*>(x);
    const auto* gb = static_cast<const __nv_bfloat16*>(gamma);
    auto* yb = static_cast<__nv_bfloat16*>(y);
    const int di = static_cast<int>(d);
    const int64_t nch = (d / 8 + kRowThreads - 1) / kRowThreads;  // 8-element chunks per thread
    const long long cap = static_cast<long long>(sms) * 16;
    const dim3 rgrid(static_cast<unsigned>(N < cap ? N : cap)), rblock(kRowThreads);
    long long wblocks = (N + kRmsWarps - 1) / kRmsWarps;
    if (wblocks > static_cast<long long>(sms) * 8) wblocks = static_cast<long long>(sms) * 8;
    {
        LaunchScope scope("rmsnorm_fwd", st);
        if (nch <= 2) rmsnorm_fwd_row_kernel<2><<<rgrid, rblock, 0, st>>>(xb, gb, N, di, eps, rstd_in, rstd_out, yb);
        else if (nch <= 4)
            rmsnorm_fwd_row_kernel<4><<<rgrid, rblock, 0, st>>>(xb, gb, N, di, eps, rstd_in, rstd_out, yb);
        else if (nch <= 8)
            rmsnorm_fwd_row_kernel<8><<<rgrid, rblock, 0, st>>>(xb, gb, N, di, eps, rstd_in, rstd_out, yb);
        else if (nch <= 16)
            rmsnorm_fwd_row_kernel<16><<<rgrid, rblock, 0, st>>>(xb, gb, N, di, eps, rstd_in, rstd_out, yb);
        else
            rmsnorm_fwd_kernel<<<static_cast<unsigned>(wblocks), kRmsWarps * 32, 0, st>>>(xb, gb, N, di, eps,
                                                                                        rstd_in, rstd_out, yb);
    }
    return last_launch_error();
}

int launch_rmsnorm_bwd(int64_t N, int64_t d, const void* x, const void* gamma, const float* rstd, const void* dy,
                       void* dx, int sms, cudaStream_t st) {
    const auto* xb = static_cast<const __nv_bfloat16*>(x);
    const auto* gb = static_cast<const __nv_bfloat16*>(gamma);
    const auto* db = static_cast<const __nv_bfloat16*>(dy);
    auto* ob = static_cast<__nv_bfloat16*>(dx);
    const int di = static_cast<int>(d);
    const int64_t nch = (d / 8 + kRowThreads - 1) / kRowThreads;
    const long long cap = static_cast<long long>(sms) * 16;
    const dim3 rgrid(static_cast<unsigned>(N < cap ? N : cap)), rblock(kRowThreads);
    long long wblocks = (N + kRmsWarps - 1) / kRmsWarps;
    if (wblocks > static_cast<long long>(sms) * 8) wblocks = static_cast<long long>(sms) * 8;
    {
        LaunchScope scope("rmsnorm_bwd", st);
        if (nch <= 2) rmsnorm_bwd_row_kernel<2><<<rgrid, rblock, 0, st>>>(xb, gb, rstd, db, N, di, ob);
        else if (nch <= 4) rmsnorm_bwd_row_kernel<4><<<rgrid, rblock, 0, st>>>(xb, gb, rstd, db, N, di, ob);
        else if (nch <= 8) rmsnorm_bwd_row_kernel<8><<<rgrid, rblock, 0, st>>>(xb, gb, rstd, db, N, di, ob);
        else
            rmsnorm_bwd_kernel<<<static_cast<unsigned>(wblocks), kRmsWarps * 32, 0, st>>>(xb, gb, rstd, db, N, di,
                                                                                        ob);
    }
    return last_launch_error();
}

int validate_norm(int64_t N, int64_t d) {
    if (N < 1 || d < 1) return LORA_MLP_ERR_INVALID_ARG;
    if (d % 8) return LORA_MLP_ERR_UNSUPPORTED_SHAPE;
    const int64_t lim = (int64_t{1} << 31) - 1;
    if (N > lim || d > lim) return LORA_MLP_ERR_UNSUPPORTED_SHAPE;
    return LORA_MLP_OK;
}

// out = bf16_rne(in * gamma) over the columns of up to two bf16 [rows, cols]
// matrices, one launch.
int launch_scale_cols(const void* in0, const void* in1, void* out0, void* out1, int64_t rows, int64_t cols,
                      const void* gamma, int sms, cudaStream_t st) {
    ScaleCols a{};
    a.in[0] = static_cast<const __nv_bfloat16*>(in0);
    a.in[1] = static_cast<const __nv_bfloat16*>(in1);
    a.out[0] = static_cast<__nv_bfloat16*>(out0);
    a.out[1] = static_cast<__nv_bfloat16*>(out1);
    a.rows[0] = a.rows[1] = rows;
    long long blocks = (rows * (cols / 8) + 255) / 256;
    if (blocks > static_cast<long long>(sms) * 8) blocks = static_cast<long long>(sms) * 8;
    if (blocks < 1) blocks = 1;
    {
        LaunchScope scope("scale_cols", st);
        scale_cols_kernel<<<dim3(static_cast<unsigned>(blocks), 2), 256, 0, st>>>(
            a, static_cast<const __nv_bfloat16*>(gamma), static_cast<int>(cols));
    }
    return last_launch_error();
}

// Workspace / saved layout of the block (offsets in bytes).
struct BlockPlan {
    size_t xn, dxn, af, mlp_f, mlp_b, f_total, b_total;  // af: Ag, Au scaled by gamma (folded block)
    size_t s_mlp, s_rstd, s_total;
};

BlockPlan make_block_plan(const lora_mlp_shape& sh) {
    const Plan pl = make_plan(sh);
    BlockPlan b{};
    const size_t xbytes = static_cast<size_t>(sh.N) * static_cast<size_t>(sh.d) * 2;
    const size_t abytes = 2 * ((static_cast<size_t>(sh.r) * static_cast<size_t>(sh.d) * 2 + kAlign - 1) / kAlign * kAlign);
    Carver f;
    b.xn = f.take(xbytes);
    b.af = f.take(abytes);
    b.mlp_f = f.take(pl.f_total);
    b.f_total = f.off;
    Carver k;
    k.take(xbytes);  // xn and af at the same offsets in both workspaces
    k.take(abytes);
    b.dxn = k.take(xbytes);
    b.mlp_b = k.take(pl.b_total);
    b.b_total = k.off;
    Carver sv;
    b.s_mlp = sv.take(pl.s_total);
    b.s_rstd = sv.take(static_cast<size_t>(sh.N) * sizeof(float));
    b.s_total = sv.off;
    return b;
}

}  // namespace

extern "C" {

int lora_rmsnorm_forward(int64_t N, int64_t d, float eps, const void* x, const void* gamma, void* y, void* rstd,
                         void* stream) {
    LMLP_TRY(validate_norm(N, d));
    if (!std::isfinite(eps) || eps < 0.0f) return LORA_MLP_ERR_INVALID_ARG;
    LMLP_TRY(check_ptrs({x, gamma, y, rstd}));
    LMLP_TRY(check_memory({x, gamma, y, rstd}));
    DevInfo di;
    LMLP_TRY(device_info(&di));
    return launch_rmsnorm_fwd(N, d, eps, x, gamma, nullptr, static_cast<float*>(rstd), y, di.sms,
                              static_cast<cudaStream_t>(stream));
}

int lora_rmsnorm_backward(int64_t N, int64_t d, const void* x, const void* gamma, const void* rstd, const void* dy,
                          void* dx, void* stream) {
    LMLP_TRY(validate_norm(N, d));
    LMLP_TRY(check_ptrs({x, gamma, rstd, dy, dx}));
    LMLP_TRY(check_memory({x, gamma, rstd, dy, dx}));
    DevInfo di;
    LMLP_TRY(device_info(&di));
    return launch_rmsnorm_bwd(N, d, x, gamma, static_cast<const float*>(rstd), dy, dx, di.sms,
                              static_cast<cudaStream_t>(stream));
}

int lora_mlp_block_sizes(const lora_mlp_shape* shape, size_t* fwd_workspace_bytes, size_t* bwd_workspace_bytes,
                         size_t* saved_bytes) {
    LMLP_TRY(validate_shape(shape));
    const BlockPlan b = make_block_plan(*shape);
    if (fwd_workspace_bytes) *fwd_workspace_bytes = b.f_total;
    if (bwd_workspace_bytes) *bwd_workspace_bytes = b.b_total;
    if (saved_bytes) *saved_bytes = b.s_total;
    return LORA_MLP_OK;
}

int lora_mlp_block_forward(const lora_mlp_shape* shape, const lora_mlp_weights* w, const void* gamma, float eps,
                           const void* X, void* out, void* g, void* u, void* saved, void* workspace,
                           size_t workspace_bytes, void* stream) {
    LMLP_TRY(validate_shape(shape));
    LMLP_TRY(check_weights(shape, w));
    if (!std::isfinite(eps) || eps < 0.0f) return LORA_MLP_ERR_INVALID_ARG;
    LMLP_TRY(check_ptrs({gamma, X, out, g, u, saved, workspace}));
    const BlockPlan b = make_block_plan(*shape);
    if (workspace_bytes < b.f_total) return LORA_MLP_ERR_WORKSPACE_TOO_SMALL;
    LMLP_TRY(check_weight_memory(shape, w));
    LMLP_TRY(check_memory({gamma, X, out, g, u, saved, workspace}));
    DevInfo di;
    LMLP_TRY(device_info(&di));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint8_t* sv = static_cast<uint8_t*>(saved);
    LMLP_TRY(launch_rmsnorm_fwd(shape->N, shape->d, eps, X, gamma, nullptr, reinterpret_cast<float*>(sv + b.s_rstd),
                                ws + b.xn, di.sms, st));
    return lora_mlp_forward(shape, w, ws + b.xn, out, g, u, sv + b.s_mlp, ws + b.mlp_f, b.f_total - b.mlp_f,
                            stream);
}

int lora_mlp_block_backward(const lora_mlp_shape* shape, const lora_mlp_weights* w, const void* gamma, const void* X,
                            const void* g, const void* u, const void* saved, const void* dOut, void* dX,
                            const lora_mlp_grads* grads, void* workspace, size_t workspace_bytes, void* stream) {
    LMLP_TRY(validate_shape(shape));
    LMLP_TRY(check_weights(shape, w));
    LMLP_TRY(check_ptrs({gamma, X, g, u, saved, dOut, dX, workspace}));
    const BlockPlan b = make_block_plan(*shape);
    if (workspace_bytes < b.b_total) return LORA_MLP_ERR_WORKSPACE_TOO_SMALL;
    LMLP_TRY(check_weight_memory(shape, w));
    LMLP_TRY(check_memory({gamma, X, g, u, saved, dOut, dX, workspace}));
    DevInfo di;
    LMLP_TRY(device_info(&di));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const uint8_t* sv = static_cast<const uint8_t*>(saved);
    const float* rstd = reinterpret_cast<const float*>(sv + b.s_rstd);
    LMLP_TRY(launch_rmsnorm_fwd(shape->N, shape->d, 0.0f, X, gamma, rstd, nullptr, ws + b.xn, di.sms, st));
    LMLP_TRY(lora_mlp_backward(shape, w, ws + b.xn, g, u, sv + b.s_mlp, dOut, ws + b.dxn, grads, ws + b.mlp_b,
                               b.b_total - b.mlp_b, stream));
    return launch_rmsnorm_bwd(shape->N, shape->d, X, gamma, rstd, ws + b.dxn, dX, di.sms, st);
}

int lora_mlp_block_fold_gamma(const lora_mlp_shape* shape, const lora_mlp_weights* w, const void* gamma,
                              void* Wg_folded, void* Wu_folded, void* stream) {
    LMLP_TRY(validate_shape(shape));
    if (shape->weight_format != LORA_MLP_WEIGHTS_BF16) return LORA_MLP_ERR_INVALID_ARG;
    LMLP_TRY(check_weights(shape, w));
    LMLP_TRY(check_ptrs({gamma, Wg_folded, Wu_folded}));
    LMLP_TRY(check_weight_memory(shape, w));
    LMLP_TRY(check_memory({gamma, Wg_folded, Wu_folded}));
    DevInfo di;
    LMLP_TRY(device_info(&di));
    return launch_scale_cols(w->Wg, w->Wu, Wg_folded, Wu_folded, shape->d_ff, shape->d, gamma, di.sms,
                             static_cast<cudaStream_t>(stream));
}

int lora_mlp_block_forward_folded(const lora_mlp_shape* shape, const lora_mlp_weights* w_folded, const void* gamma,
                                  float eps, const void* X, void* out, void* g, void* u, void* saved,
                                  void* workspace, size_t workspace_bytes, void* stream) {
    LMLP_TRY(validate_shape(shape));
    if (shape->weight_format != LORA_MLP_WEIGHTS_BF16) return LORA_MLP_ERR_INVALID_ARG;
    LMLP_TRY(check_weights(shape, w_folded));
    if (!std::isfinite(eps) || eps < 0.0f) return LORA_MLP_ERR_INVALID_ARG;
    LMLP_TRY(check_ptrs({gamma, X, out, g, u, saved, workspace}));
    const BlockPlan b = make_block_plan(*shape);
    if (workspace_bytes < b.f_total) return LORA_MLP_ERR_WORKSPACE_TOO_SMALL;
    LMLP_TRY(check_weight_memory(shape, w_folded));
    LMLP_TRY(check_memory({gamma, X, out, g, u, saved, workspace}));
    DevInfo di;
    LMLP_TRY(device_info(&di));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint8_t* sv = static_cast<uint8_t*>(saved);
    float* rstd = reinterpret_cast<float*>(sv + b.s_rstd);
    const size_t ab = (b.mlp_f - b.af) / 2;
    // rstd only (no normalised rows), then A diag(gamma) for both adapters
    LMLP_TRY(launch_rmsnorm_fwd(shape->N, shape->d, eps, X, nullptr, nullptr, rstd, nullptr, di.sms, st));
    LMLP_TRY(launch_scale_cols(w_folded->Ag, w_folded->Au, ws + b.af, ws + b.af + ab, shape->r, shape->d, gamma,
                               di.sms, st));
    const Fold f{rstd, ws + b.af, ws + b.af + ab, gamma};
    return mlp_forward_impl(shape, w_folded, X, out, g, u, sv + b.s_mlp, ws + b.mlp_f, b.f_total - b.mlp_f, stream,
                            &f);
}

int lora_mlp_block_backward_folded(const lora_mlp_shape* shape, const lora_mlp_weights* w_folded, const void* gamma,
                                   const void* X, const void* g, const void* u, const void* saved, const void* dOut,
                                   void* dX, const lora_mlp_grads* grads, void* workspace, size_t workspace_bytes,
                                   void* stream) {
    LMLP_TRY(validate_shape(shape));
    if (shape->weight_format != LORA_MLP_WEIGHTS_BF16) return LORA_MLP_ERR_INVALID_ARG;
    LMLP_TRY(check_weights(shape, w_folded));
    LMLP_TRY(check_ptrs({gamma, X, g, u, saved, dOut, dX, workspace}));
    const BlockPlan b = make_block_plan(*shape);
    if (workspace_bytes < b.b_total) return LORA_MLP_ERR_WORKSPACE_TOO_SMALL;
    LMLP_TRY(check_weight_memory(shape, w_folded));
    LMLP_TRY(check_memory({gamma, X, g, u, saved, dOut, dX, workspace}));
    DevInfo di;
    LMLP_TRY(device_info(&di));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const uint8_t* sv = static_cast<const uint8_t*>(saved);
    const float* rstd = reinterpret_cast<const float*>(sv + b.s_rstd);
    const size_t ab = (b.dxn - b.af) / 2;
    LMLP_TRY(launch_scale_cols(w_folded->Ag, w_folded->Au, ws + b.af, ws + b.af + ab, shape->r, shape->d, gamma,
                               di.sms, st));
    const Fold f{rstd, ws + b.af, ws + b.af + ab, gamma};
    // the dX GEMM on the folded weights gives dX_hat * gamma; the norm's
    // backward with gamma = 1 maps it to dX
    LMLP_TRY(mlp_backward_impl(shape, w_folded, X, g, u, sv + b.s_mlp, dOut, ws + b.dxn, grads, ws + b.mlp_b,
                               b.b_total - b.mlp_b, stream, &f));
    return launch_rmsnorm_bwd(shape->N, shape->d, X, nullptr, rstd, ws + b.dxn, dX, di.sms, st);
}

}  // extern "C"

// ============================================================================= cross-entropy
//
// Chunked cross-entropy (include/lora_ce.h): the forward reduces every
// (row, vocabulary chunk) to its (max, sum of exp) in one launch and combines
// each row's chunks in chunk order in a second; the backward is one
// streaming launch over the same (row, chunk) grid.

namespace {

int validate_ce(const lora_ce_shape* sh) {
    if (sh == nullptr) return LORA_MLP_ERR_INVALID_ARG;
    if (sh->N < 1 || sh->V < 1 || sh->ld < sh->V) return LORA_MLP_ERR_INVALID_ARG;
    if (!std::isfinite(sh->logit_scale) || sh->logit_scale == 0.0f) return LORA_MLP_ERR_INVALID_ARG;
    if (!std::isfinite(sh->softcap) || sh->softcap < 0.0f) return LORA_MLP_ERR_INVALID_ARG;
    if (sh->ld % kCeVec != 0) return LORA_MLP_ERR_UNSUPPORTED_SHAPE;
    const long long nchunk = (sh->V + kCeChunk - 1) / kCeChunk;
    if (sh->N > (static_cast<long long>(INT32_MAX) / nchunk)) return LORA_MLP_ERR_UNSUPPORTED_SHAPE;
    return LORA_MLP_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

CeArgs ce_args(const lora_ce_shape* sh, const void* logits, const int64_t* labels) {
    CeArgs a;
    a.z = static_cast<const __nv_bfloat16*>(logits);
    a.ld = sh->ld;
    a.V = sh->V;
    a.N = sh->N;
    a.nchunk = static_cast<int>((sh->V + kCeChunk - 1) / kCeChunk);
    a.labels = reinterpret_cast<const long long*>(labels);
    a.ignore = sh->ignore_index;
    a.scale = sh->logit_scale;
    a.cap = sh->softcap;
    const bool cap = sh->softcap > 0.0f;
    a.k2 = cap ? 2.0f * sh->logit_scale / sh->softcap * kLog2e : 0.0f;
    a.inv_cap = cap ? 1.0f / sh->softcap : 0.0f;
    return a;
}

struct CePlan {
    size_t part, ty, rows, total;  // rows: per-row losses of the reduced forward
};

CePlan make_ce_plan(const lora_ce_shape& sh) {
    const size_t nchunk = static_cast<size_t>((sh.V + kCeChunk - 1) / kCeChunk);
    Carver c;
    CePlan p;
    p.part = c.take(static_cast<size_t>(sh.N) * nchunk * sizeof(float2));
    p.ty = c.take(static_cast<size_t>(sh.N) * sizeof(float));
    p.rows = c.take(static_cast<size_t>(sh.N) * sizeof(float));
    p.total = c.off;
    return p;
}

// The chunk partials and their per-row combination into loss [N] and lse [N].
int ce_forward_rows(const lora_ce_shape* shape, const CePlan& pl, const CeArgs& a, uint8_t* ws, float* loss,
                    float* lse, cudaStream_t st) {
    float2* part = reinterpret_cast<float2*>(ws + pl.part);
    float* ty = reinterpret_cast<float*>(ws + pl.ty);
    {
        LaunchScope scope("CE_fwd_chunks", st);
        ce_fwd_partial_kernel<<<static_cast<unsigned>(shape->N * a.nchunk), kCeThreads, 0, st>>>(a, part, ty);
    }
    LMLP_TRY(last_launch_error());
    {
        LaunchScope scope("CE_fwd_combine", st);
        ce_fwd_combine_kernel<<<static_cast<unsigned>((shape->N + 255) / 256), 256, 0, st>>>(a, part, ty, loss,
                                                                                            lse);
    }
    return last_launch_error();
}

int ce_backward_impl(const lora_ce_shape* shape, const void* logits, const int64_t* labels, const float* lse,
                     const float* dloss, long long dloss_stride, const float* dfactor, void* dlogits,
                     cudaStream_t st) {
    const CeArgs a = ce_args(shape, logits, labels);
    {
        LaunchScope scope("CE_bwd", st);
        ce_bwd_kernel<<<static_cast<unsigned>(shape->N * a.nchunk), kCeThreads, 0, st>>>(
            a, lse, dloss, dloss_stride, dfactor, static_cast<__nv_bfloat16*>(dlogits), shape->ld);
    }
    return last_launch_error();
}

}  // namespace

extern "C" {

int lora_ce_sizes(const lora_ce_shape* shape, size_t* workspace_bytes) {
    LMLP_TRY(validate_ce(shape));
    if (workspace_bytes) *workspace_bytes = make_ce_plan(*shape).total;
    return LORA_MLP_OK;
}

int lora_ce_forward(const lora_ce_shape* shape, const void* logits, const int64_t* labels, float* loss, float* lse,
                    void* workspace, size_t workspace_bytes, void* stream) {
    LMLP_TRY(validate_ce(shape));
    if (logits == nullptr || labels == nullptr || loss == nullptr || lse == nullptr || workspace == nullptr)
        return LORA_MLP_ERR_INVALID_ARG;
    if (!aligned(logits, 16) || !aligned(labels, 8) || !aligned(loss, 4) || !aligned(lse, 4) ||
        !aligned(workspace, 16))
        return LORA_MLP_ERR_MISALIGNED;
    const CePlan pl = make_ce_plan(*shape);
    if (workspace_bytes < pl.total) return LORA_MLP_ERR_WORKSPACE_TOO_SMALL;
    LMLP_TRY(check_memory({logits, labels, loss, lse, workspace}));
    DevInfo di;
    LMLP_TRY(device_info(&di));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const CeArgs a = ce_args(shape, logits, labels);
    return ce_forward_rows(shape, pl, a, static_cast<uint8_t*>(workspace), loss, lse, st);
}

int lora_ce_forward_reduced(const lora_ce_shape* shape, const void* logits, const int64_t* labels, int reduction,
                            float* out, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
    LMLP_TRY(validate_ce(shape));
    if (reduction != LORA_CE_REDUCTION_SUM && reduction != LORA_CE_REDUCTION_MEAN) return LORA_MLP_ERR_INVALID_ARG;
    if (logits == nullptr || labels == nullptr || out == nullptr || lse == nullptr || workspace == nullptr)
        return LORA_MLP_ERR_INVALID_ARG;
    if (!aligned(logits, 16) || !aligned(labels, 8) || !aligned(out, 8) || !aligned(lse, 4) ||
        !aligned(workspace, 16))
        return LORA_MLP_ERR_MISALIGNED;
    const CePlan pl = make_ce_plan(*shape);
    if (workspace_bytes < pl.total) return LORA_MLP_ERR_WORKSPACE_TOO_SMALL;
    LMLP_TRY(check_memory({logits, labels, out, lse, workspace}));
    DevInfo di;
    LMLP_TRY(device_info(&di));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const CeArgs a = ce_args(shape, logits, labels);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* rows = reinterpret_cast<float*>(ws + pl.rows);
    LMLP_TRY(ce_forward_rows(shape, pl, a, ws, rows, lse, st));
    {
        LaunchScope scope("CE_fwd_reduce", st);
        ce_reduce_kernel<<<1, kCeReduceThreads, 0, st>>>(a, rows, reduction == LORA_CE_REDUCTION_MEAN, out);
    }
    return last_launch_error();
}

int lora_ce_backward(const lora_ce_shape* shape, const void* logits, const int64_t* labels, const float* lse,
                     const float* dloss, void* dlogits, void* stream) {
    LMLP_TRY(validate_ce(shape));
    if (logits == nullptr || labels == nullptr || lse == nullptr || dloss == nullptr || dlogits == nullptr)
        return LORA_MLP_ERR_INVALID_ARG;
    if (!aligned(logits, 16) || !aligned(dlogits, 16) || !aligned(labels, 8) || !aligned(lse, 4) ||
        !aligned(dloss, 4))
        return LORA_MLP_ERR_MISALIGNED;
    LMLP_TRY(check_memory({logits, labels, lse, dloss, dlogits}));
    DevInfo di;
    LMLP_TRY(device_info(&di));
    return ce_backward_impl(shape, logits, labels, lse, dloss, 1, nullptr, dlogits, static_cast<cudaStream_t>(stream));
}

int lora_ce_backward_reduced(const lora_ce_shape* shape, const void* logits, const int64_t* labels,
                             const float* lse, const float* dout, const float* fwd_out, void* dlogits,
                             void* stream) {
    LMLP_TRY(validate_ce(shape));
    if (logits == nullptr || labels == nullptr || lse == nullptr || dout == nullptr || fwd_out == nullptr ||
        dlogits == nullptr)
        return LORA_MLP_ERR_INVALID_ARG;
    if (!aligned(logits, 16) || !aligned(dlogits, 16) || !aligned(labels, 8) || !aligned(lse, 4) ||
        !aligned(dout, 4) || !aligned(fwd_out, 8))
        return LORA_MLP_ERR_MISALIGNED;
    LMLP_TRY(check_memory({logits, labels, lse, dout, fwd_out, dlogits}));
    DevInfo di;
    LMLP_TRY(device_info(&di));
    return ce_backward_impl(shape, logits, labels, lse, dout, 0, fwd_out, dlogits, static_cast<cudaStream_t>(stream));
}

int lora_ce_device_status(void* stream, int* status) {
    if (status == nullptr) return LORA_MLP_ERR_INVALID_ARG;
    DevInfo di;
    LMLP_TRY(device_info(&di));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_ce_status) != cudaSuccess) return LORA_MLP_ERR_CUDA;
    int v = 0;
    const int zero = 0;
    if (cudaMemcpyAsync(&v, addr, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaMemcpyAsync(addr, &zero, sizeof(int), cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return LORA_MLP_ERR_CUDA;
    *status = v;
    return LORA_MLP_OK;
}

}  // extern "C"
