/*
 * lora_mlp.h — C ABI of the fused LoRA + SwiGLU MLP for NVIDIA B200 (sm_100a).
 *
 * The operation.  A SwiGLU MLP whose gate, up and down projections each carry
 * a LoRA adapter, run forward and backward as one fused unit with
 * hand-derived gradients, so that the intermediates autograd would keep are
 * never stored ("Unsloth 深度分析报告", nightvoyager.top, section 核心价值提炼 /
 * 创新之处, item "融合 LoRA MLP 反向传播 Kernel"; matmul and LoRA fused into
 * single kernels: "Unsloth 还是 AirLLM？一个炼丹，一个硬跑", section 核心原理).
 * With s = alpha / r and the nn.Linear layout (W [out, in], A [r, in], B [out, r]):
 *
 *   G   = X Wg^T + s (X Ag^T) Bg^T          U = X Wu^T + s (X Au^T) Bu^T
 *   H   = silu(G) * U                        out = H Wd^T + s (H Ad^T) Bd^T
 *
 * and the backward gives dX and the six adapter gradients for an upstream dOut
 * (the frozen W get no gradient).
 *
 * Conventions shared by every entry point
 *  - Every pointer is caller-owned memory; the library never allocates or
 *    frees device memory, and never synchronises the stream (except
 *    lora_mlp_device_status, which says so).  Work is enqueued on `stream`
 *    (a cudaStream_t passed as void*; NULL = the legacy default stream) on
 *    the current CUDA device.  int4 and FP8 frozen weights are dequantised
 *    inside the GEMM kernels that read them; no bf16 copy of a weight is made.
 *  - Float tensors are bf16, row-major, densely packed (leading dimension =
 *    the row length).  Device pointers must be 16-byte aligned.
 *  - Sizes: N >= 1 tokens; d, d_ff multiples of 8 (of 64 for int4 and FP8 weights);
 *    r a multiple of 8 in [8, 128]; alpha finite.
 *  - Results are written, never accumulated into.  Results are deterministic:
 *    the same inputs give the same bits on every run.
 *  - Return value: LORA_MLP_OK or a negative LORA_MLP_ERR_* code.  Argument
 *    errors are detected on the host before anything is enqueued.
 *  - Not thread-safe on one stream; independent streams may be used from
 *    several threads.
 */
#ifndef LORA_MLP_H
#define LORA_MLP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LORA_MLP_OK 0
#define LORA_MLP_ERR_INVALID_ARG (-1)         /* null pointer, memory that is not the current device's
                                                 (host, another device's, unknown), non-positive size,
                                                 non-finite alpha */
#define LORA_MLP_ERR_UNSUPPORTED_SHAPE (-2)   /* divisibility or range rule above violated        */
#define LORA_MLP_ERR_MISALIGNED (-3)          /* a device pointer is not 16-byte aligned          */
#define LORA_MLP_ERR_WORKSPACE_TOO_SMALL (-4) /* workspace_bytes below lora_mlp_sizes()           */
#define LORA_MLP_ERR_UNSUPPORTED_ARCH (-5)    /* current device is not compute capability 10.0    */
#define LORA_MLP_ERR_CUDA (-6)                /* a CUDA runtime call or launch failed             */
#define LORA_MLP_ERR_DEVICE_TIMEOUT (-7)      /* a kernel's bounded wait expired (see device_status) */

/* Storage format of the frozen weights Wg, Wu, Wd. */
#define LORA_MLP_WEIGHTS_BF16 0
/* Symmetric int4 codes in [-7, 7], blocks of 64 consecutive input-dimension
 * elements, one fp16 scale (the block's absolute maximum) per block:
 * w = bf16_rne((fp32(q) * fp32(scale)) / 7.0f).  Packed as uint8
 * [out, in/2] with element 2k in the low nibble of byte k (two's complement);
 * scales fp16 [out, in/64] row-major.  ("native 4-bit QLoRA": blog.cn-res.vip
 * page, 核心原理; the block layout itself is this library's choice.) */
#define LORA_MLP_WEIGHTS_INT4_B64 1
/* FP8 codes: OCP 8-bit floating point E4M3 (1 sign, 4 exponent bits with
 * bias 7, 3 mantissa bits; subnormals m/8 * 2^-6; no infinities; S.1111.111
 * is NaN), one byte per element, uint8 [out, in]; one fp32 scale per 64
 * consecutive input-dimension elements, fp32 [out, in/64] row-major:
 * w = bf16_rne(fp32(e4m3) * scale), the fp32 product rounded once.  (The
 * pages name FP8 as a kernel family and a weight format without defining
 * one: "Unsloth 深度分析报告", 关键设计决策; "Unsloth 还是 AirLLM", 核心原理.
 * The block layout and scale type are this library's choice.) */
#define LORA_MLP_WEIGHTS_FP8_B64 2

typedef struct lora_mlp_shape {
    int64_t N;             /* tokens (rows of X)          */
    int64_t d;             /* model width                 */
    int64_t d_ff;          /* MLP hidden width            */
    int64_t r;             /* LoRA rank                   */
    float alpha;           /* LoRA scale numerator, s = alpha / r */
    int32_t weight_format; /* LORA_MLP_WEIGHTS_*          */
} lora_mlp_shape;

/* Device pointers.  bf16 format: Wg, Wu [d_ff, d], Wd [d, d_ff] and Sg = Su =
 * Sd = NULL.  int4 format: Wg, Wu uint8 [d_ff, d/2], Wd uint8 [d, d_ff/2]
 * packed codes; Sg, Su fp16 [d_ff, d/64], Sd fp16 [d, d_ff/64].  FP8 format:
 * Wg, Wu uint8 [d_ff, d], Wd uint8 [d, d_ff] E4M3 codes; Sg, Su fp32
 * [d_ff, d/64], Sd fp32 [d, d_ff/64].
 * Adapters, always bf16: Ag, Au [r, d]; Bg, Bu [d_ff, r]; Ad [r, d_ff]; Bd [d, r]. */
typedef struct lora_mlp_weights {
    const void *Wg, *Wu, *Wd;
    const void *Sg, *Su, *Sd;
    const void *Ag, *Bg, *Au, *Bu, *Ad, *Bd;
} lora_mlp_weights;

/* Device pointers to the adapter gradients, bf16, same shapes as the adapters. */
typedef struct lora_mlp_grads {
    void *dAg, *dBg, *dAu, *dBu, *dAd, *dBd;
} lora_mlp_grads;

/* Byte sizes the caller must provide: the scratch workspace of forward and of
 * backward (one buffer may serve both in turn), and the `saved` buffer that
 * forward fills with the rank-r projections s·X·Ag^T, s·X·Au^T, s·H·Ad^T and
 * backward reads back (an opaque layout; keep it alive from forward to
 * backward together with g and u).  Pure host function, no CUDA call.
 * Any output pointer may be NULL. */
int lora_mlp_sizes(const lora_mlp_shape* shape, size_t* fwd_workspace_bytes,
                   size_t* bwd_workspace_bytes, size_t* saved_bytes);

/* The two workspace sizes alone (the same numbers lora_mlp_sizes gives),
 * for callers that size scratch separately from the saved buffer.  Host
 * only; either output pointer may be NULL. */
int lora_mlp_workspace_size(const lora_mlp_shape* shape, size_t* fwd_workspace_bytes,
                            size_t* bwd_workspace_bytes);

/* Forward.  X [N, d] in; out [N, d], g [N, d_ff] and u [N, d_ff] (the gate and
 * up pre-activations, rounded to bf16, kept for backward) and `saved` out.
 * H = silu(g) * u is formed from the bf16 g and u in the gate/up GEMM's
 * epilogue and lives only in the workspace. */
int lora_mlp_forward(const lora_mlp_shape* shape, const lora_mlp_weights* w,
                     const void* X, void* out, void* g, void* u, void* saved,
                     void* workspace, size_t workspace_bytes, void* stream);

/* Backward.  X, g, u, saved from the forward of the same X; dOut [N, d] in;
 * dX [N, d] and the six adapter gradients out.  silu and sigmoid are
 * recomputed from g and u in the epilogue of the dH GEMM. */
int lora_mlp_backward(const lora_mlp_shape* shape, const lora_mlp_weights* w,
                      const void* X, const void* g, const void* u, const void* saved,
                      const void* dOut, void* dX, const lora_mlp_grads* grads,
                      void* workspace, size_t workspace_bytes, void* stream);

/* Dequantise one block-int4 weight (format above) to bf16 [rows, cols];
 * cols a multiple of 64.  The same device routine the int4 path uses, exposed
 * so that its bits can be checked. */
int lora_mlp_dequant_int4(const void* packed, const void* scales, int64_t rows, int64_t cols,
                          void* w_bf16, void* stream);

/* Dequantise one block-FP8 weight (format above) to bf16 [rows, cols]; cols a
 * multiple of 64.  The same device routine the FP8 path uses, exposed so that
 * its bits can be checked. */
int lora_mlp_dequant_fp8(const void* codes, const void* scales, int64_t rows, int64_t cols,
                         void* w_bf16, void* stream);

/* Reads and clears the library's device status word for the current device:
 * 0, or LORA_MLP_ERR_DEVICE_TIMEOUT if any kernel gave up a bounded wait since
 * the last call.  Synchronises `stream`. */
int lora_mlp_device_status(void* stream, int* status);

/* The check every entry point applies to each pointer argument, on its own
 * (no launch): LORA_MLP_ERR_INVALID_ARG for NULL or for memory that is not
 * device or managed memory of the current device (pageable or page-locked
 * host memory, another device's memory, an address CUDA does not know);
 * LORA_MLP_ERR_MISALIGNED when p is not a multiple of `alignment` bytes
 * (0 or 1: no alignment check); else LORA_MLP_OK.  The entry points make it
 * after their other argument checks and before enqueueing anything, so a
 * host pointer is refused instead of reaching a kernel. */
int lora_mlp_check_pointer(const void* p, size_t alignment);

/* Human-readable name of a return code (static string). */
const char* lora_mlp_strerror(int code);

/* Kernel-time recording for measurement.  While enabled, every kernel launch
 * of the library is bracketed by a pair of CUDA events on its stream.
 * lora_mlp_timing_collect synchronises those events, writes up to `max`
 * (name, milliseconds) records in launch order, returns how many were
 * recorded in *count, and clears the record.  Names are static strings. */
typedef struct lora_mlp_kernel_time {
    const char* name;
    float ms;
} lora_mlp_kernel_time;
int lora_mlp_timing_enable(int enable);
int lora_mlp_timing_collect(lora_mlp_kernel_time* out, int max, int* count);

/* Number of kernels this library has launched in this process (all devices). */
int64_t lora_mlp_launch_count(void);

/* Test hook for the failure path.  While enabled, every GEMM launch makes its
 * epilogue wait on a barrier that nothing signals, and every barrier wait of
 * the library's kernels gives up after `wait_cycles` SM cycles (default
 * limit otherwise: 4e9 cycles, about 2 s).  The kernels then record
 * LORA_MLP_ERR_DEVICE_TIMEOUT for lora_mlp_device_status, wind down without
 * trapping (outputs are then garbage) and leave the CUDA context usable.
 * enable = 0 restores normal operation.  Process-wide; not for production. */
int lora_mlp_debug_force_timeout(int enable, int64_t wait_cycles);

/* ---------------------------------------------------------------------------
 * Forward pass that allocates nothing.  (The pages have no counterpart: this
 * entry point exists for how the library is called, not for the method.)
 *
 * Some callers cannot allocate device memory: a plugin running inside a host
 * framework that owns all device memory and forbids allocations behind its
 * allocator, a latency-critical loop where cudaMalloc's implicit device
 * synchronisation cannot be afforded, or a deployment whose memory is
 * budgeted up front.  For them this call does what lora_mlp_forward does
 * with the same arguments, but takes no workspace: its scratch is a fixed
 * device array of LORA_MLP_NOALLOC_SCRATCH_BYTES inside the library.  The
 * caller still passes X, out, g, u and saved.
 *  - Shapes whose forward workspace (lora_mlp_sizes) exceeds
 *    LORA_MLP_NOALLOC_SCRATCH_BYTES are rejected with
 *    LORA_MLP_ERR_WORKSPACE_TOO_SMALL before anything is enqueued.
 *  - Under CUDA's lazy module loading (CUDA_MODULE_LOADING=LAZY, the
 *    default of current CUDA releases) the array is reserved on a device when
 *    this entry point is first used there.  With CUDA_MODULE_LOADING=EAGER
 *    every context that loads this library reserves it, 64 MiB per device,
 *    whether or not the entry point is ever called.  Either way it is held
 *    until the process exits.  The first call on a device also looks up the
 *    array's device address and caches it; make it before any stream
 *    capture begins.
 *  - Every call on a device shares the one array.  Calls whose work may
 *    overlap on the GPU (unordered streams) race and corrupt each other's
 *    results: order them, e.g. on one stream.  Each call clears the part of
 *    the array that must start at zero, so nothing carries over between calls.
 *  - No cudaMalloc, cudaFree or allocating library routine is called. */
#define LORA_MLP_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
int lora_mlp_forward_noalloc(const lora_mlp_shape* shape, const lora_mlp_weights* w, const void* X, void* out,
                             void* g, void* u, void* saved, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LORA_MLP_H */
