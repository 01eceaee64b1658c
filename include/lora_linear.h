/*
 * lora_linear.h — C ABI of a single LoRA-adapted linear projection for
 * NVIDIA B200 (sm_100a), forward and backward.
 *
 * The operation.  One frozen projection W with a LoRA adapter, the case of an
 * attention q/k/v/o projection, with the adapter's rank-r product fused into
 * the dense GEMM instead of run as separate small matmuls ("Unsloth 还是
 * AirLLM？一个炼丹，一个硬跑", blog.cn-res.vip, section 核心原理: matrix
 * multiplies and LoRA fused into single kernels).  With s = alpha / r and the
 * nn.Linear layout (W [out, in], A [r, in], B [out, r]):
 *
 *   Y = X (W + s B A)^T = X W^T + s (X A^T) B^T
 *
 * and, for an upstream gradient dY (W frozen, no gradient for it):
 *
 *   T = s dY B,   dX = dY W + T A,   dA = T^T X,   dB = s dY^T (X A^T).
 *
 * Conventions are those of lora_mlp.h (return codes, bf16 row-major dense
 * tensors, 16-byte-aligned device pointers, caller-owned memory, work
 * enqueued on `stream`, nothing allocated, deterministic results, argument
 * errors detected on the host before anything is enqueued).
 * Sizes: N >= 1; d_in, d_out multiples of 8 (d_in a multiple of 64 for int4
 * weights); r a multiple of 8 in [8, 128]; alpha finite.
 * Kernels: the same tcgen05 engines as the MLP.  Forward is two launches
 * (split-K rank-r product R = s X A^T; CTA-pair GEMM over K = d_in + r),
 * backward three (T and dB in one split-K launch; CTA-pair dX GEMM over
 * K = d_out + r; split-K token reduction for dA).  int4 weights are
 * dequantised inside the two CTA-pair GEMMs.
 */
#ifndef LORA_LINEAR_H
#define LORA_LINEAR_H

#include "lora_mlp.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct lora_linear_shape {
    int64_t N;             /* tokens (rows of X)                   */
    int64_t d_in;          /* input features                       */
    int64_t d_out;         /* output features                      */
    int64_t r;             /* LoRA rank                            */
    float alpha;           /* s = alpha / r                        */
    int32_t weight_format; /* LORA_MLP_WEIGHTS_BF16 or _INT4_B64   */
} lora_linear_shape;

/* Device pointers.  bf16 format: W bf16 [d_out, d_in], S = NULL.  int4
 * format (the block layout of lora_mlp.h): W uint8 [d_out, d_in/2] packed
 * codes, S fp16 [d_out, d_in/64] scales.  A bf16 [r, d_in]; B bf16 [d_out, r]. */
typedef struct lora_linear_weights {
    const void *W, *S, *A, *B;
} lora_linear_weights;

/* Byte sizes of the forward and backward scratch workspaces and of `saved`,
 * the buffer forward fills with s X A^T (opaque layout) for backward.  Pure
 * host function.  Any output pointer may be NULL. */
int lora_linear_sizes(const lora_linear_shape* shape, size_t* fwd_workspace_bytes,
                      size_t* bwd_workspace_bytes, size_t* saved_bytes);

/* Forward.  X [N, d_in] in; Y [N, d_out] and `saved` out. */
int lora_linear_forward(const lora_linear_shape* shape, const lora_linear_weights* w, const void* X,
                        void* Y, void* saved, void* workspace, size_t workspace_bytes, void* stream);

/* Backward.  X and `saved` from the forward of the same X; dY [N, d_out] in;
 * dX [N, d_in], dA [r, d_in] and dB [d_out, r] out (bf16). */
int lora_linear_backward(const lora_linear_shape* shape, const lora_linear_weights* w, const void* X,
                         const void* saved, const void* dY, void* dX, void* dA, void* dB,
                         void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LORA_LINEAR_H */
