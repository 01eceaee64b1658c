/*
 * lora_ce.h — chunked cross-entropy loss with logit scaling and softcapping
 * for NVIDIA B200 (sm_100a): C ABI.
 *
 * The operation.  Per row z of a bf16 logits matrix [N, V] with an integer
 * label y:
 *
 *   t    = s * z                        logit scaling (s = logit_scale)
 *   t    = c * tanh(t / c)   if c > 0   softcapping (c = softcap)
 *   lse  = log sum_j exp(t_j),  computed chunk by chunk over the vocabulary
 *          and combined as log sum_k exp(lse_k)
 *   loss = lse - t_y,   0 for a row whose label equals ignore_index
 *
 *   backward, for an upstream gradient dloss of each row:
 *   dz_j = dloss * (exp(t_j - lse) - [j == y]) * dt_j/dz_j,
 *   dt/dz = s, or s * (1 - (t/c)^2) with softcapping;  dz = 0 for ignored rows
 *
 * "Unsloth 深度分析报告" (nightvoyager.top), section 核心价值提炼 /
 * 创新之处, item 分块 Triton Cross Entropy Loss, describes this kernel: the
 * loss of a very large vocabulary (256K) is computed in chunks through the
 * separability of logsumexp, with softcapping (Gemma 2) and logit scaling
 * (Cohere).  The pages print no formula; the above is the plain definition
 * and its chain rule.
 *
 * Layout and types.  logits and dlogits are bf16 row-major with row stride
 * `ld` elements (ld >= V, a multiple of 8); labels are int64 [N]; loss, lse
 * and dloss are fp32 [N].  loss holds the per-row losses: a mean over the
 * rows that are not ignored is dloss = 1 / (number of such rows).
 *
 * Conventions (as lora_mlp.h): return 0 or a negative LORA_MLP_ERR_* code;
 * pointers are caller-owned device memory, logits/dlogits 16-byte aligned,
 * labels 8-byte and the fp32 arrays 4-byte aligned; all work is enqueued on
 * `stream` (a cudaStream_t, NULL = legacy default stream); nothing is
 * allocated or synchronised; argument errors are found on the host before
 * anything is enqueued; results are bitwise deterministic.  A label outside
 * [0, V) that is not ignore_index is a device-side finding: its row's loss
 * is NaN and lora_ce_device_status reports LORA_MLP_ERR_INVALID_ARG.
 */
#ifndef LORA_CE_H
#define LORA_CE_H

#include <stddef.h>
#include <stdint.h>

#include "lora_mlp.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    int64_t N;             /* rows (tokens), >= 1 */
    int64_t V;             /* logits per row (vocabulary size), >= 1 */
    int64_t ld;            /* row stride of logits and dlogits in elements: >= V, multiple of 8 */
    float logit_scale;     /* s, finite and non-zero (1 = no scaling) */
    float softcap;         /* c: 0 = no softcapping, else finite and > 0 */
    int64_t ignore_index;  /* label of rows that take no part (e.g. -100) */
} lora_ce_shape;

/* Workspace bytes of lora_ce_forward and lora_ce_forward_reduced (per-chunk
 * partial sums and per-row losses).  Host only. */
int lora_ce_sizes(const lora_ce_shape* shape, size_t* workspace_bytes);

/* loss [N] and lse [N] (the per-row log-sum-exp of the transformed logits,
 * kept for the backward) from logits [N, ld] and labels [N].  Two launches:
 * the chunk partials, then their in-order combination per row. */
int lora_ce_forward(const lora_ce_shape* shape, const void* logits, const int64_t* labels, float* loss,
                    float* lse, void* workspace, size_t workspace_bytes, void* stream);

/* dlogits [N, ld] (bf16; columns >= V untouched) for the upstream per-row
 * gradient dloss [N], from the logits, labels and the forward's lse.
 * dlogits may be the logits buffer itself (the gradient then overwrites the
 * logits in place).  One launch. */
int lora_ce_backward(const lora_ce_shape* shape, const void* logits, const int64_t* labels, const float* lse,
                     const float* dloss, void* dlogits, void* stream);

/* Reductions of the per-row losses into one loss. */
#define LORA_CE_REDUCTION_SUM 1  /* sum of the per-row losses                                   */
#define LORA_CE_REDUCTION_MEAN 2 /* that sum over the number of rows whose label is not
                                    ignore_index (over 1 when every row is ignored)              */

/* The loss reduced over the rows, computed in the library.  out[0] receives
 * the reduced loss; out[1] receives d out[0] / d loss_row for a row that
 * takes part: 1 for SUM, 1 / (rows taking part) for MEAN.  The per-row
 * losses stay in the workspace; lse [N] as in lora_ce_forward.  The sum runs
 * in fp64 in a fixed order, so the result is bitwise deterministic.  out is
 * fp32 [2], 8-byte aligned.  Three launches: the chunk partials, their
 * per-row combination, and the reduction (one CTA). */
int lora_ce_forward_reduced(const lora_ce_shape* shape, const void* logits, const int64_t* labels, int reduction,
                            float* out, float* lse, void* workspace, size_t workspace_bytes, void* stream);

/* dlogits [N, ld] for the upstream gradient dout[0] (device fp32 [1]) of the
 * loss lora_ce_forward_reduced returned: every row that takes part gets
 * dloss = dout[0] * fwd_out[1], fwd_out being that call's `out` [2];
 * ignored rows get zeros.  dlogits may be the logits buffer itself, as in
 * lora_ce_backward.  One launch. */
int lora_ce_backward_reduced(const lora_ce_shape* shape, const void* logits, const int64_t* labels,
                             const float* lse, const float* dout, const float* fwd_out, void* dlogits,
                             void* stream);

/* Reads and clears the device-side status of the cross-entropy kernels
 * (LORA_MLP_OK, or LORA_MLP_ERR_INVALID_ARG after an out-of-range label).
 * Synchronises `stream`. */
int lora_ce_device_status(void* stream, int* status);

#ifdef __cplusplus
}
#endif

#endif /* LORA_CE_H */
