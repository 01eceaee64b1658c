/*
 * lora_rmsnorm.h — RMSNorm and the pre-norm LoRA MLP block for NVIDIA B200
 * (sm_100a): C ABI.
 *
 * The operation.  Per row x of a bf16 matrix [N, d] with a frozen gain
 * gamma [d]:
 *
 *   rstd = 1 / sqrt(mean(x^2) + eps),    y = x * rstd * gamma
 *   dx   = rstd * (dy*gamma - x_hat * mean(dy*gamma*x_hat)),   x_hat = x * rstd
 *
 * The RMS layer norm is one of the operations the pages name among the
 * hand-written forward + backward kernels ("Unsloth 深度分析报告",
 * nightvoyager.top, section 关键设计决策); its backward reuses the rstd the
 * forward cached instead of recomputing the mean of squares ("Unsloth支持哪些
 * 模型？主流LLM兼容性一览", pwwt.cn, section 4.2; section 2.6 quotes
 * rms_norm_eps = 1e-5).  gamma is frozen: no gradient is produced for it.
 *
 * The block is the pre-norm MLP of a transformer layer, out = MLP(RMSNorm(X)),
 * with the LoRA SwiGLU MLP of lora_mlp.h; the residual add stays with the
 * caller.  Its backward returns dX for the block input and the six adapter
 * gradients.
 *
 * Conventions are those of lora_mlp.h (return codes, bf16 row-major dense
 * tensors, 16-byte-aligned device pointers, caller-owned memory, work
 * enqueued on `stream`, nothing allocated, deterministic results, argument
 * errors detected on the host).  rstd is fp32 [N].  d must be a multiple of 8
 * (and satisfy the MLP's rules for the block); eps finite and >= 0.
 */
#ifndef LORA_RMSNORM_H
#define LORA_RMSNORM_H

#include "lora_mlp.h"

#ifdef __cplusplus
extern "C" {
#endif

/* y [N, d] = RMSNorm(x) * gamma; rstd [N] out (fp32).  One launch. */
int lora_rmsnorm_forward(int64_t N, int64_t d, float eps, const void* x, const void* gamma, void* y,
                         void* rstd, void* stream);

/* dx [N, d] for upstream dy [N, d], from x, gamma and the forward's rstd.
 * One launch. */
int lora_rmsnorm_backward(int64_t N, int64_t d, const void* x, const void* gamma, const void* rstd,
                          const void* dy, void* dx, void* stream);

/* Byte sizes for the block: forward and backward workspaces and `saved`
 * (the MLP's saved rank-r projections followed by rstd).  Host only. */
int lora_mlp_block_sizes(const lora_mlp_shape* shape, size_t* fwd_workspace_bytes,
                         size_t* bwd_workspace_bytes, size_t* saved_bytes);

/* Block forward.  X [N, d] (the block input, before the norm) in; out [N, d],
 * g, u [N, d_ff] and `saved` out.  The normalised input lives only in the
 * workspace. */
int lora_mlp_block_forward(const lora_mlp_shape* shape, const lora_mlp_weights* w, const void* gamma,
                           float eps, const void* X, void* out, void* g, void* u, void* saved,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Block backward.  X, g, u and `saved` from the forward of the same X; dOut
 * [N, d] in; dX [N, d] (gradient of the block input) and the adapter
 * gradients out.  The normalised input is recomputed from X and the saved
 * rstd (bit for bit the forward's), not stored between the passes. */
int lora_mlp_block_backward(const lora_mlp_shape* shape, const lora_mlp_weights* w, const void* gamma,
                            const void* X, const void* g, const void* u, const void* saved,
                            const void* dOut, void* dX, const lora_mlp_grads* grads, void* workspace,
                            size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * The block with the norm fused into the gate/up GEMM (bf16 frozen weights).
 *
 * With x_hat = diag(rstd) X diag(gamma), the gate and up projections are
 * x_hat W^T = diag(rstd) X (W diag(gamma))^T: once gamma is folded into Wg and
 * Wu (lora_mlp_block_fold_gamma, done once, since W and gamma are frozen), the
 * gate/up GEMM reads the raw rows X and its epilogue scales each row by rstd,
 * so the normalised rows are never written.  The rank-r path takes
 * A diag(gamma) (formed each call, A being trainable) the same way.  The
 * backward's dX GEMM on the folded weights yields dx_hat * gamma, which the
 * norm's backward maps to dX; the adapter gradients take the rstd and gamma
 * factors where their partial sums are finalised.  Results match the unfused block up
 * to the rounding of the folded weights and the order of the products.
 * Workspace and saved sizes: lora_mlp_block_sizes.
 */

/* Wg_folded = bf16_rne(Wg * gamma) and Wu_folded = bf16_rne(Wu * gamma), each
 * column e of Wg, Wu [d_ff, d] times gamma[e].  bf16 weights only
 * (LORA_MLP_ERR_INVALID_ARG otherwise).  One launch. */
int lora_mlp_block_fold_gamma(const lora_mlp_shape* shape, const lora_mlp_weights* w, const void* gamma,
                              void* Wg_folded, void* Wu_folded, void* stream);

/* Block forward with the folded weights: w_folded is w with Wg, Wu replaced
 * by the outputs of lora_mlp_block_fold_gamma (Wd and the adapters
 * unchanged); gamma, eps, X and the outputs as in lora_mlp_block_forward.
 * bf16 frozen weights only (LORA_MLP_ERR_INVALID_ARG otherwise).
 * Launches: rstd only, A diag(gamma) for both adapters, then the MLP's. */
int lora_mlp_block_forward_folded(const lora_mlp_shape* shape, const lora_mlp_weights* w_folded,
                                  const void* gamma, float eps, const void* X, void* out, void* g, void* u,
                                  void* saved, void* workspace, size_t workspace_bytes, void* stream);

/* Block backward with the folded weights; arguments as in
 * lora_mlp_block_backward, `saved` from lora_mlp_block_forward_folded; bf16
 * frozen weights only.  Launches: A diag(gamma) for both adapters, the
 * MLP's backward, then the norm's backward with gamma = 1. */
int lora_mlp_block_backward_folded(const lora_mlp_shape* shape, const lora_mlp_weights* w_folded,
                                   const void* gamma, const void* X, const void* g, const void* u,
                                   const void* saved, const void* dOut, void* dX, const lora_mlp_grads* grads,
                                   void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LORA_RMSNORM_H */
