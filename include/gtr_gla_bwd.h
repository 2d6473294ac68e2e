/*
 * gtr_gla_bwd.h -- C ABI of the backward pass of the chunkwise key-gated
 * linear attention on B200 (sm_100a, CUDA cores).
 *
 * Operation ("GTR: Gated Token Recurrence for Efficient Dense Prediction",
 * x-techcon article, section 算子: the operator there is inference-only, the
 * training used another library's kernel; this is the reverse mode of the
 * forward recurrence of gtr_gla.h): for the loss
 *     L = sum(d_out . out) + sum(d_final_state . final_state)
 * of the forward pass with the same q, k, v, log_alpha and direction, the
 * gradients dq = dL/dq, dk, dv and dlog_alpha = dL/dlog_alpha.  Reverse mode
 * through S_t = diag(alpha_t) S_{t-1} + k_t^T v_t, o_t = q_t S_t:
 *     G_t = dL/dS_t = q_t^T dO_t + diag(alpha_{t+1}) G_{t+1}  (G after the
 *           last token = d_final_state),
 *     dq_t = dO_t S_t^T,  dk_t = G_t v_t^T,  dv_t = k_t G_t,
 *     dlog_alpha_t = alpha_t . rowsum(G_t . S_{t-1}),
 * computed chunk by chunk (64 tokens) in fp32 with every gate factor <= 1.
 *
 * Tensors (device pointers, contiguous, 16-byte aligned; layouts of gtr_gla.h):
 *   q, k, dq, dk          [B, H, grid_h, grid_w, 64]  I/O dtype
 *   v, d_out, dv          [B, H, grid_h, grid_w, 64]  I/O dtype
 *   log_alpha, dlog_alpha [B, H, grid_h, grid_w, 64]  fp32
 *   d_final_state         [B, H, 64, 64]              fp32, or NULL (zero)
 * dtype GTR_GLA_F16, GTR_GLA_BF16 or GTR_GLA_F32; d_k = d_v = 64.  The
 * outputs must not overlap any input or each other.  workspace: at least
 * gtr_gla_bwd_workspace_size(...) bytes, 256-byte aligned (no zero-fill
 * needed), overlapping no tensor argument.  Asynchronous and stream-ordered.
 *
 * Errors (codes of gtr_gla.h, before anything is launched): GTR_GLA_ERR_NULL,
 * _SHAPE, _HEAD_DIM (d_k or d_v not 64), _DIRECTION, _ALIGN, _DTYPE,
 * _WORKSPACE, _ALIAS; _CUDA if a launch fails.
 */
#ifndef GTR_GLA_BWD_H
#define GTR_GLA_BWD_H

#include <cuda_runtime.h>
#include <stddef.h>

#include "gtr_gla.h"

#ifdef __cplusplus
extern "C" {
#endif

int gtr_gla_bwd(const void *q, const void *k, const void *v, const float *log_alpha, const void *d_out,
                const float *d_final_state, void *dq, void *dk, void *dv, float *dlog_alpha, int B, int H,
                int grid_h, int grid_w, int d_k, int d_v, int direction, int dtype, void *workspace,
                size_t workspace_bytes, cudaStream_t stream);

/* Workspace bytes of gtr_gla_bwd (0 for invalid sizes). */
size_t gtr_gla_bwd_workspace_size(int B, int H, int grid_h, int grid_w, int d_k, int d_v);

#ifdef __cplusplus
}
#endif

#endif /* GTR_GLA_BWD_H */
