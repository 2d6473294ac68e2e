/*
 * gtr_swiglu.h -- C ABI of the Spatial SwiGLU forward pass on B200 (sm_100a),
 * the channel mixer that follows the gated linear attention in every GTR
 * layer.
 *
 * Operation ("GTR: Gated Token Recurrence for Efficient Dense Prediction",
 * x-techcon article, section 架构 "architecture": a SwiGLU whose value branch
 * gets a 3 x 3 per-channel convolution so that neighbouring patches exchange
 * information).  Reading used (the pages give no formula): for every token of
 * the grid_h x grid_w patch grid,
 *     g = x W_g^T + b_g,   u = x W_u^T + b_u          (W_gu = [W_g; W_u])
 *     v = b_dw + DW3x3(u)   per-channel 3 x 3 cross-correlation over the grid,
 *                           stride 1, zero padding of one patch at the border:
 *                           v[y,x,f] = b_dw[f] + sum_{a,c=0..2} w_dw[f,a,c] u[y+a-1, x+c-1, f]
 *     h = SiLU(g) * v,      SiLU(z) = z / (1 + e^{-z})
 *     y = h W_d^T + b_d
 *
 * Tensors (device pointers, contiguous, row-major):
 *   x       [B, grid_h, grid_w, C]   I/O dtype (fp16 or bf16)
 *   w_gu    [2F, C]                  I/O dtype, rows 0..F-1 gate, F..2F-1 value
 *   b_gu    [2F]                     fp32
 *   w_dw    [F, 3, 3]                fp32
 *   b_dw    [F]                      fp32
 *   w_down  [C, F]                   I/O dtype
 *   b_down  [C]                      fp32
 *   y       [B, grid_h, grid_w, C]   I/O dtype, must not overlap any input
 * C and F must be multiples of 8 and every pointer 16-byte aligned.  The two
 * projections run on this library's tensor-core GEMM (gtr_gemm.h: tcgen05,
 * fp32 accumulation); b_g, b_u, b_dw, the depthwise convolution, the SiLU gate and
 * the product run in this library's own kernel, in fp32, between them; b_down
 * is rounded once to the I/O dtype and added in fp32 in the down projection's
 * epilogue.  The projected gate/value and the gated product are kept in the
 * workspace in the I/O dtype.
 *
 * Return codes are those of gtr_gla.h.  Calls are asynchronous and
 * stream-ordered.
 */
#ifndef GTR_SWIGLU_H
#define GTR_SWIGLU_H

#include <stddef.h>
#include <cuda_runtime.h>

#include "gtr_gla.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Workspace bytes gtr_swiglu_fwd needs (0 for invalid arguments). */
size_t gtr_swiglu_workspace_size(int B, int grid_h, int grid_w, int C, int F, int dtype);

/*
 * gtr_swiglu_fwd -- y = Spatial SwiGLU(x) as above.
 *   dtype:     GTR_GLA_F16 or GTR_GLA_BF16 (else GTR_GLA_ERR_DTYPE).
 *   workspace: device buffer of at least gtr_swiglu_workspace_size(...)
 *              bytes, 256-byte aligned, overlapping no tensor argument
 *              (GTR_GLA_ERR_ALIAS); calls sharing it must not overlap on
 *              the GPU.
 * Errors: GTR_GLA_ERR_NULL, _SHAPE (B, grid or C, F <= 0, or C, F not
 * multiples of 8), _DTYPE, _ALIGN, _ALIAS, _WORKSPACE, _CUDA; all but the
 * last are reported before anything is launched.  A wait inside the kernel
 * that runs out of time (it never should) is reported later, by
 * gtr_gla_status(), as GTR_GLA_ERR_TIMEOUT.
 */
int gtr_swiglu_fwd(const void *x, const void *w_gu, const float *b_gu, const float *w_dw,
                   const float *b_dw, const void *w_down, const float *b_down, void *y, int B,
                   int grid_h, int grid_w, int C, int F, int dtype, void *workspace,
                   size_t workspace_bytes, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GTR_SWIGLU_H */
