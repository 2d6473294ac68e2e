/*
 * gtr_output_tail.h -- C ABI of the output tail of GTR's token mixer on B200
 * (sm_100a): the per-token epilogue between the gated linear attention and
 * the layer's output projection.
 *
 * Operation ("GTR: Gated Token Recurrence for Efficient Dense Prediction",
 * x-techcon article, section 算子: the operator benchmark leaves the fusion of
 * the operator's output tail out, and the pages do not define the tail).
 * Reading used: for every token t of the grid_h x grid_w grid and head h,
 *     n[t, h, j] = o[h, t, j] / sqrt(mean_j' o[h, t, j']^2 + eps) * w[h, j]
 *     y[t, h * d_v + j] = n[t, h, j] * SiLU(z[t, h * d_v + j]),
 *     SiLU(x) = x / (1 + e^{-x}),
 * i.e. a per-head RMS norm with weight, an output gate from a separate
 * projection z, and the heads merged channels-last.
 *
 * Tensors (device pointers, contiguous, row-major, 16-byte aligned):
 *   o  [B, H, grid_h, grid_w, d_v]   I/O dtype (the attention's output layout)
 *   z  [B, grid_h, grid_w, H * d_v]  I/O dtype
 *   w  [H, d_v]                      fp32
 *   y  [B, grid_h, grid_w, H * d_v]  I/O dtype, must not overlap o, z or w
 * dtype GTR_GLA_F16 or GTR_GLA_BF16; d_v 64 or 128; eps finite and >= 0.  The
 * norm, the gate and the product run in fp32; y is rounded once.  One launch,
 * no workspace; asynchronous and stream-ordered.
 *
 * Errors (codes of gtr_gla.h, all reported before anything is launched):
 * GTR_GLA_ERR_NULL, _SHAPE (B, H, grid <= 0, too many tokens, or eps < 0 or
 * not finite), _HEAD_DIM (d_v not 64 or 128), _DTYPE, _ALIGN, _ALIAS; _CUDA if
 * the launch fails.
 */
#ifndef GTR_OUTPUT_TAIL_H
#define GTR_OUTPUT_TAIL_H

#include <cuda_runtime.h>

#include "gtr_gla.h"

#ifdef __cplusplus
extern "C" {
#endif

int gtr_output_tail_fwd(const void *o, const void *z, const float *w, void *y, int B, int H,
                        int grid_h, int grid_w, int d_v, float eps, int dtype,
                        cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GTR_OUTPUT_TAIL_H */
