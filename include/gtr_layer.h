/*
 * gtr_layer.h -- C ABI of the GTR backbone on B200 (sm_100a): one layer (the
 * GLA token mixer and the Spatial SwiGLU channel mixer with pre-norm
 * residuals) and the direction-cycled stack of layers.
 *
 * Operation ("GTR: Gated Token Recurrence for Efficient Dense Prediction",
 * x-techcon article, section 架构): 12 layers on the fixed patch grid, each a
 * GLA for long-range context followed by a Spatial SwiGLU for neighbouring
 * patches, the scan direction cycling L->R, R->L, T->B, B->T over consecutive
 * layers, the grid order restored after every scan.  The pages give no
 * projections, norms or residual layout; the reading used is the pre-norm
 * residual layer of a vision transformer with the attention replaced:
 *     x1 = LN1(x);  [q | k | v | a | z] = x1 W_proj^T,
 *         W_proj = [W_q; W_k; W_v; W_a; W_z]   ([5C, C])
 *     k = k / 8 (1 / sqrt(64));  log_alpha = logsigmoid(a + b_a) / 16
 *     o = GLA(q, k, v, log_alpha, direction)         (chunk 64)
 *     x = x + OutputTail(o, z, w_n) W_o^T            (eps 1e-5; both in one
 *                                                     gtr_gla_fwd_tail call)
 *     x = x + SpatialSwiGLU(LN2(x))                  (gtr_swiglu.h)
 * with heads of 64 (H = C / 64), LayerNorm eps 1e-6 with weight and bias, and
 * in the stack direction = layer index mod 4.  The patch embedding and the
 * task head are not part of it.
 *
 * Weights (device pointers, contiguous, 16-byte aligned; the matrices in the
 * I/O dtype, the vectors fp32): see GtrLayerWeights.  Activations x
 * [B, grid_h, grid_w, C] in the I/O dtype (GTR_GLA_F16 or _BF16), updated in
 * place.  C a multiple of 64, at most 2048; F a multiple of 8 (the stack
 * uses F = 4 C, but any F is accepted).
 *
 * Workspace: caller-owned device memory of gtr_layer_workspace_size bytes,
 * 256-byte aligned and zero-filled before its first use (it holds the GLA's
 * look-back header, which every call leaves zero again), for the intermediate
 * activations, the GLA's scratch and the GEMM scratch; calls sharing one must
 * be stream-ordered.
 * Calls are asynchronous and stream-ordered; device-side GLA errors are read
 * by gtr_gla_status.  Every step runs in this library's kernels (the
 * projections on its tensor-core GEMM, gtr_gemm.h).
 *
 * Errors (codes of gtr_gla.h, reported before anything is launched):
 * GTR_GLA_ERR_NULL (x, w or any weight pointer NULL), _SHAPE (B, grid <= 0,
 * C not a positive multiple of 64 or above 2048, F <= 0 or not a multiple of
 * 8, too many tokens, n_layers < 1), _DIRECTION, _DTYPE, _ALIGN (a pointer not
 * 16-byte aligned), _WORKSPACE (NULL, too small or not 256-byte aligned),
 * _ALIAS (x, the bytes of the workspace the call uses and the weights do not
 * all stay apart; weights may share memory among themselves), _CUDA (a
 * launch failed).
 */
#ifndef GTR_LAYER_H
#define GTR_LAYER_H

#include <cuda_runtime.h>
#include <stddef.h>

#include "gtr_gla.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    const float *ln1_w, *ln1_b;  /* [C] first LayerNorm */
    const void *w_proj;          /* [5C, C] W_q, W_k, W_v, W_a, W_z stacked */
    const float *b_a;            /* [C] gate bias */
    const float *w_n;            /* [H, 64] output-tail norm weights */
    const void *w_o;             /* [C, C] output projection */
    const float *ln2_w, *ln2_b;  /* [C] second LayerNorm */
    const void *w_gu;            /* [2F, C] SwiGLU gate / value projection */
    const float *b_gu;           /* [2F] */
    const float *w_dw;           /* [F, 3, 3] depthwise taps of the value branch */
    const float *b_dw;           /* [F] */
    const void *w_down;          /* [C, F] down projection */
    const float *b_down;         /* [C] */
} GtrLayerWeights;

/* Workspace bytes of one layer (and of the stack) on this shape; 0 if the
 * sizes are invalid. */
size_t gtr_layer_workspace_size(int B, int grid_h, int grid_w, int C, int F, int dtype);

/* One layer, x updated in place. */
int gtr_layer_fwd(void *x, const GtrLayerWeights *w, int B, int grid_h, int grid_w, int C, int F,
                  int direction, int dtype, void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* n_layers layers (host array of weight structs), layer l scanning in
 * direction l mod 4; x updated in place. */
int gtr_backbone_fwd(void *x, const GtrLayerWeights *layers, int n_layers, int B, int grid_h, int grid_w,
                     int C, int F, int dtype, void *workspace, size_t workspace_bytes, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GTR_LAYER_H */
