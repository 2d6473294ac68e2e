/*
 * gtr_gemm.h -- C ABI of the library's own tensor-core GEMM on B200
 * (sm_100a), the dense projections of the GTR backbone layer and of the
 * Spatial SwiGLU block ("GTR: Gated Token Recurrence for Efficient Dense
 * Prediction", x-techcon article, section 架构: every layer's token mixer and
 * channel mixer project the patch tokens' channels):
 *     out[M, N] = in[M, K] . W[N, K]^T (+ bias[N]) (+ resid[M, N])
 * all row-major in the I/O dtype (GTR_GLA_F16 or GTR_GLA_BF16), products and
 * sums in fp32 on the tensor cores (tcgen05, accumulators in tensor memory),
 * bias and residual added in fp32 and the result rounded once.
 *
 * Arguments: device pointers, 16-byte aligned; bias and resid may be NULL;
 * resid may be out itself (out += in . W^T), otherwise out must not overlap
 * any input.  M > 0; N and K positive multiples of 8.  One launch, no
 * workspace; asynchronous and stream-ordered.  A device-side wait that gives
 * up is reported by gtr_gla_status as GTR_GLA_ERR_TIMEOUT.
 *
 * Errors (codes of gtr_gla.h, before anything is launched): GTR_GLA_ERR_NULL
 * (in, w or out NULL), _SHAPE, _DTYPE, _ALIGN, _ALIAS; _CUDA if the launch
 * fails.
 */
#ifndef GTR_GEMM_H
#define GTR_GEMM_H

#include <cuda_runtime.h>

#include "gtr_gla.h"

#ifdef __cplusplus
extern "C" {
#endif

int gtr_gemm_fwd(const void *in, const void *w, const void *bias, const void *resid, void *out,
                 long long M, int N, int K, int dtype, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GTR_GEMM_H */
