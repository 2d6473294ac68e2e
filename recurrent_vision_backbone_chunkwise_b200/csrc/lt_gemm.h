// lt_gemm.h -- the dense projections of the backbone layer and the Spatial
// SwiGLU block on cuBLASLt (internal to libgtr_gla.so, not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace gtr {

// cuBLASLt scratch that every lt_gemm call needs (caller-owned, 256-aligned).
constexpr size_t kLtWorkspace = 32u << 20;

// out[M, N] = in[M, K] . W[N, K]^T (+ bias[N]) (+ resid[M, N]), all row-major,
// fp16 or bf16 operands (dtype GTR_GLA_F16 / _BF16) with fp32 accumulation and
// one rounding to the output type.  bias is a vector in the output type;
// resid may be out itself (x += ...).  Plans are cached per device and shape.
int lt_gemm(int dev, int dtype, long long M, int N, int K, const void *in, const void *w, const void *bias,
            const void *resid, void *out, void *lt_ws, cudaStream_t st);

}  // namespace gtr
