// lt_gemm.cu -- cached cuBLASLt plans for the row-major projections
// out = in . W^T (+ bias) (+ resid) of the backbone layer and the Spatial
// SwiGLU block.
#include <cublasLt.h>

#include <map>
#include <mutex>
#include <tuple>

#include "gla_internal.h"
#include "lt_gemm.h"

namespace gtr {
namespace {

struct LtPlan {
    cublasLtMatmulDesc_t op = nullptr;
    cublasLtMatrixLayout_t a = nullptr, b = nullptr, d = nullptr;
    cublasLtMatmulAlgo_t algo;
    bool ok = false;
};

std::mutex g_lt_mu;
cublasLtHandle_t g_lt[64];
std::map<std::tuple<int, int, long long, int, int, bool, bool>, LtPlan> g_plans;

// In cuBLASLt's column-major terms: out^T (N x M) = W (N x K) . in^T (K x M),
// with W stored as a K x N column-major matrix (transposed in the op); the
// residual is the C operand with beta = 1.  Called with g_lt_mu held.
int lt_plan(int dev, int dtype, long long M, int N, int K, bool bias, bool resid, LtPlan **out) {
    if (!g_lt[dev] && cublasLtCreate(&g_lt[dev]) != CUBLAS_STATUS_SUCCESS) return GTR_GLA_ERR_CUDA;
    auto key = std::make_tuple(dev, dtype, M, N, K, bias, resid);
    auto it = g_plans.find(key);
    if (it != g_plans.end()) {
        *out = &it->second;
        return it->second.ok ? GTR_GLA_OK : GTR_GLA_ERR_CUDA;
    }
    LtPlan &pl = g_plans[key];
    const cudaDataType_t dt = dtype == GTR_GLA_BF16 ? CUDA_R_16BF : CUDA_R_16F;
    bool good = cublasLtMatmulDescCreate(&pl.op, CUBLAS_COMPUTE_32F, CUDA_R_32F) == CUBLAS_STATUS_SUCCESS;
    const cublasOperation_t opT = CUBLAS_OP_T, opN = CUBLAS_OP_N;
    good = good && cublasLtMatmulDescSetAttribute(pl.op, CUBLASLT_MATMUL_DESC_TRANSA, &opT, sizeof(opT)) ==
                       CUBLAS_STATUS_SUCCESS;
    good = good && cublasLtMatmulDescSetAttribute(pl.op, CUBLASLT_MATMUL_DESC_TRANSB, &opN, sizeof(opN)) ==
                       CUBLAS_STATUS_SUCCESS;
    if (bias) {  // bias vector in the output type
        const cublasLtEpilogue_t epi = CUBLASLT_EPILOGUE_BIAS;
        good = good && cublasLtMatmulDescSetAttribute(pl.op, CUBLASLT_MATMUL_DESC_EPILOGUE, &epi, sizeof(epi)) ==
                           CUBLAS_STATUS_SUCCESS;
    }
    good = good && cublasLtMatrixLayoutCreate(&pl.a, dt, K, N, K) == CUBLAS_STATUS_SUCCESS;
    good = good && cublasLtMatrixLayoutCreate(&pl.b, dt, K, M, K) == CUBLAS_STATUS_SUCCESS;
    good = good && cublasLtMatrixLayoutCreate(&pl.d, dt, N, M, N) == CUBLAS_STATUS_SUCCESS;
    cublasLtMatmulPreference_t pref = nullptr;
    good = good && cublasLtMatmulPreferenceCreate(&pref) == CUBLAS_STATUS_SUCCESS;
    const size_t wsb = kLtWorkspace;
    good = good && cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &wsb,
                                                        sizeof(wsb)) == CUBLAS_STATUS_SUCCESS;
    cublasLtMatmulHeuristicResult_t res;
    int n = 0;
    good = good && cublasLtMatmulAlgoGetHeuristic(g_lt[dev], pl.op, pl.a, pl.b, pl.d, pl.d, pref, 1, &res, &n) ==
                       CUBLAS_STATUS_SUCCESS &&
           n > 0;
    if (pref) cublasLtMatmulPreferenceDestroy(pref);
    if (good) pl.algo = res.algo;
    pl.ok = good;
    *out = &pl;
    return good ? GTR_GLA_OK : GTR_GLA_ERR_CUDA;
}

}  // namespace

int lt_gemm(int dev, int dtype, long long M, int N, int K, const void *in, const void *w, const void *bias,
            const void *resid, void *out, void *lt_ws, cudaStream_t st) {
    if (dev < 0 || dev >= 64) return GTR_GLA_ERR_CUDA;
    // one lock across the plan lookup, the bias pointer (an attribute of the
    // shared descriptor) and the enqueue
    std::lock_guard<std::mutex> lock(g_lt_mu);
    LtPlan *pl;
    int rc = lt_plan(dev, dtype, M, N, K, bias != nullptr, resid != nullptr, &pl);
    if (rc) return rc;
    if (bias && cublasLtMatmulDescSetAttribute(pl->op, CUBLASLT_MATMUL_DESC_BIAS_POINTER, &bias,
                                               sizeof(bias)) != CUBLAS_STATUS_SUCCESS)
        return GTR_GLA_ERR_CUDA;
    const float one = 1.f, zero = 0.f;
    return cublasLtMatmul(g_lt[dev], pl->op, &one, w, pl->a, in, pl->b, resid ? &one : &zero,
                          resid ? resid : out, pl->d, out, pl->d, &pl->algo, lt_ws, kLtWorkspace,
                          st) == CUBLAS_STATUS_SUCCESS
               ? GTR_GLA_OK
               : GTR_GLA_ERR_CUDA;
}

}  // namespace gtr
