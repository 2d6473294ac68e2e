// swiglu.cu -- Spatial SwiGLU forward (GTR's channel mixer) on sm_100a:
// the two dense projections as cuBLASLt GEMMs on the tensor cores, and one
// kernel of this library between them for everything that is not a GEMM:
// the projection biases, the 3 x 3 depthwise convolution of the value branch
// over the patch grid, the SiLU gate and the product.
//
// "GTR: Gated Token Recurrence for Efficient Dense Prediction", x-techcon
// article, section 架构: a SwiGLU whose value branch gets a 3 x 3 per-channel
// convolution, so that neighbouring patches exchange information directly.
#include <cublasLt.h>

#include <map>
#include <mutex>
#include <tuple>

#include "../../include/gtr_swiglu.h"
#include "gla_common.cuh"
#include "gla_internal.h"

namespace gtr {
namespace {

template <typename T> struct Pair;
template <> struct Pair<__half> {
    static __device__ __forceinline__ float2 unpack(uint32_t w) {
        return __half22float2(*reinterpret_cast<__half2 *>(&w));
    }
    static __device__ __forceinline__ uint32_t pack(float a, float b) {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&h);
    }
};
template <> struct Pair<__nv_bfloat16> {
    static __device__ __forceinline__ float2 unpack(uint32_t w) {
        return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&w));
    }
    static __device__ __forceinline__ uint32_t pack(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&h);
    }
};

constexpr int kPairs = 32;   // channel pairs per block (64 channels)
constexpr int kTokens = 8;   // consecutive tokens of one grid row per block

// h[m, f] = SiLU(g) * (b_dw[f] + sum_{a,c} w_dw[f,a,c] u[y+a-1, x+c-1, f]) with
// g = gu[m, f] + b_gu[f] and u = gu[., F + f] + b_gu[F + f] (0 off the grid).
// One thread per (token, channel pair); a block covers 64 channels of 8
// consecutive tokens of one grid row, so the 3 x 3 neighbourhoods of its
// tokens overlap in L1.  All arithmetic in fp32.
template <typename T>
__global__ void __launch_bounds__(kPairs * kTokens) swiglu_dw_gate_kernel(
    const T *__restrict__ gu, const float *__restrict__ b_gu, const float *__restrict__ w_dw,
    const float *__restrict__ b_dw, T *__restrict__ h, int gh, int gw, int F) {
    __shared__ float s_w[2 * kPairs][9];
    const int f0 = blockIdx.y * 2 * kPairs;
    const int tx = threadIdx.x, ty = threadIdx.y, t = ty * kPairs + tx;
    for (int e = t; e < 2 * kPairs * 9; e += kPairs * kTokens) {
        const int c = e / 9;
        s_w[c][e % 9] = (f0 + c < F) ? w_dw[(size_t)(f0 + c) * 9 + e % 9] : 0.f;
    }
    __syncthreads();
    const int f = f0 + 2 * tx;
    const int xblocks = (gw + kTokens - 1) / kTokens;
    const int row = blockIdx.x / xblocks;  // b * gh + y
    const int x = (blockIdx.x % xblocks) * kTokens + ty;
    if (f >= F || x >= gw) return;
    const int b = row / gh, y = row % gh;
    const size_t ld = 2 * (size_t)F;  // row length of gu in elements
    const size_t m = (size_t)row * gw + x;
    const float2 bg = make_float2(b_gu[f], b_gu[f + 1]);
    const float2 bu = make_float2(b_gu[F + f], b_gu[F + f + 1]);
    float2 v = make_float2(b_dw[f], b_dw[f + 1]);
#pragma unroll
    for (int a = 0; a < 3; ++a) {
        const int yy = y + a - 1;
        if (yy < 0 || yy >= gh) continue;
#pragma unroll
        for (int c = 0; c < 3; ++c) {
            const int xx = x + c - 1;
            if (xx < 0 || xx >= gw) continue;
            const size_t mm = ((size_t)b * gh + yy) * gw + xx;
            const float2 u = Pair<T>::unpack(*reinterpret_cast<const uint32_t *>(gu + mm * ld + F + f));
            v.x = fmaf(s_w[2 * tx][3 * a + c], u.x + bu.x, v.x);
            v.y = fmaf(s_w[2 * tx + 1][3 * a + c], u.y + bu.y, v.y);
        }
    }
    const float2 g0 = Pair<T>::unpack(*reinterpret_cast<const uint32_t *>(gu + m * ld + f));
    const float gx = g0.x + bg.x, gy = g0.y + bg.y;
    const float hx = gx / (1.f + __expf(-gx)) * v.x;
    const float hy = gy / (1.f + __expf(-gy)) * v.y;
    *reinterpret_cast<uint32_t *>(h + m * (size_t)F + f) = Pair<T>::pack(hx, hy);
}

// y[m, c] += bias[c] (used only when cuBLASLt takes no fp32 bias in its
// epilogue for these types).
template <typename T>
__global__ void add_bias_kernel(T *y, const float *bias, size_t M, int C) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;  // pair index
    if (i >= M * (size_t)C / 2) return;
    const int c = (int)((2 * i) % C);
    uint32_t *p = reinterpret_cast<uint32_t *>(y) + i;
    const float2 o = Pair<T>::unpack(*p);
    *p = Pair<T>::pack(o.x + bias[c], o.y + bias[c + 1]);
}

// ---------------------------------------------------------------- cuBLASLt

constexpr size_t kLtWorkspace = 32u << 20;

struct LtPlan {
    cublasLtMatmulDesc_t op = nullptr;
    cublasLtMatrixLayout_t a = nullptr, b = nullptr, d = nullptr;
    cublasLtMatmulAlgo_t algo;
    bool ok = false;
};

std::mutex g_lt_mu;
cublasLtHandle_t g_lt[64];
std::map<std::tuple<int, int, long long, int, int, bool>, LtPlan> g_plans;

// out[M, N] (row-major) = in[M, K] (row-major) . W[N, K]^T (+ bias[N], fp32).
// In cuBLASLt's column-major terms: out^T (N x M) = W (N x K) . in^T (K x M),
// with W stored as a K x N column-major matrix (transposed in the op).
// Called with g_lt_mu held.
int lt_plan(int dev, int dtype, long long M, int N, int K, bool bias, LtPlan **out) {
    if (!g_lt[dev] && cublasLtCreate(&g_lt[dev]) != CUBLAS_STATUS_SUCCESS) return GTR_GLA_ERR_CUDA;
    auto key = std::make_tuple(dev, dtype, M, N, K, bias);
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
    if (bias) {
        const cublasLtEpilogue_t epi = CUBLASLT_EPILOGUE_BIAS;
        const cudaDataType_t bt = CUDA_R_32F;
        good = good && cublasLtMatmulDescSetAttribute(pl.op, CUBLASLT_MATMUL_DESC_EPILOGUE, &epi, sizeof(epi)) ==
                           CUBLAS_STATUS_SUCCESS;
        good = good && cublasLtMatmulDescSetAttribute(pl.op, CUBLASLT_MATMUL_DESC_BIAS_DATA_TYPE, &bt,
                                                      sizeof(bt)) == CUBLAS_STATUS_SUCCESS;
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

int lt_gemm(int dev, int dtype, long long M, int N, int K, const void *in, const void *w, const float *bias,
            void *out, void *lt_ws, cudaStream_t st) {
    // one lock across the plan lookup, the bias pointer (an attribute of the
    // shared descriptor) and the enqueue
    std::lock_guard<std::mutex> lock(g_lt_mu);
    LtPlan *pl;
    int rc = lt_plan(dev, dtype, M, N, K, bias != nullptr, &pl);
    if (rc) return rc;
    if (bias && cublasLtMatmulDescSetAttribute(pl->op, CUBLASLT_MATMUL_DESC_BIAS_POINTER, &bias,
                                               sizeof(bias)) != CUBLAS_STATUS_SUCCESS)
        return GTR_GLA_ERR_CUDA;
    const float one = 1.f, zero = 0.f;
    return cublasLtMatmul(g_lt[dev], pl->op, &one, w, pl->a, in, pl->b, &zero, out, pl->d, out, pl->d,
                          &pl->algo, lt_ws, kLtWorkspace, st) == CUBLAS_STATUS_SUCCESS
               ? GTR_GLA_OK
               : GTR_GLA_ERR_CUDA;
}

struct SwLayout {
    size_t gu, h, lt, total;
};

SwLayout sw_layout(long long M, int F, size_t es) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    SwLayout l;
    l.gu = 0;
    l.h = up((size_t)M * 2 * F * es);
    l.lt = up(l.h + (size_t)M * F * es);
    l.total = l.lt + kLtWorkspace;
    return l;
}

bool overlap(const void *a, size_t na, const void *b, size_t nb) {
    const char *pa = (const char *)a, *pb = (const char *)b;
    return pa < pb + nb && pb < pa + na;
}

int sw_validate_shape(int B, int gh, int gw, int C, int F, int dtype) {
    if (B <= 0 || gh <= 0 || gw <= 0 || C <= 0 || F <= 0 || C % 8 || F % 8) return GTR_GLA_ERR_SHAPE;
    if ((long long)B * gh * gw > (1LL << 28) || C > 65536 || F > 65536) return GTR_GLA_ERR_SHAPE;
    if (dtype != GTR_GLA_F16 && dtype != GTR_GLA_BF16) return GTR_GLA_ERR_DTYPE;
    return GTR_GLA_OK;
}

}  // namespace
}  // namespace gtr

using namespace gtr;

extern "C" size_t gtr_swiglu_workspace_size(int B, int grid_h, int grid_w, int C, int F, int dtype) {
    if (sw_validate_shape(B, grid_h, grid_w, C, F, dtype)) return 0;
    return sw_layout((long long)B * grid_h * grid_w, F, 2).total;
}

extern "C" int gtr_swiglu_fwd(const void *x, const void *w_gu, const float *b_gu, const float *w_dw,
                              const float *b_dw, const void *w_down, const float *b_down, void *y, int B,
                              int grid_h, int grid_w, int C, int F, int dtype, void *workspace,
                              size_t workspace_bytes, cudaStream_t stream) {
    if (!x || !w_gu || !b_gu || !w_dw || !b_dw || !w_down || !b_down || !y) return GTR_GLA_ERR_NULL;
    int rc = sw_validate_shape(B, grid_h, grid_w, C, F, dtype);
    if (rc) return rc;
    const void *ptrs[] = {x, w_gu, b_gu, w_dw, b_dw, w_down, b_down, y, workspace};
    for (const void *p : ptrs)
        if (((uintptr_t)p & 15u) != 0) return GTR_GLA_ERR_ALIGN;
    const long long M = (long long)B * grid_h * grid_w;
    const size_t es = 2;
    const size_t ny = (size_t)M * C * es;
    if (overlap(y, ny, x, ny) || overlap(y, ny, w_gu, (size_t)2 * F * C * es) ||
        overlap(y, ny, w_down, (size_t)C * F * es) || overlap(y, ny, b_gu, (size_t)2 * F * 4) ||
        overlap(y, ny, w_dw, (size_t)F * 36) || overlap(y, ny, b_dw, (size_t)F * 4) ||
        overlap(y, ny, b_down, (size_t)C * 4))
        return GTR_GLA_ERR_ALIAS;
    const SwLayout l = sw_layout(M, F, es);
    if (!workspace || workspace_bytes < l.total || ((uintptr_t)workspace & 255u)) return GTR_GLA_ERR_WORKSPACE;
    if (overlap(y, ny, workspace, l.total)) return GTR_GLA_ERR_ALIAS;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GTR_GLA_ERR_CUDA;
    char *ws = static_cast<char *>(workspace);
    void *gu = ws + l.gu, *h = ws + l.h, *lt_ws = ws + l.lt;
    // 1. [g | u] without biases (the kernel adds them in fp32)
    rc = lt_gemm(dev, dtype, M, 2 * F, C, x, w_gu, nullptr, gu, lt_ws, stream);
    if (rc) return rc;
    // 2. biases, depthwise 3 x 3 on the value branch, SiLU gate, product
    const int xblocks = (grid_w + kTokens - 1) / kTokens;
    const dim3 grid((unsigned)((long long)B * grid_h * xblocks), (F + 2 * kPairs - 1) / (2 * kPairs));
    const dim3 block(kPairs, kTokens);
    if (dtype == GTR_GLA_BF16)
        swiglu_dw_gate_kernel<__nv_bfloat16><<<grid, block, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(gu), b_gu, w_dw, b_dw, static_cast<__nv_bfloat16 *>(h), grid_h,
            grid_w, F);
    else
        swiglu_dw_gate_kernel<__half><<<grid, block, 0, stream>>>(static_cast<const __half *>(gu), b_gu, w_dw,
                                                                   b_dw, static_cast<__half *>(h), grid_h,
                                                                   grid_w, F);
    note_launch();
    if (cudaPeekAtLastError() != cudaSuccess) return GTR_GLA_ERR_CUDA;
    // 3. y = h W_d^T + b_d (bias in the GEMM's epilogue when cuBLASLt takes an
    //    fp32 bias for these types, else one pass of this library)
    rc = lt_gemm(dev, dtype, M, C, F, h, w_down, b_down, y, lt_ws, stream);
    if (rc) {
        rc = lt_gemm(dev, dtype, M, C, F, h, w_down, nullptr, y, lt_ws, stream);
        if (rc) return rc;
        const size_t pairs = (size_t)M * C / 2;
        const unsigned blocks = (unsigned)((pairs + 255) / 256);
        if (dtype == GTR_GLA_BF16)
            add_bias_kernel<__nv_bfloat16><<<blocks, 256, 0, stream>>>(static_cast<__nv_bfloat16 *>(y), b_down,
                                                                       (size_t)M, C);
        else
            add_bias_kernel<__half><<<blocks, 256, 0, stream>>>(static_cast<__half *>(y), b_down, (size_t)M, C);
        note_launch();
        if (cudaPeekAtLastError() != cudaSuccess) return GTR_GLA_ERR_CUDA;
    }
    return GTR_GLA_OK;
}
