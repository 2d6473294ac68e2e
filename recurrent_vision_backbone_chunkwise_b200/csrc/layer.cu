// layer.cu -- one GTR backbone layer and the direction-cycled stack on
// sm_100a: LayerNorm, the fused q/k/v/gate/output-gate projection, the head
// split with the key scale and the gate activation, the fused GLA kernel with
// the output tail, the output projection with the residual as the GEMM's C
// operand, LayerNorm and the Spatial SwiGLU block whose down projection adds
// its residual the same way.  The output tail runs inside the GLA kernel's
// stores (gtr_gla_fwd_tail).
//
// "GTR: Gated Token Recurrence for Efficient Dense Prediction", x-techcon
// article, section 架构 (12 layers of GLA + Spatial SwiGLU on the patch grid,
// the scan direction cycling over consecutive layers).
#include "../../include/gtr_layer.h"
#include "../../include/gtr_swiglu.h"
#include "gla_common.cuh"
#include "gla_internal.h"
#include "io_pack.cuh"

namespace gtr {
namespace {

constexpr float kLnEps = 1e-6f, kTailEps = 1e-5f;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// y = (x - mean) / sqrt(var + eps) * w + b over the C channels of each token;
// one warp per token (grid-stride over whole warps), 16-byte chunks, NC chunks
// per lane (C <= 256 * NC), two passes over registers for the variance.
template <typename T, int NC>
__global__ void __launch_bounds__(256) layer_norm_kernel(const T *__restrict__ x, const float *__restrict__ w,
                                                         const float *__restrict__ b, T *__restrict__ y,
                                                         long long M, int C, float eps) {
    const int lane = threadIdx.x & 31;
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long m = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); m < M; m += nwarps) {
        const T *xr = x + m * C;
        float2 v[NC][4];
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const int idx = (lane + 32 * c) * 8;
            if (idx < C) {
                unpack8<T>(*reinterpret_cast<const uint4 *>(xr + idx), v[c]);
#pragma unroll
                for (int e = 0; e < 4; ++e) s += v[c][e].x + v[c][e].y;
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) v[c][e] = make_float2(0.f, 0.f);
            }
        }
        const float mean = warp_sum(s) / C;
        float q = 0.f;
#pragma unroll
        for (int c = 0; c < NC; ++c)
            if ((lane + 32 * c) * 8 < C)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float dx = v[c][e].x - mean, dy = v[c][e].y - mean;
                    q = fmaf(dx, dx, fmaf(dy, dy, q));
                }
        const float r = rsqrtf(warp_sum(q) / C + eps);
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const int idx = (lane + 32 * c) * 8;
            if (idx < C) {
                const float4 w0 = __ldg(reinterpret_cast<const float4 *>(w + idx));
                const float4 w1 = __ldg(reinterpret_cast<const float4 *>(w + idx + 4));
                const float4 b0 = __ldg(reinterpret_cast<const float4 *>(b + idx));
                const float4 b1 = __ldg(reinterpret_cast<const float4 *>(b + idx + 4));
                const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                uint32_t o[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    o[e] = Pair<T>::pack(fmaf((v[c][e].x - mean) * r, wv[2 * e], bv[2 * e]),
                                         fmaf((v[c][e].y - mean) * r, wv[2 * e + 1], bv[2 * e + 1]));
                *reinterpret_cast<uint4 *>(y + m * C + idx) = make_uint4(o[0], o[1], o[2], o[3]);
            }
        }
    }
}

// log(sigmoid(a)) = min(a, 0) - log(1 + e^{-|a|}), without overflow.
__device__ __forceinline__ float log_sigmoid(float a) { return fminf(a, 0.f) - log1pf(expf(-fabsf(a))); }

// P [M, 5C] = [q | k | v | a | z] per token -> q, k / 8, v in [B, H, N, 64]
// (the attention's layout), log_alpha = log_sigmoid(a + b_a) / 16 in fp32 in
// the same layout, z [M, C] contiguous.  One thread per 8 channels.
template <typename T>
__global__ void __launch_bounds__(256) split_heads_kernel(const T *__restrict__ P, const float *__restrict__ b_a,
                                                          T *__restrict__ q, T *__restrict__ k, T *__restrict__ v,
                                                          float *__restrict__ la, T *__restrict__ z, long long M,
                                                          long long N, int C) {
    const int H = C / 64, row8 = 5 * C / 8;
    const long long total = M * row8;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long m = i / row8;
        const int c = (int)(i % row8) * 8;
        const int part = c / C, within = c % C;
        const uint4 raw = *reinterpret_cast<const uint4 *>(P + m * 5 * C + c);
        if (part == 4) {
            *reinterpret_cast<uint4 *>(z + m * C + within) = raw;
            continue;
        }
        const long long bimg = m / N, n = m % N;
        const int h = within / 64, d0 = within % 64;
        const size_t dst = ((size_t)(bimg * H + h) * N + n) * 64 + d0;
        if (part == 0) {
            *reinterpret_cast<uint4 *>(q + dst) = raw;
        } else if (part == 2) {
            *reinterpret_cast<uint4 *>(v + dst) = raw;
        } else {
            float2 f[4];
            unpack8<T>(raw, f);
            if (part == 1) {
                uint32_t o[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) o[e] = Pair<T>::pack(0.125f * f[e].x, 0.125f * f[e].y);
                *reinterpret_cast<uint4 *>(k + dst) = make_uint4(o[0], o[1], o[2], o[3]);
            } else {
                float out[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    out[2 * e] = 0.0625f * log_sigmoid(f[e].x + b_a[within + 2 * e]);
                    out[2 * e + 1] = 0.0625f * log_sigmoid(f[e].y + b_a[within + 2 * e + 1]);
                }
                *reinterpret_cast<float4 *>(la + dst) = make_float4(out[0], out[1], out[2], out[3]);
                *reinterpret_cast<float4 *>(la + dst + 4) = make_float4(out[4], out[5], out[6], out[7]);
            }
        }
    }
}

// ------------------------------------------------------------- workspace
struct Layout {
    size_t x1, P, q, k, v, la, z, t, gla, sw, total;
    size_t gla_bytes, sw_bytes;
};

Layout layout(int B, int gh, int gw, int C, int F, int dtype) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t M = (size_t)B * gh * gw, e = 2, act = M * C * e;
    Layout l;
    l.x1 = 0;
    l.P = up(l.x1 + act);
    l.q = up(l.P + 5 * act);
    l.k = up(l.q + act);
    l.v = up(l.k + act);
    l.la = up(l.v + act);
    l.z = up(l.la + M * C * 4);
    l.t = up(l.z + act);
    l.gla_bytes = gtr_gla_tail_workspace_size(B, C / 64, gh, gw, 64, 64, dtype);
    l.sw_bytes = gtr_swiglu_workspace_size(B, gh, gw, C, F, dtype);
    l.gla = up(l.t + act);
    l.sw = up(l.gla + l.gla_bytes);
    l.total = up(l.sw + l.sw_bytes);
    return l;
}

unsigned grid_for(long long work, int per_block) {
    long long g = (work + per_block - 1) / per_block;
    if (g > 148LL * 16) g = 148LL * 16;
    return (unsigned)(g < 1 ? 1 : g);
}

template <typename T>
int layer_norm(const T *x, const float *w, const float *b, T *y, long long M, int C, cudaStream_t st) {
    const unsigned grid = grid_for(M, 8);
    if (C <= 256)
        layer_norm_kernel<T, 1><<<grid, 256, 0, st>>>(x, w, b, y, M, C, kLnEps);
    else if (C <= 512)
        layer_norm_kernel<T, 2><<<grid, 256, 0, st>>>(x, w, b, y, M, C, kLnEps);
    else if (C <= 1024)
        layer_norm_kernel<T, 4><<<grid, 256, 0, st>>>(x, w, b, y, M, C, kLnEps);
    else
        layer_norm_kernel<T, 8><<<grid, 256, 0, st>>>(x, w, b, y, M, C, kLnEps);
    note_launch();
    return cudaPeekAtLastError() == cudaSuccess ? GTR_GLA_OK : GTR_GLA_ERR_CUDA;
}

template <typename T>
int layer_impl(T *x, const GtrLayerWeights *w, int B, int gh, int gw, int C, int F, int dir, int dtype, char *ws,
               const Layout &l, cudaStream_t st) {
    const long long M = (long long)B * gh * gw, N = (long long)gh * gw;
    const int H = C / 64;
    T *x1 = reinterpret_cast<T *>(ws + l.x1), *P = reinterpret_cast<T *>(ws + l.P);
    T *q = reinterpret_cast<T *>(ws + l.q), *k = reinterpret_cast<T *>(ws + l.k);
    T *v = reinterpret_cast<T *>(ws + l.v), *z = reinterpret_cast<T *>(ws + l.z);
    T *t = reinterpret_cast<T *>(ws + l.t);
    float *la = reinterpret_cast<float *>(ws + l.la);
    int rc;
    // token mixer
    if ((rc = layer_norm<T>(x, w->ln1_w, w->ln1_b, x1, M, C, st))) return rc;
    if ((rc = dense_gemm(dtype, M, 5 * C, C, x1, w->w_proj, nullptr, nullptr, P, st))) return rc;
    split_heads_kernel<T><<<grid_for(M * 5 * C / 8, 256), 256, 0, st>>>(P, w->b_a, q, k, v, la, z, M, N, C);
    note_launch();
    if (cudaPeekAtLastError() != cudaSuccess) return GTR_GLA_ERR_CUDA;
    // attention with the output tail fused into its stores: t = Tail(o, z, w_n)
    if ((rc = gtr_gla_fwd_tail(q, k, v, la, z, w->w_n, kTailEps, t, nullptr, B, H, gh, gw, 64, 64, dir, dtype,
                               ws + l.gla, l.gla_bytes, st)))
        return rc;
    if ((rc = dense_gemm(dtype, M, C, C, t, w->w_o, nullptr, x, x, st))) return rc;
    // channel mixer
    if ((rc = layer_norm<T>(x, w->ln2_w, w->ln2_b, x1, M, C, st))) return rc;
    return swiglu_apply(x1, w->w_gu, w->b_gu, w->w_dw, w->b_dw, w->w_down, w->b_down, x, x, B, gh, gw, C, F, dtype,
                        ws + l.sw, st);
}

int validate(int B, int gh, int gw, int C, int F, int dir, int dtype) {
    if (B <= 0 || gh <= 0 || gw <= 0 || C <= 0 || C % 64 || C > 2048 || F <= 0 || F % 8) return GTR_GLA_ERR_SHAPE;
    if ((long long)B * gh * gw > (1LL << 26)) return GTR_GLA_ERR_SHAPE;
    if (dir < 0 || dir > 3) return GTR_GLA_ERR_DIRECTION;
    if (dtype != GTR_GLA_F16 && dtype != GTR_GLA_BF16) return GTR_GLA_ERR_DTYPE;
    return GTR_GLA_OK;
}

}  // namespace
}  // namespace gtr

using namespace gtr;

extern "C" size_t gtr_layer_workspace_size(int B, int grid_h, int grid_w, int C, int F, int dtype) {
    if (validate(B, grid_h, grid_w, C, F, 0, dtype)) return 0;
    return layout(B, grid_h, grid_w, C, F, dtype).total;
}

namespace {

int check_weights(const GtrLayerWeights *w) {
    if (!w || !w->ln1_w || !w->ln1_b || !w->w_proj || !w->b_a || !w->w_n || !w->w_o || !w->ln2_w || !w->ln2_b ||
        !w->w_gu || !w->b_gu || !w->w_dw || !w->b_dw || !w->w_down || !w->b_down)
        return GTR_GLA_ERR_NULL;
    const void *ptrs[] = {w->ln1_w, w->ln1_b, w->w_proj, w->b_a, w->w_n, w->w_o, w->ln2_w, w->ln2_b,
                          w->w_gu, w->b_gu, w->w_dw, w->b_dw, w->w_down, w->b_down};
    for (const void *p : ptrs)
        if (((uintptr_t)p & 15u) != 0) return GTR_GLA_ERR_ALIGN;
    return GTR_GLA_OK;
}

// Checks of everything but the weights; on success *l is the workspace layout.
int check_call(const void *x, int B, int gh, int gw, int C, int F, int dir, int dtype, const void *workspace,
               size_t workspace_bytes, Layout *l) {
    if (!x) return GTR_GLA_ERR_NULL;
    int rc = validate(B, gh, gw, C, F, dir, dtype);
    if (rc) return rc;
    if (((uintptr_t)x & 15u) != 0) return GTR_GLA_ERR_ALIGN;
    *l = layout(B, gh, gw, C, F, dtype);
    if (!workspace || workspace_bytes < l->total || ((uintptr_t)workspace & 255u)) return GTR_GLA_ERR_WORKSPACE;
    return GTR_GLA_OK;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    const char *pa = static_cast<const char *>(a), *pb = static_cast<const char *>(b);
    return pa < pb + nb && pb < pa + na;
}

// x is updated in place and the workspace written, so neither may overlap
// the other or any weight (weights may share memory among themselves).
int check_alias(const void *x, const GtrLayerWeights *w, int B, int gh, int gw, int C, int F,
                const void *workspace, const Layout &l) {
    const size_t e = 2, M = (size_t)B * gh * gw, nx = M * C * e;
    if (overlaps(x, nx, workspace, l.total)) return GTR_GLA_ERR_ALIAS;
    const struct {
        const void *p;
        size_t n;
    } wts[] = {{w->ln1_w, (size_t)C * 4},          {w->ln1_b, (size_t)C * 4},
               {w->w_proj, (size_t)5 * C * C * e}, {w->b_a, (size_t)C * 4},
               {w->w_n, (size_t)C * 4},            {w->w_o, (size_t)C * C * e},
               {w->ln2_w, (size_t)C * 4},          {w->ln2_b, (size_t)C * 4},
               {w->w_gu, (size_t)2 * F * C * e},   {w->b_gu, (size_t)2 * F * 4},
               {w->w_dw, (size_t)9 * F * 4},       {w->b_dw, (size_t)F * 4},
               {w->w_down, (size_t)C * F * e},     {w->b_down, (size_t)C * 4}};
    for (const auto &t : wts)
        if (overlaps(t.p, t.n, x, nx) || overlaps(t.p, t.n, workspace, l.total)) return GTR_GLA_ERR_ALIAS;
    return GTR_GLA_OK;
}

int run_layer(void *x, const GtrLayerWeights *w, int B, int gh, int gw, int C, int F, int dir, int dtype,
              void *workspace, const Layout &l, cudaStream_t st) {
    char *ws = static_cast<char *>(workspace);
    if (dtype == GTR_GLA_BF16)
        return layer_impl<__nv_bfloat16>(static_cast<__nv_bfloat16 *>(x), w, B, gh, gw, C, F, dir, dtype, ws, l,
                                         st);
    return layer_impl<__half>(static_cast<__half *>(x), w, B, gh, gw, C, F, dir, dtype, ws, l, st);
}

}  // namespace

extern "C" int gtr_layer_fwd(void *x, const GtrLayerWeights *w, int B, int grid_h, int grid_w, int C, int F,
                             int direction, int dtype, void *workspace, size_t workspace_bytes,
                             cudaStream_t stream) {
    int rc = check_weights(w);
    if (rc) return rc;
    Layout l;
    if ((rc = check_call(x, B, grid_h, grid_w, C, F, direction, dtype, workspace, workspace_bytes, &l))) return rc;
    if ((rc = check_alias(x, w, B, grid_h, grid_w, C, F, workspace, l))) return rc;
    return run_layer(x, w, B, grid_h, grid_w, C, F, direction, dtype, workspace, l, stream);
}

extern "C" int gtr_backbone_fwd(void *x, const GtrLayerWeights *layers, int n_layers, int B, int grid_h,
                                int grid_w, int C, int F, int dtype, void *workspace, size_t workspace_bytes,
                                cudaStream_t stream) {
    if (!layers) return GTR_GLA_ERR_NULL;
    if (n_layers < 1) return GTR_GLA_ERR_SHAPE;
    int rc;
    for (int i = 0; i < n_layers; ++i)
        if ((rc = check_weights(&layers[i]))) return rc;
    Layout l;
    if ((rc = check_call(x, B, grid_h, grid_w, C, F, 0, dtype, workspace, workspace_bytes, &l))) return rc;
    for (int i = 0; i < n_layers; ++i)
        if ((rc = check_alias(x, &layers[i], B, grid_h, grid_w, C, F, workspace, l))) return rc;
    for (int i = 0; i < n_layers; ++i)
        if ((rc = run_layer(x, &layers[i], B, grid_h, grid_w, C, F, i % 4, dtype, workspace, l, stream))) return rc;
    return GTR_GLA_OK;
}
