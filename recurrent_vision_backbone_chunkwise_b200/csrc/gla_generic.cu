// gla_generic.cu -- three-phase chunkwise GLA forward on CUDA cores (fp32
// arithmetic), for every I/O dtype.  It is the exact-arithmetic path of the
// library: fp32 I/O always runs here; fp16/bf16 run here only when asked for
// explicitly (the tensor-core path is the default for them).
//
// The three phases follow the chunkwise reorganisation of "GTR: Gated Token
// Recurrence for Efficient Dense Prediction" (x-techcon article, section 算子):
//   1. every chunk computes its own contribution dS_c to the state and its
//      gate product gamma_c, in parallel           (gla_chunk_state_kernel)
//   2. the chunk-boundary states are passed along: S_in(c+1) =
//      diag(gamma_c) S_in(c) + dS_c, in place over dS (gla_state_scan_kernel)
//   3. every chunk produces its output in parallel (gla_chunk_output_kernel)
//      o_t = (q_t . e^{b_t}) S_in(c) + sum_{s<=t} A[t,s] v_s,
//      A[t,s] = sum_i q_ti k_si e^{b_ti - b_si}, computed pair by pair so
//      that no gate factor can overflow whatever the gates are.
// b_t is the inclusive prefix sum of log_alpha inside the chunk (scan order).
#include "gla_common.cuh"
#include "gla_internal.h"

namespace gtr {

constexpr int kGenThreads = 256;

template <typename T, int DK, int DV, int C>
__global__ void __launch_bounds__(kGenThreads)
gla_chunk_state_kernel(const T *__restrict__ k, const T *__restrict__ v,
                       const float *__restrict__ la, float *__restrict__ dS,
                       float *__restrict__ gam, int n, int gh, int gw, int dir, int nc, int *err) {
    extern __shared__ float sm[];
    float *b = sm;            // [C][DK]  log-gate prefix sums
    float *kh = b + C * DK;   // [C][DK]  k, then k . e^{g - b}
    float *vs = kh + C * DK;  // [C][DV]
    const int c = blockIdx.x, bh = blockIdx.y;
    const int t0 = c * C;
    const int len = min(C, n - t0);
    const size_t pk = (size_t)bh * n * DK, pv = (size_t)bh * n * DV;

    for (int e = threadIdx.x; e < C * DK; e += blockDim.x) {
        const int u = e / DK, i = e % DK;
        float lv = 0.f, kv = 0.f;
        const size_t r = (size_t)scan_to_raster(t0 + u, n, gh, gw, dir);
        if (u < len && index_ok(r < (size_t)n, err)) {
            lv = la[pk + r * DK + i];
            kv = to_f32(k[pk + r * DK + i]);
        }
        b[e] = lv;
        kh[e] = kv;
    }
    for (int e = threadIdx.x; e < C * DV; e += blockDim.x) {
        const int u = e / DV, j = e % DV;
        float vv = 0.f;
        const size_t r = (size_t)scan_to_raster(t0 + u, n, gh, gw, dir);
        if (u < len && index_ok(r < (size_t)n, err)) vv = to_f32(v[pv + r * DV + j]);
        vs[e] = vv;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < DK; i += blockDim.x) {
        float acc = 0.f;
        for (int u = 0; u < len; ++u) {
            acc += b[u * DK + i];
            b[u * DK + i] = acc;
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < len * DK; e += blockDim.x) {
        const int i = e % DK;
        kh[e] *= expf(b[(len - 1) * DK + i] - b[e]);  // factor <= 1
    }
    __syncthreads();

    constexpr int RI = DK / 16, RJ = DV / 16;
    const int ti = threadIdx.x / 16, tj = threadIdx.x % 16;
    float acc[RI][RJ];
#pragma unroll
    for (int a = 0; a < RI; ++a)
#pragma unroll
        for (int q = 0; q < RJ; ++q) acc[a][q] = 0.f;
    for (int u = 0; u < len; ++u) {
        float kv[RI], vv[RJ];
#pragma unroll
        for (int a = 0; a < RI; ++a) kv[a] = kh[u * DK + ti + 16 * a];
#pragma unroll
        for (int q = 0; q < RJ; ++q) vv[q] = vs[u * DV + tj + 16 * q];
#pragma unroll
        for (int a = 0; a < RI; ++a)
#pragma unroll
            for (int q = 0; q < RJ; ++q) acc[a][q] = fmaf(kv[a], vv[q], acc[a][q]);
    }
    float *out = dS + ((size_t)bh * nc + c) * DK * DV;
#pragma unroll
    for (int a = 0; a < RI; ++a)
#pragma unroll
        for (int q = 0; q < RJ; ++q) out[(ti + 16 * a) * DV + tj + 16 * q] = acc[a][q];
    for (int i = threadIdx.x; i < DK; i += blockDim.x)
        gam[((size_t)bh * nc + c) * DK + i] = expf(b[(len - 1) * DK + i]);
}

// One thread per state element (i, j) of one (b, h); walks the chunks in scan
// order.  dS[c] is replaced by S_in(c); the state after the last chunk goes to
// final_state.  Loads are issued ahead of the dependent multiply-adds.
template <int DK, int DV>
__global__ void __launch_bounds__(kGenThreads)
gla_state_scan_kernel(float *__restrict__ dS, const float *__restrict__ gam,
                      float *__restrict__ final_state, int nc) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    const int bh = blockIdx.y;
    if (e >= DK * DV) return;
    const int i = e / DV;
    float *p = dS + (size_t)bh * nc * DK * DV + e;
    const float *g = gam + (size_t)bh * nc * DK + i;
    float S = 0.f;
    constexpr int U = 8;
    int c = 0;
    for (; c + U <= nc; c += U) {
        float d[U], gm[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            d[u] = p[(size_t)(c + u) * DK * DV];
            gm[u] = g[(size_t)(c + u) * DK];
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            p[(size_t)(c + u) * DK * DV] = S;
            S = fmaf(gm[u], S, d[u]);
        }
    }
    for (; c < nc; ++c) {
        const float d = p[(size_t)c * DK * DV];
        const float gm = g[(size_t)c * DK];
        p[(size_t)c * DK * DV] = S;
        S = fmaf(gm, S, d);
    }
    if (final_state) final_state[(size_t)bh * DK * DV + e] = S;
}

// grid = (chunks, B*H, DV / VT); each CTA writes a C x VT tile of the output.
template <typename T, int DK, int DV, int C, int VT>
__global__ void __launch_bounds__(kGenThreads)
gla_chunk_output_kernel(const T *__restrict__ q, const T *__restrict__ k,
                        const T *__restrict__ v, const float *__restrict__ la,
                        const float *__restrict__ Sin, T *__restrict__ o, int n, int gh,
                        int gw, int dir, int nc, int *err) {
    constexpr int DKP = DK + 1;  // padded rows: pair loops read one row per lane
    constexpr int CP = C + 1;
    extern __shared__ float sm[];
    float *qh = sm;               // [C][DKP]  q, later q . e^{b}
    float *b = qh + C * DKP;      // [C][DKP]
    float *kk = b + C * DKP;      // [C][DKP]
    float *vs = kk + C * DKP;     // [C][VT]
    float *S = vs + C * VT;       // [DK][VT]
    float *A = S + DK * VT;       // [C][CP]
    const int c = blockIdx.x, bh = blockIdx.y, j0 = blockIdx.z * VT;
    const int t0 = c * C;
    const int len = min(C, n - t0);
    const size_t pk = (size_t)bh * n * DK, pv = (size_t)bh * n * DV;

    for (int e = threadIdx.x; e < C * DK; e += blockDim.x) {
        const int u = e / DK, i = e % DK;
        float qv = 0.f, kv = 0.f, lv = 0.f;
        const size_t r = (size_t)scan_to_raster(t0 + u, n, gh, gw, dir);
        if (u < len && index_ok(r < (size_t)n, err)) {
            qv = to_f32(q[pk + r * DK + i]);
            kv = to_f32(k[pk + r * DK + i]);
            lv = la[pk + r * DK + i];
        }
        qh[u * DKP + i] = qv;
        kk[u * DKP + i] = kv;
        b[u * DKP + i] = lv;
    }
    for (int e = threadIdx.x; e < C * VT; e += blockDim.x) {
        const int u = e / VT, j = e % VT;
        float vv = 0.f;
        const size_t r = (size_t)scan_to_raster(t0 + u, n, gh, gw, dir);
        if (u < len && index_ok(r < (size_t)n, err)) vv = to_f32(v[pv + r * DV + j0 + j]);
        vs[e] = vv;
    }
    const float *Sg = Sin + ((size_t)bh * nc + c) * DK * DV;
    for (int e = threadIdx.x; e < DK * VT; e += blockDim.x) {
        const int i = e / VT, j = e % VT;
        S[e] = Sg[i * DV + j0 + j];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < DK; i += blockDim.x) {
        float acc = 0.f;
        for (int u = 0; u < len; ++u) {
            acc += b[u * DKP + i];
            b[u * DKP + i] = acc;
        }
    }
    __syncthreads();
    // intra-chunk scores, lower triangle with the diagonal, exact gate per pair
    for (int e = threadIdx.x; e < C * C; e += blockDim.x) {
        const int t = e / C, s = e % C;
        float a = 0.f;
        if (s <= t && t < len) {
            const float *qt = qh + t * DKP, *bt = b + t * DKP;
            const float *ks = kk + s * DKP, *bs = b + s * DKP;
            for (int i = 0; i < DK; ++i) a = fmaf(qt[i] * ks[i], expf(bt[i] - bs[i]), a);
        }
        A[t * CP + s] = a;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < len * DK; e += blockDim.x) {
        const int u = e / DK, i = e % DK;
        qh[u * DKP + i] *= expf(b[u * DKP + i]);  // factor <= 1
    }
    __syncthreads();

    constexpr int RT = C / 16, RJ = VT / 16;
    const int tt = threadIdx.x / 16, tj = threadIdx.x % 16;
    float acc[RT][RJ];
#pragma unroll
    for (int a = 0; a < RT; ++a)
#pragma unroll
        for (int w = 0; w < RJ; ++w) acc[a][w] = 0.f;
    for (int i = 0; i < DK; ++i) {  // inter-chunk part
        float sv[RJ];
#pragma unroll
        for (int w = 0; w < RJ; ++w) sv[w] = S[i * VT + tj + 16 * w];
#pragma unroll
        for (int a = 0; a < RT; ++a) {
            const float x = qh[(tt + 16 * a) * DKP + i];
#pragma unroll
            for (int w = 0; w < RJ; ++w) acc[a][w] = fmaf(x, sv[w], acc[a][w]);
        }
    }
    for (int s = 0; s < len; ++s) {  // intra-chunk part (A is zero above the diagonal)
        float vv[RJ];
#pragma unroll
        for (int w = 0; w < RJ; ++w) vv[w] = vs[s * VT + tj + 16 * w];
#pragma unroll
        for (int a = 0; a < RT; ++a) {
            const float x = A[(tt + 16 * a) * CP + s];
#pragma unroll
            for (int w = 0; w < RJ; ++w) acc[a][w] = fmaf(x, vv[w], acc[a][w]);
        }
    }
#pragma unroll
    for (int a = 0; a < RT; ++a) {
        const int u = tt + 16 * a;
        if (u >= len) continue;
        const size_t r = (size_t)scan_to_raster(t0 + u, n, gh, gw, dir);
        if (!index_ok(r < (size_t)n, err)) continue;
#pragma unroll
        for (int w = 0; w < RJ; ++w) o[pv + r * DV + j0 + tj + 16 * w] = from_f32<T>(acc[a][w]);
    }
}

size_t generic_workspace_bytes(const Problem &p) {
    const size_t nc = (size_t)(p.n + p.chunk - 1) / p.chunk;
    const size_t bh = (size_t)p.B * p.H;
    size_t bytes = kWsHeaderBytes + bh * nc * (size_t)p.dk * p.dv * sizeof(float);
    bytes = (bytes + 255) & ~(size_t)255;
    bytes += bh * nc * (size_t)p.dk * sizeof(float);
    return (bytes + 255) & ~(size_t)255;
}

template <typename T, int DK, int DV, int C>
static int launch_generic_t(const Problem &p, void *ws, cudaStream_t st) {
    const int nc = (p.n + C - 1) / C;
    const int bh = p.B * p.H;
    char *data = (char *)ws + kWsHeaderBytes;  // the header belongs to the fused path
    float *dS = (float *)data;
    size_t off = ((size_t)bh * nc * DK * DV * sizeof(float) + 255) & ~(size_t)255;
    float *gam = (float *)(data + off);

    const size_t sm1 = (size_t)(2 * C * DK + C * DV) * sizeof(float);
    auto k1 = gla_chunk_state_kernel<T, DK, DV, C>;
    if (ensure_smem((const void *)k1, sm1)) return GTR_GLA_ERR_CUDA;
    k1<<<dim3(nc, bh), kGenThreads, sm1, st>>>((const T *)p.k, (const T *)p.v, p.la, dS, gam,
                                               p.n, p.gh, p.gw, p.dir, nc, p.err);
    note_launch();

    auto k2 = gla_state_scan_kernel<DK, DV>;
    k2<<<dim3((DK * DV + kGenThreads - 1) / kGenThreads, bh), kGenThreads, 0, st>>>(
        dS, gam, p.final_state, nc);
    note_launch();

    constexpr int VT = 64;
    const size_t sm3 =
        (size_t)(3 * C * (DK + 1) + C * VT + DK * VT + C * (C + 1)) * sizeof(float);
    auto k3 = gla_chunk_output_kernel<T, DK, DV, C, VT>;
    if (ensure_smem((const void *)k3, sm3)) return GTR_GLA_ERR_CUDA;
    k3<<<dim3(nc, bh, DV / VT), kGenThreads, sm3, st>>>((const T *)p.q, (const T *)p.k,
                                                         (const T *)p.v, p.la, dS, (T *)p.out,
                                                         p.n, p.gh, p.gw, p.dir, nc, p.err);
    note_launch();
    return cudaPeekAtLastError() == cudaSuccess ? GTR_GLA_OK : GTR_GLA_ERR_CUDA;
}

template <typename T, int C>
static int launch_generic_dims(const Problem &p, void *ws, cudaStream_t st) {
    if (p.dk == 64 && p.dv == 64) return launch_generic_t<T, 64, 64, C>(p, ws, st);
    if (p.dk == 128 && p.dv == 128) return launch_generic_t<T, 128, 128, C>(p, ws, st);
    if (p.dk == 64 && p.dv == 128) return launch_generic_t<T, 64, 128, C>(p, ws, st);
    if (p.dk == 128 && p.dv == 64) return launch_generic_t<T, 128, 64, C>(p, ws, st);
    return GTR_GLA_ERR_HEAD_DIM;
}

template <typename T>
static int launch_generic_chunk(const Problem &p, void *ws, cudaStream_t st) {
    if (p.chunk == 32) return launch_generic_dims<T, 32>(p, ws, st);
    if (p.chunk == 64) return launch_generic_dims<T, 64>(p, ws, st);
    if (p.chunk == 128 && p.dk == 64) {  // d_k = 128 would not fit shared memory
        if (p.dv == 64) return launch_generic_t<T, 64, 64, 128>(p, ws, st);
        if (p.dv == 128) return launch_generic_t<T, 64, 128, 128>(p, ws, st);
    }
    return GTR_GLA_ERR_CHUNK;
}

int launch_generic(const Problem &p, void *ws, cudaStream_t st) {
    switch (p.dtype) {
        case GTR_GLA_F16: return launch_generic_chunk<__half>(p, ws, st);
        case GTR_GLA_BF16: return launch_generic_chunk<__nv_bfloat16>(p, ws, st);
        case GTR_GLA_F32: return launch_generic_chunk<float>(p, ws, st);
        default: return GTR_GLA_ERR_DTYPE;
    }
}

}  // namespace gtr
