// gla_backward.cu -- gradients of the chunkwise GLA forward pass on CUDA
// cores (fp32 arithmetic, every gate factor <= 1), chunk 64, d_k = d_v = 64.
// "GTR: Gated Token Recurrence for Efficient Dense Prediction", x-techcon
// article, section 算子: the pages' operator is inference-only (training used
// another library's kernel); this is the reverse mode of the same recurrence
// (include/gtr_gla_bwd.h), organised by chunks like the forward pass:
//   1. per chunk: b (inclusive in-chunk log-gate sums), g, gamma = e^g and
//      dS_c = sum_s (k_s . e^{g - b_s})^T v_s                 (bwd_chunk_state)
//   2. per plane: S_in(c) = diag(gamma_{c-1}) S_in(c-1) + dS_{c-1}, in place,
//      and S_final                                              (bwd_state_scan)
//   3. per chunk: Z_c = sum_t (q_t . e^{b_t})^T dO_t            (bwd_chunk_dstate)
//   4. per plane, last chunk first: dS_out(c) = cur; cur = diag(gamma_c) cur + Z_c,
//      starting from dS_final (or 0), in place over Z          (bwd_dstate_scan)
//   5. per chunk, with W[t,s] = dO_t . v_s and A[t,s] = sum_i q_ti k_si e^{b_ti - b_si}
//      (s <= t):  dq_t = e^{b_t} . (dO_t S_in^T) + sum_s W k_s . e^{b_t - b_s}
//                 dk_s = sum_t W q_t . e^{b_t - b_s} + e^{g - b_s} . (dS_out v_s)
//                 dv_s = sum_t A dO_t + (k_s . e^{g - b_s}) dS_out
//      and db_t = q_t . dq_t - k_t . dk_t (+ rowsum(dS_final . S_final) at the
//      scan's last token); dlog_alpha gets the in-chunk suffix sums of db and
//      the chunk's total goes to a side array                 (bwd_chunk_grads)
//   6. per plane: the totals of the later chunks, exclusive    (bwd_carry)
//   7. per token: dlog_alpha += the carry of its chunk           (bwd_add_carry)
// Tokens are addressed in place through scan_to_raster, as in the forward pass.
// The in-chunk log-gate sums b are kept in the log2 domain and every gate
// factor (all <= 1) is one hardware 2^x (relative error about 2^-22).
#include "../../include/gtr_gla_bwd.h"
#include "sm100.cuh"
#include "gla_common.cuh"
#include "gla_internal.h"

namespace gtr {
namespace {

using sm100::fast_exp2;
// bwd_chunk_grads holds one CTA per SM (its shared memory) and runs 32 warps
// to hide the latency of its shared-memory loads.  The two other chunk
// kernels (48 KB each) take the thread count NT: 1024 when the problem gives
// about one CTA per SM, else 256, so that four CTAs share an SM and overlap
// each other's serial prefix-sum phase.
constexpr int kT = 1024;
constexpr int kTSmall = 256;
constexpr float kLog2e = 1.4426950408889634f;

template <typename T, int DK, int DV, int C, int NT>
__global__ void __launch_bounds__(NT) bwd_chunk_state(const T *__restrict__ k, const T *__restrict__ v,
                                                      const float *__restrict__ la, float *__restrict__ dS,
                                                      float *__restrict__ gam, int n, int gh, int gw, int dir,
                                                      int nc) {
    extern __shared__ float sm[];
    float *b = sm, *kh = b + C * DK, *vs = kh + C * DK;
    const int c = blockIdx.x, bh = blockIdx.y, t0 = c * C, len = min(C, n - t0);
    const size_t pk = (size_t)bh * n * DK, pv = (size_t)bh * n * DV;
    for (int e = threadIdx.x; e < C * DK; e += NT) {
        const int u = e / DK, i = e % DK;
        float lv = 0.f, kv = 0.f;
        if (u < len) {
            const size_t r = (size_t)scan_to_raster(t0 + u, n, gh, gw, dir);
            lv = la[pk + r * DK + i];
            kv = to_f32(k[pk + r * DK + i]);
        }
        b[e] = lv;
        kh[e] = kv;
    }
    for (int e = threadIdx.x; e < C * DV; e += NT) {
        const int u = e / DV, j = e % DV;
        vs[e] = u < len ? to_f32(v[pv + (size_t)scan_to_raster(t0 + u, n, gh, gw, dir) * DV + j]) : 0.f;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < DK; i += NT) {  // prefix sums per key dimension
        float acc = 0.f;
        for (int u = 0; u < C; ++u) {
            acc = fmaf(b[u * DK + i], kLog2e, acc);  // log2 domain
            b[u * DK + i] = acc;
        }
        gam[((size_t)bh * nc + c) * DK + i] = fast_exp2(acc);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < C * DK; e += NT) {
        const int u = e / DK, i = e % DK;
        kh[e] = u < len ? kh[e] * fast_exp2(b[(C - 1) * DK + i] - b[e]) : 0.f;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < DK * DV; e += NT) {
        const int i = e / DV, j = e % DV;
        float acc = 0.f;
        for (int u = 0; u < len; ++u) acc = fmaf(kh[u * DK + i], vs[u * DV + j], acc);
        dS[((size_t)bh * nc + c) * DK * DV + e] = acc;
    }
}

// S_in(c) in place over dS_c (S_in(0) = 0), and S_final.
template <int DK, int DV>
__global__ void bwd_state_scan(float *__restrict__ dS, const float *__restrict__ gam, float *__restrict__ S_final,
                               int nc) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x, bh = blockIdx.y;
    if (e >= DK * DV) return;
    const int i = e / DV;
    float s = 0.f;
#pragma unroll 4
    for (int c = 0; c < nc; ++c) {
        float *p = dS + ((size_t)bh * nc + c) * DK * DV + e;
        const float d = *p;
        *p = s;
        s = gam[((size_t)bh * nc + c) * DK + i] * s + d;
    }
    S_final[(size_t)bh * DK * DV + e] = s;
}

template <typename T, int DK, int DV, int C, int NT>
__global__ void __launch_bounds__(NT) bwd_chunk_dstate(const T *__restrict__ q, const T *__restrict__ dO,
                                                       const float *__restrict__ la, float *__restrict__ Z, int n,
                                                       int gh, int gw, int dir, int nc) {
    extern __shared__ float sm[];
    float *b = sm, *qh = b + C * DK, *gs = qh + C * DK;
    const int c = blockIdx.x, bh = blockIdx.y, t0 = c * C, len = min(C, n - t0);
    const size_t pk = (size_t)bh * n * DK, pv = (size_t)bh * n * DV;
    for (int e = threadIdx.x; e < C * DK; e += NT) {
        const int u = e / DK, i = e % DK;
        float lv = 0.f, qv = 0.f;
        if (u < len) {
            const size_t r = (size_t)scan_to_raster(t0 + u, n, gh, gw, dir);
            lv = la[pk + r * DK + i];
            qv = to_f32(q[pk + r * DK + i]);
        }
        b[e] = lv;
        qh[e] = qv;
    }
    for (int e = threadIdx.x; e < C * DV; e += NT) {
        const int u = e / DV, j = e % DV;
        gs[e] = u < len ? to_f32(dO[pv + (size_t)scan_to_raster(t0 + u, n, gh, gw, dir) * DV + j]) : 0.f;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < DK; i += NT) {
        float acc = 0.f;
        for (int u = 0; u < C; ++u) {
            acc = fmaf(b[u * DK + i], kLog2e, acc);  // log2 domain
            b[u * DK + i] = acc;
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < C * DK; e += NT) qh[e] *= fast_exp2(b[e]);
    __syncthreads();
    for (int e = threadIdx.x; e < DK * DV; e += NT) {
        const int i = e / DV, j = e % DV;
        float acc = 0.f;
        for (int u = 0; u < len; ++u) acc = fmaf(qh[u * DK + i], gs[u * DV + j], acc);
        Z[((size_t)bh * nc + c) * DK * DV + e] = acc;
    }
}

// dS_out(c) in place over Z_c, last chunk first.
template <int DK, int DV>
__global__ void bwd_dstate_scan(float *__restrict__ Z, const float *__restrict__ gam,
                                const float *__restrict__ dS_final, int nc) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x, bh = blockIdx.y;
    if (e >= DK * DV) return;
    const int i = e / DV;
    float cur = dS_final ? dS_final[(size_t)bh * DK * DV + e] : 0.f;
#pragma unroll 4
    for (int c = nc - 1; c >= 0; --c) {
        float *p = Z + ((size_t)bh * nc + c) * DK * DV + e;
        const float z = *p;
        *p = cur;
        cur = gam[((size_t)bh * nc + c) * DK + i] * cur + z;
    }
}

// Per chunk: dq, dk, dv in the I/O dtype at raster positions; dlog_alpha gets
// the in-chunk suffix sums of db (fp32), the chunk total goes to tot.
template <typename T, int DK, int DV, int C>
__global__ void __launch_bounds__(kT) bwd_chunk_grads(
    const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v, const float *__restrict__ la,
    const T *__restrict__ dO, const float *__restrict__ S_in, const float *__restrict__ dS_out,
    const float *__restrict__ dS_final, const float *__restrict__ S_final, T *__restrict__ dq, T *__restrict__ dk,
    T *__restrict__ dv, float *__restrict__ dla, float *__restrict__ tot, int n, int gh, int gw, int dir, int nc) {
    // Rows padded by one float (DKP, DVP): the loops below walk a column with
    // consecutive lanes on consecutive rows, which padding keeps free of
    // shared-memory bank conflicts.  The chunk's S_in and dS_out are staged
    // the same way (their rows are read across lanes too).
    constexpr int DKP = DK + 1, DVP = DV + 1;
    extern __shared__ float sm[];
    float *b = sm;              // [C][DKP]  in-chunk log2-gate sums
    float *qs = b + C * DKP;    // [C][DKP]
    float *ks = qs + C * DKP;   // [C][DKP]
    float *vs = ks + C * DKP;   // [C][DVP]
    float *gs = vs + C * DVP;   // [C][DVP]  dO
    float *W = gs + C * DVP;    // [C][C]    dO_t . v_s, s <= t
    float *A = W + C * C;       // [C][C]    scores, s <= t
    float *db = A + C * C;      // [C][DK]
    float *Si = db + C * DK;    // [DK][DVP] S_in of the chunk
    float *Do = Si + DK * DVP;  // [DK][DVP] dS_out of the chunk
    const int c = blockIdx.x, bh = blockIdx.y, t0 = c * C, len = min(C, n - t0);
    const size_t pk = (size_t)bh * n * DK, pv = (size_t)bh * n * DV;
    const float *Sig = S_in + ((size_t)bh * nc + c) * DK * DV;
    const float *Dog = dS_out + ((size_t)bh * nc + c) * DK * DV;
    for (int e = threadIdx.x; e < C * DK; e += kT) {
        const int u = e / DK, i = e % DK;
        float lv = 0.f, qv = 0.f, kv = 0.f;
        if (u < len) {
            const size_t r = (size_t)scan_to_raster(t0 + u, n, gh, gw, dir);
            lv = la[pk + r * DK + i];
            qv = to_f32(q[pk + r * DK + i]);
            kv = to_f32(k[pk + r * DK + i]);
        }
        b[u * DKP + i] = lv;
        qs[u * DKP + i] = qv;
        ks[u * DKP + i] = kv;
    }
    for (int e = threadIdx.x; e < C * DV; e += kT) {
        const int u = e / DV, j = e % DV;
        float vv = 0.f, gv = 0.f;
        if (u < len) {
            const size_t r = (size_t)scan_to_raster(t0 + u, n, gh, gw, dir);
            vv = to_f32(v[pv + r * DV + j]);
            gv = to_f32(dO[pv + r * DV + j]);
        }
        vs[u * DVP + j] = vv;
        gs[u * DVP + j] = gv;
    }
    for (int e = threadIdx.x; e < DK * DV; e += kT) {
        const int i = e / DV, j = e % DV;
        Si[i * DVP + j] = Sig[e];
        Do[i * DVP + j] = Dog[e];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < DK; i += kT) {
        float acc = 0.f;
        for (int u = 0; u < C; ++u) {
            acc = fmaf(b[u * DKP + i], kLog2e, acc);  // log2 domain
            b[u * DKP + i] = acc;
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < C * C; e += kT) {  // W and A, pair by pair
        const int t = e / C, s = e % C;
        float w = 0.f, a = 0.f;
        if (s <= t && t < len) {
            for (int j = 0; j < DV; ++j) w = fmaf(gs[t * DVP + j], vs[s * DVP + j], w);
            for (int i = 0; i < DK; ++i)
                a = fmaf(qs[t * DKP + i] * ks[s * DKP + i], fast_exp2(b[t * DKP + i] - b[s * DKP + i]), a);
        }
        W[e] = w;
        A[e] = a;
    }
    __syncthreads();
    const float *gend = b + (C - 1) * DKP;  // g: the chunk's total (padded tokens add log 1 = 0)
    for (int e = threadIdx.x; e < C * DK; e += kT) {  // dq and dk, one (token, key dim) per step
        const int t = e / DK, i = e % DK;
        float gq = 0.f, gk = 0.f;
        if (t < len) {
            float inter = 0.f, intra = 0.f;
            for (int j = 0; j < DV; ++j) inter = fmaf(gs[t * DVP + j], Si[i * DVP + j], inter);
            for (int s = 0; s <= t; ++s)
                intra = fmaf(W[t * C + s] * ks[s * DKP + i], fast_exp2(b[t * DKP + i] - b[s * DKP + i]), intra);
            gq = fast_exp2(b[t * DKP + i]) * inter + intra;
            float st = 0.f, kk = 0.f;  // token t as the key side s
            for (int u = t; u < len; ++u)
                kk = fmaf(W[u * C + t] * qs[u * DKP + i], fast_exp2(b[u * DKP + i] - b[t * DKP + i]), kk);
            for (int j = 0; j < DV; ++j) st = fmaf(vs[t * DVP + j], Do[i * DVP + j], st);
            gk = kk + fast_exp2(gend[i] - b[t * DKP + i]) * st;
            const size_t r = (size_t)scan_to_raster(t0 + t, n, gh, gw, dir);
            dq[pk + r * DK + i] = from_f32<T>(gq);
            dk[pk + r * DK + i] = from_f32<T>(gk);
        }
        db[e] = qs[t * DKP + i] * gq - ks[t * DKP + i] * gk;
        if (t0 + t == n - 1 && dS_final) {  // the scan's last token: the final state's gate
            float f = 0.f;
            for (int j = 0; j < DV; ++j)
                f = fmaf(dS_final[(size_t)bh * DK * DV + i * DV + j], S_final[(size_t)bh * DK * DV + i * DV + j], f);
            db[e] += f;
        }
    }
    for (int e = threadIdx.x; e < C * DV; e += kT) {  // dv
        const int s = e / DV, j = e % DV;
        if (s >= len) continue;
        float acc = 0.f;
        for (int t = s; t < len; ++t) acc = fmaf(A[t * C + s], gs[t * DVP + j], acc);
        for (int i = 0; i < DK; ++i)
            acc = fmaf(ks[s * DKP + i] * fast_exp2(gend[i] - b[s * DKP + i]), Do[i * DVP + j], acc);
        const size_t r = (size_t)scan_to_raster(t0 + s, n, gh, gw, dir);
        dv[pv + r * DV + j] = from_f32<T>(acc);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < DK; i += kT) {  // suffix sums of db inside the chunk
        float acc = 0.f;
        for (int u = len - 1; u >= 0; --u) {
            acc += db[u * DK + i];
            const size_t r = (size_t)scan_to_raster(t0 + u, n, gh, gw, dir);
            dla[pk + r * DK + i] = acc;
        }
        tot[((size_t)bh * nc + c) * DK + i] = acc;
    }
}

// tot[c] <- sum of tot over the later chunks (exclusive, last chunk first).
template <int DK>
__global__ void bwd_carry(float *__restrict__ tot, int nc) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x, bh = blockIdx.y;
    if (i >= DK) return;
    float carry = 0.f;
    for (int c = nc - 1; c >= 0; --c) {
        float *p = tot + ((size_t)bh * nc + c) * DK + i;
        const float t = *p;
        *p = carry;
        carry += t;
    }
}

// dlog_alpha += the later chunks' totals, over scan positions p (chunk p / C).
template <int DK, int C>
__global__ void bwd_add_carry(float *__restrict__ dla, const float *__restrict__ tot, int n, int gh, int gw, int dir,
                              int nc, long long total) {
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const long long bh = e / ((long long)n * DK);
        const int rem = (int)(e % ((long long)n * DK)), p = rem / DK, i = rem % DK;
        const size_t r = (size_t)scan_to_raster(p, n, gh, gw, dir);
        dla[((size_t)bh * n + r) * DK + i] += tot[((size_t)bh * nc + p / C) * DK + i];
    }
}

struct BwdLayout {
    size_t S, Z, gam, tot, Sf, total;
};

BwdLayout bwd_layout(int BH, int nc, int DK, int DV) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    BwdLayout l;
    l.S = 0;
    l.Z = up((size_t)BH * nc * DK * DV * 4);
    l.gam = up(l.Z + (size_t)BH * nc * DK * DV * 4);
    l.tot = up(l.gam + (size_t)BH * nc * DK * 4);
    l.Sf = up(l.tot + (size_t)BH * nc * DK * 4);
    l.total = up(l.Sf + (size_t)BH * DK * DV * 4);
    return l;
}

template <typename T, int DK, int DV, int C>
int launch_bwd(const T *q, const T *k, const T *v, const float *la, const T *dO, const float *dSf, T *dq, T *dk,
               T *dv, float *dla, int B, int H, int gh, int gw, int dir, void *ws, cudaStream_t st) {
    const int n = gh * gw, nc = (n + C - 1) / C, BH = B * H;
    const BwdLayout l = bwd_layout(BH, nc, DK, DV);
    char *w = static_cast<char *>(ws);
    float *S = reinterpret_cast<float *>(w + l.S), *Z = reinterpret_cast<float *>(w + l.Z);
    float *gam = reinterpret_cast<float *>(w + l.gam), *tot = reinterpret_cast<float *>(w + l.tot);
    float *Sf = reinterpret_cast<float *>(w + l.Sf);
    const dim3 gchunk(nc, BH);
    const size_t sm1 = (size_t)(2 * C * DK + C * DV) * 4;
    const size_t sm5 = (size_t)(3 * C * (DK + 1) + 2 * C * (DV + 1) + 2 * C * C + C * DK + 2 * DK * (DV + 1)) * 4;
    const bool wide = (long long)nc * BH <= 2 * 148;  // about one chunk CTA per SM
    int rc;
    if ((rc = ensure_smem((const void *)bwd_chunk_state<T, DK, DV, C, kT>, sm1))) return rc;
    if ((rc = ensure_smem((const void *)bwd_chunk_state<T, DK, DV, C, kTSmall>, sm1))) return rc;
    if ((rc = ensure_smem((const void *)bwd_chunk_dstate<T, DK, DV, C, kT>, sm1))) return rc;
    if ((rc = ensure_smem((const void *)bwd_chunk_dstate<T, DK, DV, C, kTSmall>, sm1))) return rc;
    if ((rc = ensure_smem((const void *)bwd_chunk_grads<T, DK, DV, C>, sm5))) return rc;
    if (wide)
        bwd_chunk_state<T, DK, DV, C, kT><<<gchunk, kT, sm1, st>>>(k, v, la, S, gam, n, gh, gw, dir, nc);
    else
        bwd_chunk_state<T, DK, DV, C, kTSmall><<<gchunk, kTSmall, sm1, st>>>(k, v, la, S, gam, n, gh, gw, dir, nc);
    bwd_state_scan<DK, DV><<<dim3((DK * DV + 255) / 256, BH), 256, 0, st>>>(S, gam, Sf, nc);
    if (wide)
        bwd_chunk_dstate<T, DK, DV, C, kT><<<gchunk, kT, sm1, st>>>(q, dO, la, Z, n, gh, gw, dir, nc);
    else
        bwd_chunk_dstate<T, DK, DV, C, kTSmall><<<gchunk, kTSmall, sm1, st>>>(q, dO, la, Z, n, gh, gw, dir, nc);
    bwd_dstate_scan<DK, DV><<<dim3((DK * DV + 255) / 256, BH), 256, 0, st>>>(Z, gam, dSf, nc);
    bwd_chunk_grads<T, DK, DV, C><<<gchunk, kT, sm5, st>>>(q, k, v, la, dO, S, Z, dSf, Sf, dq, dk, dv, dla, tot, n,
                                                             gh, gw, dir, nc);
    bwd_carry<DK><<<dim3((DK + 63) / 64, BH), 64, 0, st>>>(tot, nc);
    const long long total = (long long)BH * n * DK;
    bwd_add_carry<DK, C><<<(unsigned)((total + 255) / 256 < 148 * 16 ? (total + 255) / 256 : 148 * 16), 256, 0,
                           st>>>(dla, tot, n, gh, gw, dir, nc, total);
    for (int i = 0; i < 7; ++i) note_launch();
    return cudaPeekAtLastError() == cudaSuccess ? GTR_GLA_OK : GTR_GLA_ERR_CUDA;
}

}  // namespace
}  // namespace gtr

using namespace gtr;

namespace {

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    const char *pa = (const char *)a, *pb = (const char *)b;
    return a && b && pa < pb + nb && pb < pa + na;
}

int check_bwd(const void *q, const void *k, const void *v, const float *la, const void *dO, const float *dSf,
              void *dq, void *dk, void *dv, float *dla, int B, int H, int gh, int gw, int dk_, int dv_, int dir,
              int dtype) {
    if (!q || !k || !v || !la || !dO || !dq || !dk || !dv || !dla) return GTR_GLA_ERR_NULL;
    if (B <= 0 || H <= 0 || gh <= 0 || gw <= 0 || (long long)B * H > 65535 || (long long)gh * gw > (1LL << 22))
        return GTR_GLA_ERR_SHAPE;
    if (dtype != GTR_GLA_F16 && dtype != GTR_GLA_BF16 && dtype != GTR_GLA_F32) return GTR_GLA_ERR_DTYPE;
    if (dk_ != 64 || dv_ != 64) return GTR_GLA_ERR_HEAD_DIM;
    if (dir < 0 || dir > 3) return GTR_GLA_ERR_DIRECTION;
    const void *ptrs[] = {q, k, v, la, dO, dSf, dq, dk, dv, dla};
    for (const void *p : ptrs)
        if (((uintptr_t)p & 15u) != 0) return GTR_GLA_ERR_ALIGN;
    const size_t es = dtype == GTR_GLA_F32 ? 4 : 2, tok = (size_t)B * H * gh * gw;
    const size_t nx = tok * 64 * es, nla = tok * 64 * 4, nfs = (size_t)B * H * 64 * 64 * 4;
    const void *ins[] = {q, k, v, dO};
    void *outs[] = {dq, dk, dv};
    for (void *o : outs) {
        for (const void *i : ins)
            if (overlaps(o, nx, i, nx)) return GTR_GLA_ERR_ALIAS;
        if (overlaps(o, nx, la, nla) || overlaps(o, nx, dSf, nfs) || overlaps(o, nx, dla, nla))
            return GTR_GLA_ERR_ALIAS;
        for (void *o2 : outs)
            if (o2 != o && overlaps(o, nx, o2, nx)) return GTR_GLA_ERR_ALIAS;
    }
    for (const void *i : ins)
        if (overlaps(dla, nla, i, nx)) return GTR_GLA_ERR_ALIAS;
    if (overlaps(dla, nla, la, nla) || overlaps(dla, nla, dSf, nfs)) return GTR_GLA_ERR_ALIAS;
    return GTR_GLA_OK;
}

template <typename T>
int run_bwd(const void *q, const void *k, const void *v, const float *la, const void *dO, const float *dSf,
            void *dq, void *dk, void *dv, float *dla, int B, int H, int gh, int gw, int dir, void *ws,
            cudaStream_t st) {
    return launch_bwd<T, 64, 64, 64>(static_cast<const T *>(q), static_cast<const T *>(k),
                                     static_cast<const T *>(v), la, static_cast<const T *>(dO), dSf,
                                     static_cast<T *>(dq), static_cast<T *>(dk), static_cast<T *>(dv), dla, B, H, gh,
                                     gw, dir, ws, st);
}

}  // namespace

extern "C" size_t gtr_gla_bwd_workspace_size(int B, int H, int grid_h, int grid_w, int d_k, int d_v) {
    if (B <= 0 || H <= 0 || grid_h <= 0 || grid_w <= 0 || d_k != 64 || d_v != 64 ||
        (long long)B * H > 65535 || (long long)grid_h * grid_w > (1LL << 22))
        return 0;
    const int n = grid_h * grid_w;
    return bwd_layout(B * H, (n + 63) / 64, 64, 64).total;
}

extern "C" int gtr_gla_bwd(const void *q, const void *k, const void *v, const float *log_alpha, const void *d_out,
                           const float *d_final_state, void *dq, void *dk, void *dv, float *dlog_alpha, int B, int H,
                           int grid_h, int grid_w, int d_k, int d_v, int direction, int dtype, void *workspace,
                           size_t workspace_bytes, cudaStream_t stream) {
    int rc = check_bwd(q, k, v, log_alpha, d_out, d_final_state, dq, dk, dv, dlog_alpha, B, H, grid_h, grid_w, d_k,
                       d_v, direction, dtype);
    if (rc) return rc;
    const size_t need = gtr_gla_bwd_workspace_size(B, H, grid_h, grid_w, d_k, d_v);
    if (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255u)) return GTR_GLA_ERR_WORKSPACE;
    {  // the workspace is written: it may overlap no tensor argument
        const size_t es = dtype == GTR_GLA_F32 ? 4 : 2, tok = (size_t)B * H * grid_h * grid_w;
        const size_t nx = tok * 64 * es, nla = tok * 64 * 4, nfs = (size_t)B * H * 64 * 64 * 4;
        const struct {
            const void *p;
            size_t n;
        } t[] = {{q, nx},  {k, nx},  {v, nx},  {d_out, nx},         {dq, nx},
                 {dk, nx}, {dv, nx}, {log_alpha, nla}, {dlog_alpha, nla}, {d_final_state, nfs}};
        for (const auto &e : t)
            if (overlaps(workspace, need, e.p, e.n)) return GTR_GLA_ERR_ALIAS;
    }
    if (dtype == GTR_GLA_F16)
        return run_bwd<__half>(q, k, v, log_alpha, d_out, d_final_state, dq, dk, dv, dlog_alpha, B, H, grid_h, grid_w,
                               direction, workspace, stream);
    if (dtype == GTR_GLA_BF16)
        return run_bwd<__nv_bfloat16>(q, k, v, log_alpha, d_out, d_final_state, dq, dk, dv, dlog_alpha, B, H, grid_h,
                                      grid_w, direction, workspace, stream);
    return run_bwd<float>(q, k, v, log_alpha, d_out, d_final_state, dq, dk, dv, dlog_alpha, B, H, grid_h, grid_w,
                          direction, workspace, stream);
}
