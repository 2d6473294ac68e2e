// output_tail.cu -- the output tail of the token mixer on sm_100a: per-head
// RMS norm of the attention output with a weight, times SiLU of the output
// gate, heads merged channels-last (see include/gtr_output_tail.h).
//
// "GTR: Gated Token Recurrence for Efficient Dense Prediction", x-techcon
// article, section 算子: the operator benchmark leaves out the fusion of the
// operator's output tail; the tail itself is the reading stated in the header.
//
// HBM bound: per token-head it reads o and z (2 d_v bytes each) and writes y
// (2 d_v bytes), with d_v / 8 threads of 16-byte loads and stores; the head's
// sum of squares is reduced with shuffles inside those threads.
#include "../../include/gtr_output_tail.h"
#include "gla_common.cuh"
#include "gla_internal.h"
#include "io_pack.cuh"

#include <math.h>

namespace gtr {
namespace {

// One thread per 8 channels of a token-head; L = d_v / 8 consecutive lanes
// share a token-head, token-heads ordered (image, token, head) with the head
// fastest, so a warp's z and y accesses are contiguous.  Grid-stride over
// whole warps: every lane reaches the shuffles, lanes past the end compute on
// zeros and store nothing.
template <typename T, int L>
__global__ void __launch_bounds__(256, 8)
    output_tail_kernel(const T *__restrict__ o, const T *__restrict__ z, const float *__restrict__ w,
                       T *__restrict__ y, long long n_tok, int H, float inv_dv, float eps, long long total) {
    constexpr int DV = 8 * L;
    const int lane = threadIdx.x & 31, l = lane % L;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long base = (long long)blockIdx.x * blockDim.x + (threadIdx.x & ~31); base < total;
         base += stride) {
        const long long i = base + lane;
        const bool active = i < total;
        const long long th = i / L;  // token-head index: (b * n_tok + t) * H + h
        const int h = (int)(th % H);
        const long long bt = th / H;  // b * n_tok + t
        const long long b = bt / n_tok, t = bt % n_tok;
        uint4 ov = make_uint4(0, 0, 0, 0), zv = make_uint4(0, 0, 0, 0);
        if (active) {
            ov = __ldcs(reinterpret_cast<const uint4 *>(o + ((b * H + h) * n_tok + t) * DV + 8 * l));
            zv = __ldcs(reinterpret_cast<const uint4 *>(z + th * DV + 8 * l));
        }
        float2 of[4], zf[4];
        unpack8<T>(ov, of);
        unpack8<T>(zv, zf);
        float ss = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) ss = fmaf(of[q].x, of[q].x, fmaf(of[q].y, of[q].y, ss));
#pragma unroll
        for (int off = L / 2; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if (active) {
            const float r = rsqrtf(fmaf(ss, inv_dv, eps));
            const float4 w0 = __ldg(reinterpret_cast<const float4 *>(w + h * DV + 8 * l));
            const float4 w1 = __ldg(reinterpret_cast<const float4 *>(w + h * DV + 8 * l + 4));
            const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            uint32_t out[4];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                out[q] = Pair<T>::pack(of[q].x * r * wv[2 * q] * silu_f32(zf[q].x),
                                       of[q].y * r * wv[2 * q + 1] * silu_f32(zf[q].y));
            *reinterpret_cast<uint4 *>(y + th * DV + 8 * l) = make_uint4(out[0], out[1], out[2], out[3]);
        }
    }
}

bool overlap(const void *a, size_t na, const void *b, size_t nb) {
    const char *pa = (const char *)a, *pb = (const char *)b;
    return pa < pb + nb && pb < pa + na;
}

template <typename T, int L>
int launch_tail(const void *o, const void *z, const float *w, void *y, long long n_tok, long long B, int H,
                float eps, cudaStream_t st) {
    const long long total = B * n_tok * H * L;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return GTR_GLA_ERR_CUDA;
    // enough resident warps to cover the memory latency: 8 blocks of 256 per SM
    const long long want = (total + 255) / 256, cap = (long long)sms * 8;
    const unsigned grid = (unsigned)(want < cap ? want : cap);
    output_tail_kernel<T, L><<<grid, 256, 0, st>>>(static_cast<const T *>(o), static_cast<const T *>(z), w,
                                                   static_cast<T *>(y), n_tok, H, 1.f / (8 * L), eps, total);
    note_launch();
    return cudaPeekAtLastError() == cudaSuccess ? GTR_GLA_OK : GTR_GLA_ERR_CUDA;
}

}  // namespace
}  // namespace gtr

using namespace gtr;

extern "C" int gtr_output_tail_fwd(const void *o, const void *z, const float *w, void *y, int B, int H,
                                   int grid_h, int grid_w, int d_v, float eps, int dtype,
                                   cudaStream_t stream) {
    if (!o || !z || !w || !y) return GTR_GLA_ERR_NULL;
    if (B <= 0 || H <= 0 || grid_h <= 0 || grid_w <= 0) return GTR_GLA_ERR_SHAPE;
    const long long n_tok = (long long)grid_h * grid_w;
    if ((long long)B * n_tok * H > (1LL << 31)) return GTR_GLA_ERR_SHAPE;
    if (!(eps >= 0.f) || !isfinite(eps)) return GTR_GLA_ERR_SHAPE;
    if (d_v != 64 && d_v != 128) return GTR_GLA_ERR_HEAD_DIM;
    if (dtype != GTR_GLA_F16 && dtype != GTR_GLA_BF16) return GTR_GLA_ERR_DTYPE;
    const void *ptrs[] = {o, z, w, y};
    for (const void *p : ptrs)
        if (((uintptr_t)p & 15u) != 0) return GTR_GLA_ERR_ALIGN;
    const size_t n = (size_t)B * n_tok * H * d_v * 2;
    if (overlap(y, n, o, n) || overlap(y, n, z, n) || overlap(y, n, w, (size_t)H * d_v * 4))
        return GTR_GLA_ERR_ALIAS;
    if (dtype == GTR_GLA_BF16)
        return d_v == 64 ? launch_tail<__nv_bfloat16, 8>(o, z, w, y, n_tok, B, H, eps, stream)
                         : launch_tail<__nv_bfloat16, 16>(o, z, w, y, n_tok, B, H, eps, stream);
    return d_v == 64 ? launch_tail<__half, 8>(o, z, w, y, n_tok, B, H, eps, stream)
                     : launch_tail<__half, 16>(o, z, w, y, n_tok, B, H, eps, stream);
}
