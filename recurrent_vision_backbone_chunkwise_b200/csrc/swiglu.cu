// swiglu.cu -- Spatial SwiGLU forward (GTR's channel mixer) on sm_100a:
// the two dense projections on the library's tensor-core GEMM (tc_gemm.cu),
// and one kernel between them for everything that is not a GEMM:
// the projection biases, the 3 x 3 depthwise convolution of the value branch
// over the patch grid, the SiLU gate and the product.
//
// "GTR: Gated Token Recurrence for Efficient Dense Prediction", x-techcon
// article, section 架构: a SwiGLU whose value branch gets a 3 x 3 per-channel
// convolution, so that neighbouring patches exchange information directly.
#include <map>
#include <mutex>
#include <tuple>

#include "../../include/gtr_swiglu.h"
#include "gla_common.cuh"
#include "gla_internal.h"
#include "io_pack.cuh"
#include "sm100.cuh"

namespace gtr {
namespace {

// ------------------------------------------------- fused depthwise / gate
//
// A persistent kernel, one CTA of 16 warps per SM.  Each CTA owns one block of
// kCh channels for the whole launch (its taps and biases are staged in shared
// memory once) and one stream of kTH x kTW token tiles: tiles s, s + S,
// s + 2S, ... over all images, the S CTAs of a channel block taking one stream
// each.  At any moment the CTAs thus read whole token rows of S neighbouring
// tiles, and each TMA row is kCh channels (512 bytes) long.
// Per tile, two TMA loads fill one slot of a kStages-deep ring: the
// (kTH+2) x (kTW+2) token halo of the value branch u (zero fill outside the
// grid is the convolution's padding) and the kTH x kTW gate tile g.  The warps
// form two groups of 8 taking alternate tiles; thread (channel group cg of 8
// channels, column col) computes a vertical strip of kTH tokens from shared
// memory, adds the biases, gates and writes h with 16-byte stores.  A warp
// covers 4 columns x 8 channel groups, so each of its shared-memory reads is
// four 128-byte rows and each weight read a broadcast.  Each warp counts itself
// out of a slot when done with it; the group's last warp out issues the loads
// of the tile kStages further on into it, so no warp waits to refill (and with
// no separate producer warp, 16 warps leave 128 registers a thread).
// Every wait is bounded: on a timeout the waiting thread latches
// kDevErrTimeout and stops, and before the CTA exits one thread waits
// (bounded) for every copy still in flight.

constexpr int kTW = 8, kTH = 4, kCh = 256;
constexpr int kStages = 4;
constexpr int kHaloBytes = (kTH + 2) * (kTW + 2) * kCh * 2;  // 30720
constexpr int kGBytes = kTH * kTW * kCh * 2;                 // 16384
constexpr int kStageBytes = kHaloBytes + kGBytes;             // 47104
// Weight rows: taps 0..8, b_g, then the bias of v for each of 16 border
// cases e = 4 * (top | 2 bottom) + (left | 2 right): b_dw + b_u times the sum
// of the taps that fall inside the grid there (the zero padding carries no
// b_u), so that no thread branches on where its token lies.
constexpr int kWRows = 10 + 16;
constexpr int kDwThreads = 32 * 16;
constexpr size_t kDwSmem = (size_t)kStages * kStageBytes + kWRows * kCh * 4 + kStages * 8 + 2 * kStages * 4 + 128;
static_assert(kHaloBytes % 128 == 0 && kStageBytes % 128 == 0, "stage alignment");
static_assert(kDwSmem <= 232448, "shared memory per CTA");

// Float index of channel c in weight row r: the 8 channels of group cg are two
// float4 at (2r)*32 + cg and (2r+1)*32 + cg, so that 32 consecutive groups
// read 512 contiguous bytes.
__host__ __device__ __forceinline__ int wslot(int r, int c) {
    return ((r * 2 + ((c >> 2) & 1)) * 32 + (c >> 3)) * 4 + (c & 3);
}

__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1,
                                            int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(sm100::smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(sm100::smem_u32(bar))
        : "memory");
}

// Bounded wait on an mbarrier phase with try_wait, which parks the thread in
// hardware between checks instead of spinning on the issue slots; gives up
// after about `limit_ns` of wall time.
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, uint64_t limit_ns = 2000000000ull) {
    if (sm100::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = sm100::global_timer_ns();
    while (true) {
        for (int i = 0; i < 16; ++i)
            if (sm100::mbar_try_wait(bar, parity)) return true;
        if (sm100::global_timer_ns() - t0 > limit_ns) return false;
    }
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;"
        : "=l"(d)
        : "l"(*reinterpret_cast<const uint64_t *>(&a)), "l"(*reinterpret_cast<const uint64_t *>(&b)));
    return *reinterpret_cast<float2 *>(&d);
}

__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// SiLU(g) * v for two lanes: SiLU(g) = g * sigmoid(g) and
// sigmoid(g) = (1 + tanh(g / 2)) / 2, so one hardware tanh per element (its
// relative error, about 2^-11, is that of the fp16 rounding of the result).
__device__ __forceinline__ float2 silu_mul2(float2 g, float2 v) {
    const float2 half = make_float2(0.5f, 0.5f);
    const float2 hg = sm100::fmul2(g, half);
    const float2 t = make_float2(tanh_approx(hg.x), tanh_approx(hg.y));
    return sm100::fmul2(sm100::ffma2(hg, t, hg), v);  // g/2 * (1 + t) * v
}

template <typename T>
__global__ void __launch_bounds__(kDwThreads, 1) swiglu_dw_gate_kernel(
    const __grid_constant__ CUtensorMap map_u, const __grid_constant__ CUtensorMap map_g,
    const float *__restrict__ b_gu, const float *__restrict__ w_dw, const float *__restrict__ b_dw,
    T *__restrict__ h, const float *__restrict__ b_down, T *__restrict__ b_down_io, int *err, int B, int gh,
    int gw, int F, int C, int cb0, int ncb, int tiles) {
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    // 128-byte aligned base, derived by pointer arithmetic so that every
    // access below stays a shared-memory access (not a generic one)
    uint8_t *smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
    float *sw = reinterpret_cast<float *>(smem + (size_t)kStages * kStageBytes);
    uint64_t *full = reinterpret_cast<uint64_t *>(sw + kWRows * kCh);
    int *released = reinterpret_cast<int *>(full + kStages);  // per slot: warps done with it
    int *last_issued = released + kStages;                      // per slot: last tile loaded, -1 if none
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cb = cb0 + (int)(blockIdx.x % ncb);
    const int S = (int)(gridDim.x / ncb), stream = (int)(blockIdx.x / ncb);
    const int n = stream < tiles ? (tiles - stream + S - 1) / S : 0;
    const int tiles_w = (gw + kTW - 1) / kTW, tiles_h = (gh + kTH - 1) / kTH;
    // loads of tile i of this stream into slot i % kStages
    auto issue = [&](int i) {
        const int s = i % kStages;
        const int tile = stream + i * S;
        const int b = tile / (tiles_w * tiles_h), r = tile % (tiles_w * tiles_h);
        const int y0 = (r / tiles_w) * kTH, x0 = (r % tiles_w) * kTW;
        uint8_t *st = smem + (size_t)s * kStageBytes;
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        tma_load_4d(st, &map_u, &full[s], F + cb * kCh, x0 - 1, y0 - 1, b);
        tma_load_4d_pol(st + kHaloBytes, &map_g, &full[s], cb * kCh, x0, y0, b, l2_policy_evict_first());
        last_issued[s] = i;
    };
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);  // the issuing thread's arrival with the byte count
            released[s] = 0;
            last_issued[s] = -1;
        }
        fence_mbar_init();
        tma_prefetch_desc(&map_u);
        tma_prefetch_desc(&map_g);
        for (int i = 0; i < kStages && i < n; ++i) issue(i);
    }
    for (int c = threadIdx.x; c < kCh; c += kDwThreads) {
        const int f = cb * kCh + c;
        const bool in = f < F;
        float w[9];
#pragma unroll
        for (int k = 0; k < 9; ++k) {
            w[k] = in ? w_dw[(size_t)f * 9 + k] : 0.f;
            sw[wslot(k, c)] = w[k];
        }
        const float bu = in ? b_gu[F + f] : 0.f, bd = in ? b_dw[f] : 0.f;
        sw[wslot(9, c)] = in ? b_gu[f] : 0.f;
        for (int e = 0; e < 16; ++e) {
            float inside = 0.f;
#pragma unroll
            for (int k = 0; k < 9; ++k) {
                const int a = k / 3, cc = k % 3;
                const bool out = (a == 0 && (e & 4)) || (a == 2 && (e & 8)) || (cc == 0 && (e & 1)) ||
                                 (cc == 2 && (e & 2));
                if (!out) inside += w[k];
            }
            sw[wslot(10 + e, c)] = bd + bu * inside;
        }
    }
    if (b_down_io && blockIdx.x == 0)
        for (int c = threadIdx.x; c < C; c += kDwThreads) b_down_io[c] = static_cast<T>(b_down[c]);
    __syncthreads();

    // ------------------------------------------------------ consumers
    const int grp = warp >> 3, wig = warp & 7;
    const int cg = (wig & 3) * 8 + (lane & 7), col = (wig >> 2) * 4 + (lane >> 3);
    const int f = cb * kCh + 8 * cg;
    const float4 *sw4 = reinterpret_cast<const float4 *>(sw);
    // eight consecutive floats of row r for this thread's channels, as pairs
    auto wrow = [&](int r, float2 *w) {
        const float4 lo4 = sw4[(2 * r) * 32 + cg], hi4 = sw4[(2 * r + 1) * 32 + cg];
        w[0] = make_float2(lo4.x, lo4.y);
        w[1] = make_float2(lo4.z, lo4.w);
        w[2] = make_float2(hi4.x, hi4.y);
        w[3] = make_float2(hi4.z, hi4.w);
    };
    for (int i = grp; i < n; i += 2) {
        const int s = i % kStages;
        if (!wait_phase(&full[s], (i / kStages) & 1)) {
            latch_error(err, kDevErrTimeout);
            break;
        }
        const int tile = stream + i * S;
        const int b = tile / (tiles_w * tiles_h), r = tile % (tiles_w * tiles_h);
        const int y0 = (r / tiles_w) * kTH, x = (r % tiles_w) * kTW + col;
        const uint8_t *st = smem + (size_t)s * kStageBytes;
        if (x < gw && f < F) {
            // start from the bias of v for the token's border case
            float2 acc[kTH][4];
            const int ecol = (x == 0 ? 1 : 0) | (x == gw - 1 ? 2 : 0);
#pragma unroll
            for (int j = 0; j < kTH; ++j) {
                const int y = y0 + j;
                wrow(10 + ((y == 0 ? 4 : 0) | (y == gh - 1 ? 8 : 0) | ecol), acc[j]);
            }
            // sum over taps (a, c): w[a][c] * u[y0 + j + a - 1, x + c - 1]
#pragma unroll
            for (int c = 0; c < 3; ++c) {
                float2 w[3][4];
#pragma unroll
                for (int a = 0; a < 3; ++a) wrow(3 * a + c, w[a]);
#pragma unroll
                for (int rr = 0; rr < kTH + 2; ++rr) {
                    const uint4 raw =
                        *reinterpret_cast<const uint4 *>(st + ((rr * (kTW + 2) + col + c) * kCh + 8 * cg) * 2);
                    float2 u[4];
                    unpack8<T>(raw, u);
#pragma unroll
                    for (int a = 0; a < 3; ++a) {
                        const int j = rr - a;
                        if (j >= 0 && j < kTH) {
#pragma unroll
                            for (int q = 0; q < 4; ++q) acc[j][q] = ffma2(w[a][q], u[q], acc[j][q]);
                        }
                    }
                }
            }
            float2 bg[4];
            wrow(9, bg);
#pragma unroll
            for (int j = 0; j < kTH; ++j) {
                const int y = y0 + j;
                if (y >= gh) break;
                const uint4 graw =
                    *reinterpret_cast<const uint4 *>(st + kHaloBytes + ((j * kTW + col) * kCh + 8 * cg) * 2);
                float2 g[4];
                unpack8<T>(graw, g);
                uint32_t o[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 hv = silu_mul2(fadd2(g[q], bg[q]), acc[j][q]);
                    o[q] = Pair<T>::pack(hv.x, hv.y);
                }
                const size_t m = ((size_t)b * gh + y) * gw + x;
                *reinterpret_cast<uint4 *>(h + m * (size_t)F + f) = make_uint4(o[0], o[1], o[2], o[3]);
            }
        }
        // release the slot; the group's last warp to do so refills it at once
        __syncwarp();
        if (lane == 0) {
            __threadfence_block();
            if (atomicAdd(&released[s], 1) == 7) {
                released[s] = 0;
                __threadfence_block();
                fence_proxy_async_smem();
                if (i + kStages < n) issue(i + kStages);
            }
        }
    }
    // no copy may still be landing in shared memory when the CTA exits
    // (only possible after a timeout above)
    __syncthreads();
    if (threadIdx.x == 0)
        for (int s = 0; s < kStages; ++s)
            if (last_issued[s] >= 0 && !wait_phase(&full[s], (last_issued[s] / kStages) & 1))
                latch_error(err, kDevErrTimeout);
}

struct SwLayout {
    size_t gu, h, bd, total;
};

SwLayout sw_layout(long long M, int C, int F, size_t es) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    SwLayout l;
    l.gu = 0;
    l.h = up((size_t)M * 2 * F * es);
    l.bd = up(l.h + (size_t)M * F * es);
    l.total = up(l.bd + (size_t)C * es);
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

int sm_count(int dev) {
    static int cache[64];
    if (!cache[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 0;
        cache[dev] = n;
    }
    return cache[dev];
}

// The fused depthwise / gate kernel over the projected [g | u] (token-major,
// 2F channels per token): two 4-D TMA views (channels, columns, rows, images),
// one per box shape.
int launch_dw_gate(int dtype, const void *gu, const float *b_gu, const float *w_dw, const float *b_dw, void *h,
                   const float *b_down, void *bd, int B, int gh, int gw, int F, int C, cudaStream_t st) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GTR_GLA_ERR_CUDA;
    const int sms = sm_count(dev);
    if (!sms) return GTR_GLA_ERR_CUDA;
    int *err = nullptr;
    int rc = error_word(&err);
    if (rc) return rc;
    const CUtensorMapDataType dt =
        dtype == GTR_GLA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const uint64_t row = 2ull * 2 * F;  // bytes per token
    const uint64_t dims[4] = {2ull * F, (uint64_t)gw, (uint64_t)gh, (uint64_t)B};
    const uint64_t strides[3] = {row, row * gw, row * gw * gh};
    const uint32_t box_u[4] = {kCh, kTW + 2, kTH + 2, 1}, box_g[4] = {kCh, kTW, kTH, 1};
    CUtensorMap mu, mg;
    if (encode_tile_map(&mu, gu, dt, 4, dims, strides, box_u, false) ||
        encode_tile_map(&mg, gu, dt, 4, dims, strides, box_g, false))
        return GTR_GLA_ERR_CUDA;
    const long long tiles_ll = (long long)B * ((gh + kTH - 1) / kTH) * ((gw + kTW - 1) / kTW);
    if (tiles_ll > (1LL << 30)) return GTR_GLA_ERR_SHAPE;
    const int tiles = (int)tiles_ll;
    const int ncb_all = (F + kCh - 1) / kCh;
    auto kern_h = swiglu_dw_gate_kernel<__half>;
    auto kern_b = swiglu_dw_gate_kernel<__nv_bfloat16>;
    if ((rc = ensure_smem(dtype == GTR_GLA_BF16 ? (const void *)kern_b : (const void *)kern_h, kDwSmem))) return rc;
    // one launch per group of at most `sms` channel blocks (a single launch
    // unless F > kCh * sms); S = sms / ncb CTAs (tile streams) per block
    for (int cb0 = 0; cb0 < ncb_all; cb0 += sms) {
        const int ncb = ncb_all - cb0 < sms ? ncb_all - cb0 : sms;
        int S = sms / ncb;
        if (S > tiles) S = tiles;
        const unsigned grid = (unsigned)(ncb * S);
        if (dtype == GTR_GLA_BF16)
            kern_b<<<grid, kDwThreads, kDwSmem, st>>>(mu, mg, b_gu, w_dw, b_dw, static_cast<__nv_bfloat16 *>(h),
                                                      b_down, cb0 == 0 ? static_cast<__nv_bfloat16 *>(bd) : nullptr,
                                                      err, B, gh, gw, F, C, cb0, ncb, tiles);
        else
            kern_h<<<grid, kDwThreads, kDwSmem, st>>>(mu, mg, b_gu, w_dw, b_dw, static_cast<__half *>(h), b_down,
                                                      cb0 == 0 ? static_cast<__half *>(bd) : nullptr, err, B, gh,
                                                      gw, F, C, cb0, ncb, tiles);
        note_launch();
        if (cudaPeekAtLastError() != cudaSuccess) return GTR_GLA_ERR_CUDA;
    }
    return GTR_GLA_OK;
}

}  // namespace

// The block after argument checks (shared with the backbone layer): y = x +
// ... when resid = x is given (the down projection's epilogue adds it; y may
// be x itself).
int swiglu_apply(const void *x, const void *w_gu, const float *b_gu, const float *w_dw, const float *b_dw,
                 const void *w_down, const float *b_down, const void *resid, void *y, int B, int grid_h,
                 int grid_w, int C, int F, int dtype, void *workspace, cudaStream_t stream) {
    const long long M = (long long)B * grid_h * grid_w;
    const SwLayout l = sw_layout(M, C, F, 2);
    int rc;
    char *ws = static_cast<char *>(workspace);
    void *gu = ws + l.gu, *h = ws + l.h, *bd = ws + l.bd;
    // 1. [g | u] without biases (the kernel adds them in fp32)
    rc = dense_gemm(dtype, M, 2 * F, C, x, w_gu, nullptr, nullptr, gu, stream);
    if (rc) return rc;
    // 2. biases, depthwise 3 x 3 on the value branch, SiLU gate, product
    rc = launch_dw_gate(dtype, gu, b_gu, w_dw, b_dw, h, b_down, bd, B, grid_h, grid_w, F, C, stream);
    if (rc) return rc;
    // 3. y = h W_d^T + b_d (+ resid): the bias (copied to the I/O dtype by the
    //    kernel above) and the residual in the GEMM's epilogue
    rc = dense_gemm(dtype, M, C, F, h, w_down, bd, resid, y, stream);
    if (rc) return rc;
    return GTR_GLA_OK;
}

}  // namespace gtr

using namespace gtr;

extern "C" size_t gtr_swiglu_workspace_size(int B, int grid_h, int grid_w, int C, int F, int dtype) {
    if (sw_validate_shape(B, grid_h, grid_w, C, F, dtype)) return 0;
    return sw_layout((long long)B * grid_h * grid_w, C, F, 2).total;
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
    const SwLayout l = sw_layout(M, C, F, es);
    if (!workspace || workspace_bytes < l.total || ((uintptr_t)workspace & 255u)) return GTR_GLA_ERR_WORKSPACE;
    if (overlap(workspace, l.total, y, ny) || overlap(workspace, l.total, x, ny) ||
        overlap(workspace, l.total, w_gu, (size_t)2 * F * C * es) ||
        overlap(workspace, l.total, w_down, (size_t)C * F * es) ||
        overlap(workspace, l.total, b_gu, (size_t)2 * F * 4) || overlap(workspace, l.total, w_dw, (size_t)F * 36) ||
        overlap(workspace, l.total, b_dw, (size_t)F * 4) || overlap(workspace, l.total, b_down, (size_t)C * 4))
        return GTR_GLA_ERR_ALIAS;
    return swiglu_apply(x, w_gu, b_gu, w_dw, b_dw, w_down, b_down, nullptr, y, B, grid_h, grid_w, C, F, dtype,
                        workspace, stream);
}
