// gla_fused.cu -- single-kernel chunkwise GLA forward on sm_100a tensor cores
// (fp16 / bf16 I/O, d_k = d_v = 64, chunk 64).
//
// The chunkwise reorganisation of "GTR: Gated Token Recurrence for Efficient
// Dense Prediction" (x-techcon article, section 算子) -- chunks compute their
// own state contribution in parallel, boundary states are passed along, each
// chunk's output is produced in parallel, scores stay on chip -- mapped onto
// one launch of 256-thread CTAs, two per SM:
//
//   * each CTA owns a segment of L consecutive 64-token chunks of one (b,h)
//     (the host picks L so that the whole grid is resident at once);
//   * pre-pass: the segment's aggregate state contribution, transposed,
//       A_seg^T = sum_c V_c^T (k_c . e^{G_after(c) + g_c - b_c})
//     and its gate totals are accumulated in TMEM (chunks visited last to
//     first, so every factor is <= 1) and published to the workspace;
//   * boundary pass: once every earlier segment of the same (b,h) has
//     published its aggregate, the incoming state is folded in one sweep,
//     nearest segment first: S_in = sum_j diag(e^{G(j..seg)}) A_j.  The fold
//     order is fixed, so results are bitwise reproducible, and no segment
//     waits on another's boundary pass (only on its pre-pass);
//   * main pass, chunk by chunk, with the fp32 state kept in TMEM as S^T:
//       MMA1 (tf32, M=64,N=128,K=64):  [scores | o] = Q^ [K~ ; S_in^T]^T
//         Q^ = q . e^{b},  K~ = k . e^{-b}   (b: in-chunk inclusive log-gate sums)
//       causal mask of the scores on CUDA cores, re-quantised to f16/bf16,
//       MMA2a (f16/bf16, M=64,N=64,K=64):  o += A V
//       MMA2b (f16/bf16, M=64,N=64,K=64):  dS^T = V^T K^,  K^ = k . e^{g - b}
//       S^T <- S^T diag(e^{g}) + dS^T;  o stored at the tokens' raster rows.
//     The gate factors come from running products of alpha = e^{log_alpha}
//     (one exponential per element).
//   Chunks whose in-chunk gate span exceeds kSpanLimit (e^{-b} would leave
//   fp32 range) take an exact CUDA-core path for the scores.
//
// Tiles are fetched in scan order by cp.async row copies (a per-chunk table of
// raster rows), so every scan direction reads and writes the row-major grid in
// place.  Every M=64 result lands in TMEM lanes 32(r/16) + r%16 (lanes 0-15
// of each warp's quadrant), so row r is handled by lane r%16 of the warps of
// quadrant r/16; each of the two warps of a quadrant takes 32 columns.
#include <type_traits>

#include "gla_common.cuh"
#include "gla_internal.h"
#include "sm100.cuh"

namespace gtr {
using namespace sm100;

namespace {

constexpr int FC = 64;              // tokens per chunk
constexpr int FD = 64;              // d_k = d_v
constexpr int kThreads = 256;       // 8 warps: two per TMEM lane quadrant
constexpr int kMaxSegments = 64;    // segments per (b,h); bounds the look-back fold
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kSpanLimit = 80.f;  // max -g (natural log) for the factorised scores

// shared-memory map (byte offsets from a 1024-aligned base)
constexpr uint32_t OFF_Q = 0;        // q tile    [64 tok][128 B]  SW128
constexpr uint32_t OFF_K = 8192;     // k tile    [64 tok][128 B]  SW128
constexpr uint32_t OFF_V = 16384;    // v tile    [64 tok][128 B]  SW128 (MMA2 B, MN-major)
constexpr uint32_t OFF_LA = 24576;   // log_alpha [64 tok][256 B]  fp32
constexpr uint32_t OFF_QH = 40960;   // MMA1 A:  Q^ tf32 K-major [kc 2][64][128 B]
constexpr uint32_t OFF_B1 = 57344;   // MMA1 B: tf32 K-major [kc 2][128 rows][128 B]:
                                     //   rows 0-63 K~ (tokens), rows 64-127 S_in^T (value dims)
constexpr uint32_t OFF_A = 90112;    // A (masked scores) f16/bf16 K-major [64 t][128 B]
constexpr uint32_t OFF_KH = 98304;   // K^ f16/bf16 K-major [64 i][128 B]
constexpr uint32_t OFF_MISC = 106496;
// pre-pass stage 1 (the operand tiles are idle during the pre-pass)
constexpr uint32_t OFF_K1 = OFF_QH, OFF_V1 = OFF_QH + 8192, OFF_LA1 = OFF_B1;
constexpr uint32_t MISC_TOT = 0;     // [8][64] fp32 row-group totals of log_alpha
constexpr uint32_t MISC_G = 2048;    // [64] fp32 e^{g} of the current chunk
constexpr uint32_t MISC_GA = 2304;   // [64] fp32 pre-pass: gate sums of later chunks
constexpr uint32_t MISC_ROW = 2816;  // [2][64] int: global row index of each token of a chunk
constexpr uint32_t MISC_BYTES = 4096;
constexpr uint32_t SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;  // + alignment slack
constexpr uint32_t kTmemCols = 256;
// TMEM columns (all M=64 results): scores, output o, dS^T, state S^T
constexpr uint32_t TM_RAW = 0, TM_O = 64, TM_DS = 128, TM_S = 192;

struct FusedParams {
    const void *q, *k, *v;
    const float *la;
    void *out;
    float *final_state;
    float *agg;    // [BH*P][64*64] segment aggregate states, transposed ([j][i])
    float *aggg;   // [BH*P][64]    segment log-gate totals
    int *flag;     // [BH*P] 0 empty, 1 aggregate published
    unsigned *ctr; // [0] ticket, [1] finished CTAs
    int *err;
    int n, gh, gw, dir, nc, P, L, BH;
};

__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(int *p, int v) {
    asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded wait (about 2 s) for a non-zero flag; 0 (and a latched error) if it
// never came.
__device__ int wait_flag(const int *f, int *err) {
    const uint64_t t0 = global_timer_ns();
    while (true) {
        const int v = ld_acquire(f);
        if (v != 0) return v;
        if (global_timer_ns() - t0 > 2000000000ull) break;
        __nanosleep(32);
    }
    latch_error(err, kDevErrTimeout);
    return 0;
}

template <typename T> struct Pack2;
template <> struct Pack2<__half> {
    static __device__ __forceinline__ uint32_t pack(float a, float b) {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&h);
    }
    static __device__ __forceinline__ float2 unpack(uint32_t w) {
        return __half22float2(*reinterpret_cast<__half2 *>(&w));
    }
};
template <> struct Pack2<__nv_bfloat16> {
    static __device__ __forceinline__ uint32_t pack(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&h);
    }
    static __device__ __forceinline__ float2 unpack(uint32_t w) {
        return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&w));
    }
};

// element (row, col) of a [rows][64] 16-bit SW128 tile
template <typename T>
__device__ __forceinline__ float tile16(const uint8_t *tile, int row, int col) {
    return to_f32(*reinterpret_cast<const T *>(tile + sw128(row, col >> 3) + (col & 7) * 2));
}

// byte offset of tf32 element (row, k) in a K-major tile with K = 64 and
// `rows` rows per 32-element K block
template <int rows>
__device__ __forceinline__ uint32_t tf32_kmaj(int row, int k) {
    return (k >> 5) * (rows * 128) + sw128(row, (k & 31) >> 2) + (k & 3) * 4;
}

// A shared-memory descriptor advanced by `bytes` (the start address field
// holds addr >> 4 in its low 14 bits; smem addresses stay far below 256 KiB).
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t bytes) {
    return d + (uint64_t)(bytes >> 4);
}

template <typename T>
__device__ __forceinline__ uint4 pack8(const float *x) {
    uint4 w;
    w.x = Pack2<T>::pack(x[0], x[1]);
    w.y = Pack2<T>::pack(x[2], x[3]);
    w.z = Pack2<T>::pack(x[4], x[5]);
    w.w = Pack2<T>::pack(x[6], x[7]);
    return w;
}

// One thread waits (bounded) for an mbarrier phase, then the CTA barrier
// releases everyone: waiting warps sleep in bar.sync instead of spinning.
// Must be reached by every thread.  Returns false if the wait gave up (or an
// earlier one did: then nobody waits any more).
__device__ __forceinline__ bool cta_wait(uint64_t *bar, uint32_t parity, bool ok, int *s_ok) {
    if (threadIdx.x == 0) *s_ok = (ok && mbar_wait(bar, parity)) ? 1 : 0;
    __syncthreads();
    return *s_ok != 0;
}

// Global row (b,h plane offset included) of every token of chunk c, in scan
// order; rows past the end of the sequence repeat the last token (they are
// masked in the arithmetic).  Threads 0..63 fill one table.
__device__ __forceinline__ void fill_rows(const FusedParams &p, int bh, int c, int *rows) {
    const int u = threadIdx.x;
    if (u < FC)
        rows[u] = bh * p.n + scan_to_raster(min(c * FC + u, p.n - 1), p.n, p.gh, p.gw, p.dir);
}

// cp.async copies of a 64-row tile of 16-bit [.., 64] rows into a SW128 tile
// (2 pieces of 16 B per thread).
__device__ __forceinline__ void copy_tile16(uint8_t *dst, const void *src, const int *rows) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int pc = threadIdx.x + kThreads * e;
        const int u = pc >> 3, w = pc & 7;
        cp_async16(dst + sw128(u, w),
                   static_cast<const uint8_t *>(src) + (size_t)rows[u] * 128 + w * 16);
    }
}

// cp.async copies of a 64-row tile of fp32 [.., 64] rows (4 pieces per thread).
__device__ __forceinline__ void copy_tile32(uint8_t *dst, const float *src, const int *rows) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int pc = threadIdx.x + kThreads * e;
        const int u = pc >> 4, w = pc & 15;
        cp_async16(dst + u * 256 + w * 16,
                   reinterpret_cast<const uint8_t *>(src) + (size_t)rows[u] * 256 + w * 16);
    }
}

// Gate factors of a 64-token chunk for the columns (p2, p2+1) and the rows
// [8 r8, 8 r8 + 8) of this thread: alpha = e^{log_alpha} per element, the
// chunk's log-gate totals g (returned), and the row-group log sums that place
// the thread's rows inside the chunk (pre: groups before, suf: groups after).
// Rows >= len count as alpha = 1.  Contains one __syncthreads.
struct GateRows {
    float a0[8], a1[8];  // alpha of the 8 rows, columns p2 and p2+1
    float pre0, pre1;    // sum of log_alpha over the rows before this group
    float suf0, suf1;    // sum of log_alpha over the rows after this group
    float g0, g1;        // chunk totals
};

__device__ __forceinline__ void gate_rows(const float *sLA, float *sTot, int p2, int r8, int len,
                                          GateRows &G) {
    float l0 = 0.f, l1 = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int u = 8 * r8 + k;
        float2 x = make_float2(0.f, 0.f);
        if (u < len) x = *reinterpret_cast<const float2 *>(sLA + u * 64 + p2);
        l0 += x.x;
        l1 += x.y;
        G.a0[k] = fast_exp2(x.x * kLog2e);
        G.a1[k] = fast_exp2(x.y * kLog2e);
    }
    *reinterpret_cast<float2 *>(sTot + r8 * 64 + p2) = make_float2(l0, l1);
    __syncthreads();
    float o0 = 0.f, o1 = 0.f, t0 = 0.f, t1 = 0.f;
#pragma unroll
    for (int gidx = 0; gidx < 8; ++gidx) {
        const float2 t = *reinterpret_cast<const float2 *>(sTot + gidx * 64 + p2);
        if (gidx < r8) {
            o0 += t.x;
            o1 += t.y;
        }
        t0 += t.x;
        t1 += t.y;
    }
    G.pre0 = o0;
    G.pre1 = o1;
    G.suf0 = t0 - o0 - l0;
    G.suf1 = t1 - o1 - l1;
    G.g0 = t0;
    G.g1 = t1;
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads, 2) gla_fused_kernel(const __grid_constant__ FusedParams p) {
    using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sQ = sm + OFF_Q, *sK = sm + OFF_K, *sV = sm + OFF_V;
    float *sLA = reinterpret_cast<float *>(sm + OFF_LA);
    uint8_t *sQH = sm + OFF_QH, *sB1 = sm + OFF_B1;
    uint8_t *sA = sm + OFF_A, *sKh = sm + OFF_KH;
    float *sTot = reinterpret_cast<float *>(sm + OFF_MISC + MISC_TOT);
    float *sGam = reinterpret_cast<float *>(sm + OFF_MISC + MISC_G);  // e^{g} of the chunk
    float *sGa = reinterpret_cast<float *>(sm + OFF_MISC + MISC_GA);
    int *sRow = reinterpret_cast<int *>(sm + OFF_MISC + MISC_ROW);  // [2][64]

    // bar_st: pre-pass stages; bar_ld / bar_v: main-pass q,k,log_alpha / v.
    __shared__ uint64_t bar_st[2], bar_ld, bar_v, bar_mma;
    __shared__ uint32_t s_tmem;
    __shared__ int s_ticket, s_last, s_fail, s_ok;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, ch = warp >> 2;  // TMEM lane quadrant, column half
    const bool act = lane < 16;                 // lanes holding M=64 rows
    const int row16 = 16 * quad + (lane & 15);  // row of the M=64 results this lane holds
    const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
    const int p2 = 2 * (tid & 31), r8 = tid >> 5;  // gate math: columns p2, p2+1; rows 8 r8..
    constexpr uint32_t kFmt = BF16 ? 1u : 0u;
    const uint32_t id_tf = idesc(2, 64, 128, 0, 0);     // tf32, both K-major, N = 128
    const uint32_t id_av = idesc(kFmt, 64, 64, 0, 1);   // A K-major, V as B (MN-major)
    const uint32_t id_vk = idesc(kFmt, 64, 64, 1, 0);   // V^T as A (MN-major), K^ as B

    if (tid == 0) {
        mbar_init(&bar_st[0], kThreads);
        mbar_init(&bar_st[1], kThreads);
        mbar_init(&bar_ld, kThreads);
        mbar_init(&bar_v, kThreads);
        mbar_init(&bar_mma, 1);
        fence_mbar_init();
        s_ticket = (int)atomicAdd(&p.ctr[0], 1u);
    }
    if (warp == 1) {
        tmem_alloc(&s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tbase = s_tmem;
    const int ticket = s_ticket;
    const int bh = ticket / p.P, seg = ticket % p.P;
    const int c_begin = seg * p.L, c_end = min(c_begin + p.L, p.nc);
    const size_t slot = (size_t)bh * p.P + seg;

    uint32_t ph_st0 = 0, ph_st1 = 0, ph_ld = 0, ph_v = 0, ph_mma = 0;
    bool ok = true;  // every bounded wait succeeded

    // ------------------------------------------------------------- pre-pass
    // A_seg^T accumulates in TM_DS:  sum_c V_c^T (k_c . e^{G_after + g_c - b})
    if (seg < p.P - 1) {
        const int nl = c_end - c_begin;
        if (tid < 64) sGa[tid] = 0.f;
        fill_rows(p, bh, c_end - 1, sRow);
        if (nl > 1) fill_rows(p, bh, c_end - 2, sRow + 64);
        __syncthreads();
        copy_tile16(sK, p.k, sRow);
        copy_tile32(reinterpret_cast<uint8_t *>(sLA), p.la, sRow);
        copy_tile16(sV, p.v, sRow);
        cp_async_arrive(&bar_st[0]);
        if (nl > 1) {
            copy_tile16(sm + OFF_K1, p.k, sRow + 64);
            copy_tile32(sm + OFF_LA1, p.la, sRow + 64);
            copy_tile16(sm + OFF_V1, p.v, sRow + 64);
            cp_async_arrive(&bar_st[1]);
        }
        for (int idx = 0; idx < nl; ++idx) {
            const int c = c_end - 1 - idx, st = idx & 1;
            const int len = min(FC, p.n - c * FC);
            const uint8_t *kt = st ? sm + OFF_K1 : sK;
            const float *lat = reinterpret_cast<const float *>(st ? sm + OFF_LA1 : sm + OFF_LA);
            const uint8_t *vt = st ? sm + OFF_V1 : sV;
            if (st == 0) {
                ok = cta_wait(&bar_st[0], ph_st0, ok, &s_ok);
                ph_st0 ^= 1;
            } else {
                ok = cta_wait(&bar_st[1], ph_st1, ok, &s_ok);
                ph_st1 ^= 1;
            }
            GateRows G;
            gate_rows(lat, sTot, p2, r8, len, G);
            {
                const float2 ga = *reinterpret_cast<const float2 *>(sGa + p2);
                // e^{G_after + g - b_u} = e^{G_after} * prod of the alphas after u
                float e0 = fast_exp2((ga.x + G.suf0) * kLog2e), e1 = fast_exp2((ga.y + G.suf1) * kLog2e);
                float kh0[8], kh1[8];
#pragma unroll
                for (int k = 7; k >= 0; --k) {
                    const int u = 8 * r8 + k;
                    float2 kv = make_float2(0.f, 0.f);
                    if (u < len)
                        kv = Pack2<T>::unpack(*reinterpret_cast<const uint32_t *>(
                            kt + sw128(u, p2 >> 3) + (p2 & 7) * 2));
                    kh0[k] = kv.x * e0;
                    kh1[k] = kv.y * e1;
                    e0 *= G.a0[k];
                    e1 *= G.a1[k];
                }
                *reinterpret_cast<uint4 *>(sKh + sw128(p2, r8)) = pack8<T>(kh0);
                *reinterpret_cast<uint4 *>(sKh + sw128(p2 + 1, r8)) = pack8<T>(kh1);
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            __syncthreads();
            tc_fence_after_sync();
            if (r8 == 7) {  // the last row group holds the chunk totals of columns p2, p2+1
                float2 ga = *reinterpret_cast<float2 *>(sGa + p2);
                ga.x += G.g0;
                ga.y += G.g1;
                *reinterpret_cast<float2 *>(sGa + p2) = ga;
            }
            if (tid == 0) {
                fence_proxy_async_smem();  // v landed by cp.async, observed by this thread
                const uint64_t vd = sdesc_sw128(smem_u32(vt), 8192, 1024);
                const uint64_t kd = sdesc_sw128(smem_u32(sKh), 16, 1024);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(tbase + TM_DS, desc_add(vd, ks * 2048), desc_add(kd, ks * 32), id_vk,
                            (idx > 0 || ks > 0) ? 1u : 0u);
                mma_commit(&bar_mma);
            }
            if (idx + 2 < nl) fill_rows(p, bh, c - 2, sRow + 64 * st);
            ok = cta_wait(&bar_mma, ph_mma, ok, &s_ok);
            ph_mma ^= 1;
            tc_fence_after_sync();
            if (idx + 2 < nl) {  // this stage is free again: fetch chunk c - 2 into it
                const int *rows = sRow + 64 * st;
                copy_tile16(st ? sm + OFF_K1 : sK, p.k, rows);
                copy_tile32(st ? sm + OFF_LA1 : sm + OFF_LA, p.la, rows);
                copy_tile16(st ? sm + OFF_V1 : sV, p.v, rows);
                cp_async_arrive(&bar_st[st]);
            }
        }
        // publish the aggregate A_seg^T ([j][i]) and the gate totals
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint32_t r[16];
            const int cb = 32 * ch + 16 * hh;
            tmem_ld16(tbase + TM_DS + lane_off + cb, r);
            tmem_ld_wait();
            if (act) {
                const size_t off = slot * 4096 + row16 * 64 + cb;
#pragma unroll
                for (int e = 0; e < 16; e += 4) {
                    const float4 v4 = make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                                                  __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
                    *reinterpret_cast<float4 *>(p.agg + off + e) = v4;
                }
            }
        }
        if (tid < 64) p.aggg[slot * 64 + tid] = sGa[tid];
        __threadfence();
        tc_fence_before_sync();
        __syncthreads();
        tc_fence_after_sync();
        if (tid == 0) st_release(p.flag + slot, 1);
    }

    // first main-pass chunk: its loads overlap the boundary pass
    fill_rows(p, bh, c_begin, sRow + 64 * (c_begin & 1));
    __syncthreads();
    {
        const int *rows = sRow + 64 * (c_begin & 1);
        copy_tile16(sQ, p.q, rows);
        copy_tile16(sK, p.k, rows);
        copy_tile32(reinterpret_cast<uint8_t *>(sLA), p.la, rows);
        cp_async_arrive(&bar_ld);
        copy_tile16(sV, p.v, rows);
        cp_async_arrive(&bar_v);
    }

    // -------------------------------------------------------- boundary pass
    // S_in^T (fp32, [j][i] row-major) is assembled in the A/K^ tiles' space.
    float *sSin = reinterpret_cast<float *>(sA);
    if (seg > 0) {
        // 1. every earlier segment of this (b,h) must have published its
        //    aggregate (bounded waits, one lane per predecessor)
        if (warp == 0) {
            int fail = 0;
            for (int j = lane; j < seg; j += 32)
                if (wait_flag(p.flag + (size_t)bh * p.P + j, p.err) == 0) fail = 1;
            fail = __any_sync(0xffffffffu, fail);
            if (lane == 0) s_fail = fail;
        }
        __syncthreads();
        const int nfold = seg;
        if (s_fail) ok = false;
        // 2. per key dim i: scale of the term of segment seg-1-d, e^{sum of the
        //    log gates of the d segments between it and this one} (in QH's space)
        float *sAg = reinterpret_cast<float *>(sQH);  // [nfold][64], nfold < kMaxSegments
        for (int e = tid; e < nfold * 64; e += kThreads)
            sAg[e] = __ldcg(p.aggg + ((size_t)bh * p.P + (seg - 1 - (e >> 6))) * 64 + (e & 63));
        __syncthreads();
        if (tid < 64) {
            float acc = 0.f;
            for (int d = 0; d < nfold; ++d) {
                const float a = sAg[d * 64 + tid];
                sAg[d * 64 + tid] = fast_exp2(acc * kLog2e);
                acc += a;
            }
        }
        __syncthreads();
        // 3. fold, nearest segment first (a fixed order: the result does not
        //    depend on timing): thread -> (row j, 16 columns i)
        {
            const int j = tid >> 2, c0 = 16 * (tid & 3);
            float acc[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) acc[e] = 0.f;
            // the loads of kFoldBatch aggregates are all issued before any of
            // them is consumed, so several L2 round trips overlap
            constexpr int kFoldBatch = 4;
            const float *base = p.agg + (size_t)bh * p.P * 4096 + j * 64 + c0;
            for (int d0 = 0; d0 < nfold; d0 += kFoldBatch) {
                float4 v[kFoldBatch][4];
#pragma unroll
                for (int b = 0; b < kFoldBatch; ++b) {
                    const int d = min(d0 + b, nfold - 1);
                    const float *src = base + (size_t)(seg - 1 - d) * 4096;
#pragma unroll
                    for (int q = 0; q < 4; ++q) v[b][q] = __ldcg(reinterpret_cast<const float4 *>(src + 4 * q));
                }
#pragma unroll
                for (int b = 0; b < kFoldBatch; ++b) {
                    if (d0 + b < nfold) {
                        const float *sc = sAg + (d0 + b) * 64 + c0;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float4 s4 = *reinterpret_cast<const float4 *>(sc + 4 * q);
                            acc[4 * q] = fmaf(s4.x, v[b][q].x, acc[4 * q]);
                            acc[4 * q + 1] = fmaf(s4.y, v[b][q].y, acc[4 * q + 1]);
                            acc[4 * q + 2] = fmaf(s4.z, v[b][q].z, acc[4 * q + 2]);
                            acc[4 * q + 3] = fmaf(s4.w, v[b][q].w, acc[4 * q + 3]);
                        }
                    }
                }
            }
#pragma unroll
            for (int q4 = 0; q4 < 16; q4 += 4)
                *reinterpret_cast<float4 *>(sSin + j * 64 + c0 + q4) =
                    make_float4(acc[q4], acc[q4 + 1], acc[q4 + 2], acc[q4 + 3]);
        }
        __syncthreads();
    } else {
        for (int e = tid; e < 4096; e += kThreads) sSin[e] = 0.f;
        __syncthreads();
    }
    // S_in^T -> TMEM state and the tf32 operand (rows j, K = i)
    {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int cb = 32 * ch + 16 * hh;
            uint32_t r[16];
            const float *src = sSin + row16 * 64 + cb;
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
                const float4 v4 = act ? *reinterpret_cast<const float4 *>(src + e) : make_float4(0.f, 0.f, 0.f, 0.f);
                r[e] = __float_as_uint(v4.x);
                r[e + 1] = __float_as_uint(v4.y);
                r[e + 2] = __float_as_uint(v4.z);
                r[e + 3] = __float_as_uint(v4.w);
            }
            tmem_st16(tbase + TM_S + lane_off + cb, r);
            if (act) {
#pragma unroll
                for (int e = 0; e < 16; e += 4)
                    *reinterpret_cast<uint4 *>(sB1 + tf32_kmaj<128>(64 + row16, cb + e)) =
                        make_uint4(tf32_round(__uint_as_float(r[e])), tf32_round(__uint_as_float(r[e + 1])),
                                   tf32_round(__uint_as_float(r[e + 2])), tf32_round(__uint_as_float(r[e + 3])));
            }
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        tc_fence_after_sync();
    }

    // ------------------------------------------------------------ main pass
    for (int c = c_begin; c < c_end; ++c) {
        const int len = min(FC, p.n - c * FC);
        const int *rows = sRow + 64 * (c & 1);
        int *rows_next = sRow + 64 * ((c + 1) & 1);
        const bool more = c + 1 < c_end;
        if (c == c_begin) {  // later chunks wait for their q,k,log_alpha at the end of the previous one
            ok = cta_wait(&bar_ld, ph_ld, ok, &s_ok);
            ph_ld ^= 1;
        }
        // ---- gate factors and operands
        GateRows G;
        gate_rows(sLA, sTot, p2, r8, len, G);
        if (r8 == 7)
            *reinterpret_cast<float2 *>(sGam + p2) =
                make_float2(fast_exp2(G.g0 * kLog2e), fast_exp2(G.g1 * kLog2e));
        if (more) fill_rows(p, bh, c + 1, rows_next);
        const bool my_unsafe = (-G.g0 > kSpanLimit) || (-G.g1 > kSpanLimit);
        {
            // Q^ = q . e^{b_u}: running product of the alphas up to u
            float e0 = fast_exp2(G.pre0 * kLog2e), e1 = fast_exp2(G.pre1 * kLog2e);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int u = 8 * r8 + k;
                float2 qv = make_float2(0.f, 0.f);
                if (u < len)
                    qv = Pack2<T>::unpack(
                        *reinterpret_cast<const uint32_t *>(sQ + sw128(u, p2 >> 3) + (p2 & 7) * 2));
                e0 *= G.a0[k];
                e1 *= G.a1[k];
                *reinterpret_cast<uint2 *>(sQH + tf32_kmaj<64>(u, p2)) =
                    make_uint2(tf32_round(qv.x * e0), tf32_round(qv.y * e1));
            }
            // K^ = k . e^{g - b_u} (product of the alphas after u), K~ = K^ . e^{-g}
            float f0 = fast_exp2(G.suf0 * kLog2e), f1 = fast_exp2(G.suf1 * kLog2e);
            const float m0 = my_unsafe ? 0.f : fast_exp2(-G.g0 * kLog2e);
            const float m1 = my_unsafe ? 0.f : fast_exp2(-G.g1 * kLog2e);
            float kh0[8], kh1[8];
#pragma unroll
            for (int k = 7; k >= 0; --k) {
                const int u = 8 * r8 + k;
                float2 kv = make_float2(0.f, 0.f);
                if (u < len)
                    kv = Pack2<T>::unpack(
                        *reinterpret_cast<const uint32_t *>(sK + sw128(u, p2 >> 3) + (p2 & 7) * 2));
                kh0[k] = kv.x * f0;
                kh1[k] = kv.y * f1;
                *reinterpret_cast<uint2 *>(sB1 + tf32_kmaj<128>(u, p2)) =
                    make_uint2(tf32_round(kh0[k] * m0), tf32_round(kh1[k] * m1));
                f0 *= G.a0[k];
                f1 *= G.a1[k];
            }
            *reinterpret_cast<uint4 *>(sKh + sw128(p2, r8)) = pack8<T>(kh0);
            *reinterpret_cast<uint4 *>(sKh + sw128(p2 + 1, r8)) = pack8<T>(kh1);
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        const int unsafe = __syncthreads_or(my_unsafe);
        tc_fence_after_sync();
        if (tid == 0) {  // [scores | o] = Q^ [K~ ; S_in^T]^T
            const uint64_t ad = sdesc_sw128(smem_u32(sQH), 16, 1024);
            const uint64_t bd = sdesc_sw128(smem_u32(sB1), 16, 1024);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_tf32(tbase + TM_RAW, desc_add(ad, (ks >> 2) * 8192 + (ks & 3) * 32),
                         desc_add(bd, (ks >> 2) * 16384 + (ks & 3) * 32), id_tf, ks > 0 ? 1u : 0u);
            mma_commit(&bar_mma);
        }
        if (unsafe) {
            // the exact score path needs b (log2 domain) of every row: keep it in sLA
            float c0 = G.pre0, c1 = G.pre1;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int u = 8 * r8 + k;
                float2 *pl = reinterpret_cast<float2 *>(sLA + u * 64 + p2);
                if (u < len) {
                    const float2 x = *pl;
                    c0 += x.x;
                    c1 += x.y;
                }
                *pl = make_float2(c0 * kLog2e, c1 * kLog2e);
            }
        } else if (more) {
            copy_tile16(sQ, p.q, rows_next);
            copy_tile16(sK, p.k, rows_next);
            copy_tile32(reinterpret_cast<uint8_t *>(sLA), p.la, rows_next);
            cp_async_arrive(&bar_ld);
        }
        ok = cta_wait(&bar_mma, ph_mma, ok, &s_ok);
        ph_mma ^= 1;
        tc_fence_after_sync();
        // ---- causal mask of the scores -> A (rows t, K = s)
        if (!unsafe) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t r[16];
                tmem_ld16(tbase + TM_RAW + lane_off + 32 * ch + 16 * hh, r);
                tmem_ld_wait();
                if (act) {
                    const int t = row16;
                    float a[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int s = 32 * ch + 16 * hh + e;
                        a[e] = (s <= t) ? __uint_as_float(r[e]) : 0.f;
                    }
                    *reinterpret_cast<uint4 *>(sA + sw128(t, 4 * ch + 2 * hh)) = pack8<T>(a);
                    *reinterpret_cast<uint4 *>(sA + sw128(t, 4 * ch + 2 * hh + 1)) = pack8<T>(a + 8);
                }
            }
        } else {
            __syncthreads();  // b of every row is in sLA
            // exact scores A[t,s] = sum_i q_ti k_si 2^{b_ti - b_si}, s <= t (every factor <= 1)
            const int t = tid >> 2, s0 = 16 * (tid & 3);
            float a[16];
#pragma unroll 1
            for (int e = 0; e < 16; ++e) {
                const int s = s0 + e;
                float acc = 0.f;
                if (s <= t && t < len) {
                    for (int i = 0; i < FD; ++i)
                        acc = fmaf(tile16<T>(sQ, t, i) * tile16<T>(sK, s, i),
                                   fast_exp2(sLA[t * 64 + i] - sLA[s * 64 + i]), acc);
                }
                a[e] = acc;
            }
            *reinterpret_cast<uint4 *>(sA + sw128(t, s0 >> 3)) = pack8<T>(a);
            *reinterpret_cast<uint4 *>(sA + sw128(t, (s0 >> 3) + 1)) = pack8<T>(a + 8);
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        ok = cta_wait(&bar_v, ph_v, ok, &s_ok);  // also publishes the A rows
        ph_v ^= 1;
        tc_fence_after_sync();
        if (unsafe && more) {
            copy_tile16(sQ, p.q, rows_next);
            copy_tile16(sK, p.k, rows_next);
            copy_tile32(reinterpret_cast<uint8_t *>(sLA), p.la, rows_next);
            cp_async_arrive(&bar_ld);
        }
        if (tid == 0) {
            fence_proxy_async_smem();  // v landed by cp.async, observed by this thread
            const uint64_t ad = sdesc_sw128(smem_u32(sA), 16, 1024);
            const uint64_t vd = sdesc_sw128(smem_u32(sV), 8192, 1024);
            const uint64_t kd = sdesc_sw128(smem_u32(sKh), 16, 1024);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {  // o += A V ;  dS^T = V^T K^
                const uint64_t v = desc_add(vd, ks * 2048);
                mma_f16(tbase + TM_O, desc_add(ad, ks * 32), v, id_av, 1u);
                mma_f16(tbase + TM_DS, v, desc_add(kd, ks * 32), id_vk, ks > 0 ? 1u : 0u);
            }
            mma_commit(&bar_mma);
        }
        ok = cta_wait(&bar_mma, ph_mma, ok, &s_ok);
        ph_mma ^= 1;
        tc_fence_after_sync();
        // ---- outputs and the state update (rows t / rows j of lanes 0..15)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int cb = 32 * ch + 16 * hh;
            const uint32_t col = lane_off + cb;
            uint32_t ro[16], rs[16], rd[16];
            tmem_ld16(tbase + TM_O + col, ro);
            tmem_ld16(tbase + TM_S + col, rs);
            tmem_ld16(tbase + TM_DS + col, rd);
            tmem_ld_wait();
            if (act && row16 < len) {
                uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<T *>(p.out) +
                                                       (size_t)rows[row16] * FD + cb);
                float o[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) o[e] = __uint_as_float(ro[e]);
                dst[0] = pack8<T>(o);
                dst[1] = pack8<T>(o + 8);
            }
            // S^T[j][i] <- e^{g_i} S^T[j][i] + dS^T[j][i]
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
                const float4 g4 = *reinterpret_cast<const float4 *>(sGam + cb + e);
                rs[e] = __float_as_uint(fmaf(g4.x, __uint_as_float(rs[e]), __uint_as_float(rd[e])));
                rs[e + 1] = __float_as_uint(fmaf(g4.y, __uint_as_float(rs[e + 1]), __uint_as_float(rd[e + 1])));
                rs[e + 2] = __float_as_uint(fmaf(g4.z, __uint_as_float(rs[e + 2]), __uint_as_float(rd[e + 2])));
                rs[e + 3] = __float_as_uint(fmaf(g4.w, __uint_as_float(rs[e + 3]), __uint_as_float(rd[e + 3])));
            }
            tmem_st16(tbase + TM_S + col, rs);
            if (act && more) {
#pragma unroll
                for (int e = 0; e < 16; e += 4)
                    *reinterpret_cast<uint4 *>(sB1 + tf32_kmaj<128>(64 + row16, cb + e)) =
                        make_uint4(tf32_round(__uint_as_float(rs[e])), tf32_round(__uint_as_float(rs[e + 1])),
                                   tf32_round(__uint_as_float(rs[e + 2])), tf32_round(__uint_as_float(rs[e + 3])));
            }
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before_sync();
        if (more) {  // the next chunk's q,k,log_alpha; the barrier also ends this epilogue
            ok = cta_wait(&bar_ld, ph_ld, ok, &s_ok);
            ph_ld ^= 1;
        } else {
            __syncthreads();
        }
        tc_fence_after_sync();
        if (more) {
            copy_tile16(sV, p.v, rows_next);
            cp_async_arrive(&bar_v);
        }
    }

    if (seg == p.P - 1 && p.final_state) {  // S^T rows -> smem -> final_state rows i
        float *sFs = reinterpret_cast<float *>(sQH);  // [64][65], inside the idle Q^/K~ tiles
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint32_t rs[16];
            const int cb = 32 * ch + 16 * hh;
            tmem_ld16(tbase + TM_S + lane_off + cb, rs);
            tmem_ld_wait();
            if (act) {
#pragma unroll
                for (int e = 0; e < 16; ++e) sFs[(cb + e) * 65 + row16] = __uint_as_float(rs[e]);
            }
        }
        __syncthreads();
        for (int e = tid; e < 4096; e += kThreads)
            p.final_state[(size_t)bh * 4096 + e] = sFs[(e >> 6) * 65 + (e & 63)];
    }
        if (!ok) latch_error(p.err, kDevErrTimeout);

    // ------------------------------------------------------------- teardown
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tbase, kTmemCols);
    if (tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&p.ctr[1], 1u);
        s_last = (prev == gridDim.x - 1) ? 1 : 0;
    }
    __syncthreads();
    if (s_last) {  // last CTA to finish: leave the workspace ready for the next call
        if (p.P > 1)
            for (int idx = tid; idx < p.BH * p.P; idx += kThreads) p.flag[idx] = 0;
        if (tid == 0) {
            p.ctr[0] = 0;
            p.ctr[1] = 0;
        }
        __threadfence();
    }
}

constexpr int kTargetCtas = 2 * 148;  // two resident CTAs on each of the B200's SMs

struct Plan {
    int nc, P, L;
};

Plan make_plan(const Problem &pr) {
    Plan pl;
    pl.nc = (pr.n + FC - 1) / FC;
    const int bh = pr.B * pr.H;
    int P = kTargetCtas / bh;
    P = P < 1 ? 1 : (P > pl.nc ? pl.nc : P);
    if (P > kMaxSegments) P = kMaxSegments;
    if ((long long)bh * P > kWsMaxFlags) P = 1;
    pl.L = (pl.nc + P - 1) / P;
    pl.P = (pl.nc + pl.L - 1) / pl.L;
    return pl;
}

struct WsLayout {
    size_t agg, aggg, flag, ctr, total;
};

// ctr and flags live in the shared workspace header; the segment states after it.
WsLayout ws_layout(const Problem &pr, const Plan &pl) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t slots = pl.P > 1 ? (size_t)pr.B * pr.H * pl.P : 0;
    WsLayout w;
    w.ctr = 0;
    w.flag = 256;
    w.agg = kWsHeaderBytes;
    w.aggg = up(w.agg + slots * 4096 * 4);
    w.total = up(w.aggg + slots * 64 * 4);
    return w;
}

}  // namespace

bool fused_supported(const Problem &pr) {
    if (pr.dtype != GTR_GLA_F16 && pr.dtype != GTR_GLA_BF16) return false;
    if (pr.dk != 64 || pr.dv != 64 || pr.chunk != 64) return false;
    if ((long long)pr.B * pr.H * pr.n >= (1LL << 31)) return false;
    return true;
}

size_t fused_workspace_bytes(const Problem &pr) { return ws_layout(pr, make_plan(pr)).total; }

int launch_fused(const Problem &pr, void *ws, cudaStream_t st) {
    const Plan pl = make_plan(pr);
    const WsLayout wl = ws_layout(pr, pl);
    FusedParams p;
    memset(&p, 0, sizeof(p));
    char *w = static_cast<char *>(ws);
    p.q = pr.q;
    p.k = pr.k;
    p.v = pr.v;
    p.la = pr.la;
    p.out = pr.out;
    p.final_state = pr.final_state;
    p.agg = reinterpret_cast<float *>(w + wl.agg);
    p.aggg = reinterpret_cast<float *>(w + wl.aggg);
    p.flag = reinterpret_cast<int *>(w + wl.flag);
    p.ctr = reinterpret_cast<unsigned *>(w + wl.ctr);
    p.err = pr.err;
    p.n = pr.n;
    p.gh = pr.gh;
    p.gw = pr.gw;
    p.dir = pr.dir;
    p.nc = pl.nc;
    p.P = pl.P;
    p.L = pl.L;
    p.BH = pr.B * pr.H;
    const dim3 grid(p.BH * p.P);
    if (pr.dtype == GTR_GLA_BF16) {
        if (ensure_smem((const void *)gla_fused_kernel<true>, SMEM_BYTES)) return GTR_GLA_ERR_CUDA;
        gla_fused_kernel<true><<<grid, kThreads, SMEM_BYTES, st>>>(p);
    } else {
        if (ensure_smem((const void *)gla_fused_kernel<false>, SMEM_BYTES)) return GTR_GLA_ERR_CUDA;
        gla_fused_kernel<false><<<grid, kThreads, SMEM_BYTES, st>>>(p);
    }
    note_launch();
    return cudaPeekAtLastError() == cudaSuccess ? GTR_GLA_OK : GTR_GLA_ERR_CUDA;
}

}  // namespace gtr
