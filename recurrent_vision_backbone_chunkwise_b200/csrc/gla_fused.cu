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
//   * pre-pass: the segment's aggregate state contribution
//       A_seg = sum_c diag(e^{G_after(c)}) (k_c . e^{g_c - b_c})^T v_c
//     and its gate total are accumulated in TMEM (chunks visited last to
//     first, so every factor is <= 1) and published to the workspace;
//   * boundary pass: decoupled look-back over the earlier segments of the
//     same (b,h): the flags of the predecessors are read at once, the
//     aggregates after the nearest inclusive state are folded in one sweep
//     (S_in = sum_j diag(e^{G(j..seg)}) X_j), then the segment's own
//     inclusive state diag(e^{G_seg}) S_in + A_seg is published;
//   * main pass, chunk by chunk, with the fp32 state S kept in TMEM:
//       MMA1a (tf32, M=64,N=64,K=64):  scores = Q^ K~^T
//       MMA1b (tf32, M=64,N=64,K=64):  q^ S_in
//         Q^ = q . e^{b},  K~ = k . e^{-b}   (b: in-chunk inclusive log-gate sums)
//       causal mask of the scores on CUDA cores, re-quantised to f16/bf16,
//       MMA2 (f16/bf16, M=128,N=64,K=64):  [A ; K^^T] V -> [o_intra ; dS]
//         K^ = k . e^{g - b}  (rows interleaved so both products share lanes)
//       o = o_intra + q^ S_in,  S <- diag(e^{g}) S + dS.
//   Chunks whose in-chunk gate span exceeds kSpanLimit (e^{-b} would leave
//   fp32 range) take an exact CUDA-core path for the scores.
//
// Tiles are fetched in scan order with TMA row gathers, so every scan
// direction reads and writes the row-major grid in place.
//
// TMEM lane map (warp w reaches lanes 32(w%4)..32(w%4)+31): M=64 results put
// row r in lane 32(r/16) + r%16 ("token lanes"); the MMA2 A rows are ordered
// so that token t lands in the same lane and key dimension i in lane
// 32(i/16) + 16 + i%16 ("key lanes"), which also hold the state rows.
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
constexpr uint32_t OFF_KT = 57344;   // MMA1a B: K~ tf32 K-major [kc 2][64][128 B]
constexpr uint32_t OFF_SO = 73728;   // MMA1b B: S_in^T tf32 K-major [kc 2][64 j][128 B]
constexpr uint32_t OFF_A2 = 90112;   // MMA2 A:  128 rows x 128 B f16/bf16
constexpr uint32_t OFF_MISC = 106496;
constexpr uint32_t MISC_TOT = 0;     // [8][64] fp32 row-group totals of log_alpha
constexpr uint32_t MISC_G = 2048;    // [64] fp32 chunk gate totals g
constexpr uint32_t MISC_GA = 2304;   // [64] fp32 pre-pass: gate sums of later chunks
constexpr uint32_t MISC_SCL = 2560;  // [64] fp32 look-back: log scale of the inclusive term
constexpr uint32_t MISC_BYTES = 4096;
constexpr uint32_t SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;  // + alignment slack
constexpr uint32_t kTmemCols = 256;
// TMEM columns: scores (M=64), q^S_in (M=64), [o_intra ; dS] (M=128), state S
constexpr uint32_t TM_RAW = 0, TM_INT = 64, TM_D2 = 128, TM_S = 192;

struct alignas(64) FusedParams {
    CUtensorMap tm_q, tm_k, tm_v, tm_la;
    void *out;
    float *final_state;
    float *agg;    // [BH*P][64*64] segment aggregate states
    float *aggg;   // [BH*P][64]    segment log-gate totals
    float *incl;   // [BH*P][64*64] inclusive states
    int *flag;     // [BH*P] 0 empty, 1 aggregate, 2 inclusive
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

// byte offset of tf32 element (row, k) in a 64-row K-major tile with K = 64
__device__ __forceinline__ uint32_t tf32_kmaj(int row, int k) {
    return (k >> 5) * 8192 + sw128(row, (k & 31) >> 2) + (k & 3) * 4;
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

// MMA2 A-tile row of key dimension i
__device__ __forceinline__ int key_row(int i) { return 32 * (i >> 4) + 16 + (i & 15); }

// Issue the TMA loads of chunk c (warp 0 only): q/k/log_alpha on bar_ld, v on bar_v.
__device__ void issue_loads(const FusedParams &p, int bh, int c, bool q, bool kla, bool v,
                            uint8_t *sm, uint64_t *bar_ld, uint64_t *bar_v) {
    const int lane = threadIdx.x & 31;
    if (lane == 0) {
        const uint32_t ld_bytes = (q ? 8192u : 0u) + (kla ? 8192u + 16384u : 0u);
        if (ld_bytes) mbar_arrive_expect_tx(bar_ld, ld_bytes);
        if (v) mbar_arrive_expect_tx(bar_v, 8192u);
    }
    __syncwarp();
    if (lane < 16) {
        const int base = bh * p.n;
        const int u = lane * 4;
        int r[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            r[e] = base + scan_to_raster(min(c * FC + u + e, p.n - 1), p.n, p.gh, p.gw, p.dir);
        if (q) tma_gather4(sm + OFF_Q + u * 128, &p.tm_q, bar_ld, 0, r[0], r[1], r[2], r[3]);
        if (kla) {
            tma_gather4(sm + OFF_K + u * 128, &p.tm_k, bar_ld, 0, r[0], r[1], r[2], r[3]);
            tma_gather4(sm + OFF_LA + u * 256, &p.tm_la, bar_ld, 0, r[0], r[1], r[2], r[3]);
        }
        if (v) tma_gather4(sm + OFF_V + u * 128, &p.tm_v, bar_v, 0, r[0], r[1], r[2], r[3]);
    }
}

// In-chunk inclusive prefix sums of log_alpha for columns (p2, p2+1) and rows
// [8 r8, 8 r8 + 8); rows >= len count as 0.  g receives the chunk totals.
// Contains one __syncthreads.
__device__ __forceinline__ void chunk_cumsum(const float *sLA, float *sTot, int p2, int r8,
                                             int len, float b0[8], float b1[8], float2 &g) {
    float c0 = 0.f, c1 = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int u = 8 * r8 + k;
        float2 x = make_float2(0.f, 0.f);
        if (u < len) x = *reinterpret_cast<const float2 *>(sLA + u * 64 + p2);
        c0 += x.x;
        c1 += x.y;
        b0[k] = c0;
        b1[k] = c1;
    }
    *reinterpret_cast<float2 *>(sTot + r8 * 64 + p2) = make_float2(c0, c1);
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
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        b0[k] += o0;
        b1[k] += o1;
    }
    g = make_float2(t0, t1);
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads, 2) gla_fused_kernel(const __grid_constant__ FusedParams p) {
    using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sQ = sm + OFF_Q, *sK = sm + OFF_K, *sV = sm + OFF_V;
    float *sLA = reinterpret_cast<float *>(sm + OFF_LA);
    uint8_t *sQH = sm + OFF_QH, *sKT = sm + OFF_KT, *sSO = sm + OFF_SO, *sA2 = sm + OFF_A2;
    float *sTot = reinterpret_cast<float *>(sm + OFF_MISC + MISC_TOT);
    float *sG = reinterpret_cast<float *>(sm + OFF_MISC + MISC_G);
    float *sGa = reinterpret_cast<float *>(sm + OFF_MISC + MISC_GA);
    float *sScl = reinterpret_cast<float *>(sm + OFF_MISC + MISC_SCL);

    __shared__ uint64_t bar_ld, bar_v, bar_mma;
    __shared__ uint32_t s_tmem;
    __shared__ int s_ticket, s_last, s_jstar, s_nfold, s_fail;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, ch = warp >> 2;  // TMEM lane quadrant, column half
    const bool key_lane = lane >= 16;
    const int row16 = 16 * quad + (lane & 15);  // token (token lanes) or key dim (key lanes)
    const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
    const int p2 = 2 * (tid & 31), r8 = tid >> 5;  // gate math: columns p2, p2+1; rows 8 r8..
    constexpr uint32_t kFmt2 = BF16 ? 1u : 0u;
    const uint32_t id1 = idesc(2, 64, 64, 0, 0);       // tf32, both K-major
    const uint32_t id2 = idesc(kFmt2, 128, 64, 0, 1);  // f16/bf16, B MN-major

    if (tid == 0) {
        mbar_init(&bar_ld, 1);
        mbar_init(&bar_v, 1);
        mbar_init(&bar_mma, 1);
        fence_mbar_init();
        s_ticket = (int)atomicAdd(&p.ctr[0], 1u);
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_k);
        tma_prefetch_desc(&p.tm_v);
        tma_prefetch_desc(&p.tm_la);
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
    uint32_t ph_ld = 0, ph_v = 0, ph_mma = 0;
    bool ok = true;  // every bounded wait succeeded

    // ------------------------------------------------------------- pre-pass
    if (seg < p.P - 1) {
        if (tid < 64) sGa[tid] = 0.f;
        if (warp == 0) issue_loads(p, bh, c_end - 1, false, true, true, sm, &bar_ld, &bar_v);
        for (int c = c_end - 1; c >= c_begin; --c) {
            const int len = min(FC, p.n - c * FC);
            ok = ok && mbar_wait(&bar_ld, ph_ld);
            ph_ld ^= 1;
            float b0[8], b1[8];
            float2 g;
            chunk_cumsum(sLA, sTot, p2, r8, len, b0, b1, g);
            {
                const float2 ga = *reinterpret_cast<const float2 *>(sGa + p2);
                const float s0 = (ga.x + g.x) * kLog2e, s1 = (ga.y + g.y) * kLog2e;
                float kh0[8], kh1[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int u = 8 * r8 + k;
                    float2 kv = make_float2(0.f, 0.f);
                    if (u < len)
                        kv = Pack2<T>::unpack(*reinterpret_cast<const uint32_t *>(
                            sK + sw128(u, p2 >> 3) + (p2 & 7) * 2));
                    kh0[k] = kv.x * fast_exp2(s0 - b0[k] * kLog2e);
                    kh1[k] = kv.y * fast_exp2(s1 - b1[k] * kLog2e);
                }
                *reinterpret_cast<uint4 *>(sA2 + sw128(key_row(p2), r8)) = pack8<T>(kh0);
                *reinterpret_cast<uint4 *>(sA2 + sw128(key_row(p2 + 1), r8)) = pack8<T>(kh1);
            }
            fence_proxy_async_smem();
            __syncthreads();
            if (warp == 0 && c > c_begin) issue_loads(p, bh, c - 1, false, true, false, sm, &bar_ld, &bar_v);
            ok = ok && mbar_wait(&bar_v, ph_v);
            ph_v ^= 1;
            tc_fence_after_sync();
            if (tid == 0) {
                const uint32_t a0 = smem_u32(sA2), v0 = smem_u32(sV);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(tbase + TM_D2, sdesc_sw128(a0 + ks * 32, 16, 1024),
                            sdesc_sw128(v0 + ks * 2048, 8192, 1024), id2,
                            (c != c_end - 1 || ks > 0) ? 1u : 0u);
                mma_commit(&bar_mma);
            }
            __syncwarp();
            ok = ok && mbar_wait(&bar_mma, ph_mma);
            ph_mma ^= 1;
            tc_fence_after_sync();
            if (r8 == 7) {  // the last row group holds the chunk totals of columns p2, p2+1
                float2 ga = *reinterpret_cast<float2 *>(sGa + p2);
                ga.x += g.x;
                ga.y += g.y;
                *reinterpret_cast<float2 *>(sGa + p2) = ga;
            }
            __syncthreads();
            if (warp == 0 && c > c_begin) issue_loads(p, bh, c - 1, false, false, true, sm, &bar_ld, &bar_v);
        }
        // publish the aggregate (key lanes hold its rows in D2)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint32_t r[16];
            tmem_ld16(tbase + TM_D2 + lane_off + 32 * ch + 16 * hh, r);
            tmem_ld_wait();
            if (key_lane) {
                const size_t off = slot * 4096 + row16 * 64 + 32 * ch + 16 * hh;
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    const float4 v4 = make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                                  __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
                    *reinterpret_cast<float4 *>(p.agg + off + j) = v4;
                    if (seg == 0) *reinterpret_cast<float4 *>(p.incl + off + j) = v4;
                }
            }
        }
        if (key_lane && ch == 0) p.aggg[slot * 64 + row16] = sGa[row16];
        __threadfence();
        tc_fence_before_sync();
        __syncthreads();
        tc_fence_after_sync();
        if (tid == 0) st_release(p.flag + slot, seg == 0 ? 2 : 1);
    }

    // -------------------------------------------------------- boundary pass
    // S_in (fp32, [64][64] row-major) is assembled in the A2 tile's space.
    float *sSin = reinterpret_cast<float *>(sA2);
    if (seg > 0) {
        // 1. flags of the predecessors: nearest inclusive j* (-1 = none, start
        //    from zero), every segment after it at least an aggregate (a
        //    missing one is waited for, bounded)
        if (warp == 0) {
            int jstar = -1, fail = 0;
            int hi = seg - 1;
            while (!fail) {
                const int j = hi - lane;
                const int f = (j >= 0) ? ld_acquire(p.flag + (size_t)bh * p.P + j) : 2;
                const unsigned inc = __ballot_sync(0xffffffffu, f == 2);
                const int l_inc = inc ? __ffs(inc) - 1 : 32;
                const unsigned below = l_inc == 32 ? 0xffffffffu : ((1u << l_inc) - 1u);
                const unsigned zero = __ballot_sync(0xffffffffu, f == 0) & below;
                if (zero) {
                    const int l0 = __ffs(zero) - 1;
                    int ff = 0;
                    if (lane == 0) ff = wait_flag(p.flag + (size_t)bh * p.P + (hi - l0), p.err);
                    ff = __shfl_sync(0xffffffffu, ff, 0);
                    if (ff == 0) fail = 1;
                    continue;  // re-read this window
                }
                if (inc) {
                    jstar = hi - l_inc;
                    break;
                }
                hi -= 32;
            }
            if (lane == 0) {
                s_jstar = jstar;
                s_nfold = seg - 1 - jstar;
                s_fail = fail;
            }
        }
        __syncthreads();
        const int jstar = s_jstar, nfold = s_nfold;
        if (s_fail) ok = false;
        // 2. log-gate sums of the folded segments, per key dim (in QH's space)
        float *sAg = reinterpret_cast<float *>(sQH);  // [nfold][64], nfold < kMaxSegments
        for (int e = tid; e < nfold * 64; e += kThreads)
            sAg[e] = __ldcg(p.aggg + ((size_t)bh * p.P + (seg - 1 - (e >> 6))) * 64 + (e & 63));
        __syncthreads();
        if (tid < 64) {  // entry d is scaled by the gates of the d segments nearer to seg
            float acc = 0.f;
            for (int d = 0; d < nfold; ++d) {
                const float a = sAg[d * 64 + tid];
                sAg[d * 64 + tid] = acc;
                acc += a;
            }
            sScl[tid] = acc;
        }
        __syncthreads();
        // 3. fold: thread -> (row i, 16 columns)
        {
            const int i = tid >> 2, c0 = 16 * (tid & 3);
            float acc[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) acc[e] = 0.f;
            if (jstar >= 0) {
                const float sc = fast_exp2(sScl[i] * kLog2e);
                const float *src = p.incl + ((size_t)bh * p.P + jstar) * 4096 + i * 64 + c0;
#pragma unroll
                for (int q4 = 0; q4 < 16; q4 += 4) {
                    const float4 v4 = __ldcg(reinterpret_cast<const float4 *>(src + q4));
                    acc[q4] = sc * v4.x;
                    acc[q4 + 1] = sc * v4.y;
                    acc[q4 + 2] = sc * v4.z;
                    acc[q4 + 3] = sc * v4.w;
                }
            }
#pragma unroll 4
            for (int d = 0; d < nfold; ++d) {
                const float sc = fast_exp2(sAg[d * 64 + i] * kLog2e);
                const float *src = p.agg + ((size_t)bh * p.P + (seg - 1 - d)) * 4096 + i * 64 + c0;
#pragma unroll
                for (int q4 = 0; q4 < 16; q4 += 4) {
                    const float4 v4 = __ldcg(reinterpret_cast<const float4 *>(src + q4));
                    acc[q4] = fmaf(sc, v4.x, acc[q4]);
                    acc[q4 + 1] = fmaf(sc, v4.y, acc[q4 + 1]);
                    acc[q4 + 2] = fmaf(sc, v4.z, acc[q4 + 2]);
                    acc[q4 + 3] = fmaf(sc, v4.w, acc[q4 + 3]);
                }
            }
#pragma unroll
            for (int q4 = 0; q4 < 16; q4 += 4)
                *reinterpret_cast<float4 *>(sSin + i * 64 + c0 + q4) =
                    make_float4(acc[q4], acc[q4 + 1], acc[q4 + 2], acc[q4 + 3]);
        }
        __syncthreads();
    } else {
        for (int e = tid; e < 4096; e += kThreads) sSin[e] = 0.f;
        __syncthreads();
    }
    // S_in -> TMEM state (key lanes), the tf32 S_in^T operand, and (for a
    // segment with successors) the inclusive state diag(e^{G_seg}) S_in + A_seg.
    {
        const bool publish = seg > 0 && seg < p.P - 1;
        const float gam = publish ? fast_exp2(sGa[row16] * kLog2e) : 0.f;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int cb = 32 * ch + 16 * hh;
            uint32_t r[16], a[16];
            const float *src = sSin + row16 * 64 + cb;
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(key_lane ? src[e] : 0.f);
            tmem_st16(tbase + TM_S + lane_off + cb, r);
            if (publish) {
                tmem_ld16(tbase + TM_D2 + lane_off + cb, a);
                tmem_ld_wait();
            }
            if (key_lane) {
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    *reinterpret_cast<uint32_t *>(sSO + tf32_kmaj(cb + e, row16)) =
                        to_tf32(__uint_as_float(r[e]));
                if (publish) {
                    float *dst = p.incl + slot * 4096 + row16 * 64 + cb;
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        *reinterpret_cast<float4 *>(dst + e) = make_float4(
                            fmaf(gam, __uint_as_float(r[e]), __uint_as_float(a[e])),
                            fmaf(gam, __uint_as_float(r[e + 1]), __uint_as_float(a[e + 1])),
                            fmaf(gam, __uint_as_float(r[e + 2]), __uint_as_float(a[e + 2])),
                            fmaf(gam, __uint_as_float(r[e + 3]), __uint_as_float(a[e + 3])));
                }
            }
        }
        tmem_st_wait();
        if (publish) __threadfence();
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        tc_fence_after_sync();
        if (publish && tid == 0) st_release(p.flag + slot, 2);
    }

    // ------------------------------------------------------------ main pass
    if (warp == 0) issue_loads(p, bh, c_begin, true, true, true, sm, &bar_ld, &bar_v);
    for (int c = c_begin; c < c_end; ++c) {
        const int t0 = c * FC;
        const int len = min(FC, p.n - t0);
        ok = ok && mbar_wait(&bar_ld, ph_ld);
        ph_ld ^= 1;
        // ---- gate factors and operands
        float b0[8], b1[8];
        float2 g;
        chunk_cumsum(sLA, sTot, p2, r8, len, b0, b1, g);
        if (r8 == 7) *reinterpret_cast<float2 *>(sG + p2) = g;
        const bool my_unsafe = (-g.x > kSpanLimit) || (-g.y > kSpanLimit);
        {
            const float g20 = g.x * kLog2e, g21 = g.y * kLog2e;
            const float gam0 = fast_exp2(g20), gam1 = fast_exp2(g21);
            float kh0[8], kh1[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int u = 8 * r8 + k;
                float2 qv = make_float2(0.f, 0.f), kv = make_float2(0.f, 0.f);
                if (u < len) {
                    const uint32_t off = sw128(u, p2 >> 3) + (p2 & 7) * 2;
                    qv = Pack2<T>::unpack(*reinterpret_cast<const uint32_t *>(sQ + off));
                    kv = Pack2<T>::unpack(*reinterpret_cast<const uint32_t *>(sK + off));
                }
                const float bl0 = b0[k] * kLog2e, bl1 = b1[k] * kLog2e;
                const float ep0 = fast_exp2(bl0), ep1 = fast_exp2(bl1);
                const uint32_t toff = tf32_kmaj(u, p2);
                *reinterpret_cast<uint2 *>(sQH + toff) =
                    make_uint2(to_tf32(qv.x * ep0), to_tf32(qv.y * ep1));
                if (!my_unsafe) {
                    const float en0 = fast_exp2(-bl0), en1 = fast_exp2(-bl1);
                    *reinterpret_cast<uint2 *>(sKT + toff) =
                        make_uint2(to_tf32(kv.x * en0), to_tf32(kv.y * en1));
                    kh0[k] = kv.x * (en0 * gam0);
                    kh1[k] = kv.y * (en1 * gam1);
                } else {
                    *reinterpret_cast<uint2 *>(sKT + toff) = make_uint2(0u, 0u);
                    kh0[k] = kv.x * fast_exp2(g20 - bl0);
                    kh1[k] = kv.y * fast_exp2(g21 - bl1);
                }
                b0[k] = bl0;  // keep b in the log2 domain for the exact score path
                b1[k] = bl1;
            }
            *reinterpret_cast<uint4 *>(sA2 + sw128(key_row(p2), r8)) = pack8<T>(kh0);
            *reinterpret_cast<uint4 *>(sA2 + sw128(key_row(p2 + 1), r8)) = pack8<T>(kh1);
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        const int unsafe = __syncthreads_or(my_unsafe);
        tc_fence_after_sync();
        if (tid == 0) {
            const uint32_t a0 = smem_u32(sQH), k0 = smem_u32(sKT), s0 = smem_u32(sSO);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t koff = (ks >> 2) * 8192 + (ks & 3) * 32;
                const uint64_t ad = sdesc_sw128(a0 + koff, 16, 1024);
                mma_tf32(tbase + TM_RAW, ad, sdesc_sw128(k0 + koff, 16, 1024), id1, ks > 0 ? 1u : 0u);
                mma_tf32(tbase + TM_INT, ad, sdesc_sw128(s0 + koff, 16, 1024), id1, ks > 0 ? 1u : 0u);
            }
            mma_commit(&bar_mma);
        }
        if (unsafe) {  // the exact path needs b of every row: park it in sLA
#pragma unroll
            for (int k = 0; k < 8; ++k)
                *reinterpret_cast<float2 *>(sLA + (8 * r8 + k) * 64 + p2) = make_float2(b0[k], b1[k]);
        } else if (warp == 0 && c + 1 < c_end) {
            issue_loads(p, bh, c + 1, true, true, false, sm, &bar_ld, &bar_v);
        }
        ok = ok && mbar_wait(&bar_mma, ph_mma);
        ph_mma ^= 1;
        tc_fence_after_sync();
        // ---- causal mask of the scores -> MMA2 A token rows
        if (!unsafe) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t r[16];
                tmem_ld16(tbase + TM_RAW + lane_off + 32 * ch + 16 * hh, r);
                tmem_ld_wait();
                if (!key_lane) {
                    const int t = row16;
                    float a[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int s = 32 * ch + 16 * hh + e;
                        a[e] = (s <= t) ? __uint_as_float(r[e]) : 0.f;
                    }
                    const int m = 32 * quad + lane;
                    *reinterpret_cast<uint4 *>(sA2 + sw128(m, 4 * ch + 2 * hh)) = pack8<T>(a);
                    *reinterpret_cast<uint4 *>(sA2 + sw128(m, 4 * ch + 2 * hh + 1)) = pack8<T>(a + 8);
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
            const int m = 32 * (t >> 4) + (t & 15);
            *reinterpret_cast<uint4 *>(sA2 + sw128(m, s0 >> 3)) = pack8<T>(a);
            *reinterpret_cast<uint4 *>(sA2 + sw128(m, (s0 >> 3) + 1)) = pack8<T>(a + 8);
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        tc_fence_after_sync();
        if (unsafe && warp == 0 && c + 1 < c_end)
            issue_loads(p, bh, c + 1, true, true, false, sm, &bar_ld, &bar_v);
        ok = ok && mbar_wait(&bar_v, ph_v);
        ph_v ^= 1;
        if (tid == 0) {
            const uint32_t a0 = smem_u32(sA2), v0 = smem_u32(sV);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_f16(tbase + TM_D2, sdesc_sw128(a0 + ks * 32, 16, 1024),
                        sdesc_sw128(v0 + ks * 2048, 8192, 1024), id2, ks > 0 ? 1u : 0u);
            mma_commit(&bar_mma);
        }
        __syncwarp();
        ok = ok && mbar_wait(&bar_mma, ph_mma);
        ph_mma ^= 1;
        tc_fence_after_sync();
        // ---- outputs and the state update
        {
            const float gam = key_lane ? fast_exp2(sG[row16] * kLog2e) : 0.f;
            const int t = row16;
            const bool store_out = !key_lane && t < len;
            uint4 *dst = nullptr;
            if (store_out) {
                const size_t r = (size_t)bh * p.n + scan_to_raster(t0 + t, p.n, p.gh, p.gw, p.dir);
                dst = reinterpret_cast<uint4 *>(reinterpret_cast<T *>(p.out) + r * FD + 32 * ch);
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int cb = 32 * ch + 16 * hh;
                const uint32_t col = lane_off + cb;
                uint32_t ro[16], rd[16], rs[16];
                tmem_ld16(tbase + TM_INT + col, ro);
                tmem_ld16(tbase + TM_D2 + col, rd);
                tmem_ld16(tbase + TM_S + col, rs);
                tmem_ld_wait();
                if (!key_lane) {
                    float o[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) o[e] = __uint_as_float(ro[e]) + __uint_as_float(rd[e]);
                    if (store_out) {
                        dst[2 * hh] = pack8<T>(o);
                        dst[2 * hh + 1] = pack8<T>(o + 8);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        rs[e] = __float_as_uint(fmaf(gam, __uint_as_float(rs[e]), __uint_as_float(rd[e])));
                    if (c + 1 < c_end) {
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            *reinterpret_cast<uint32_t *>(sSO + tf32_kmaj(cb + e, row16)) =
                                to_tf32(__uint_as_float(rs[e]));
                    }
                }
                tmem_st16(tbase + TM_S + col, rs);
            }
            tmem_st_wait();
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        tc_fence_after_sync();
        if (warp == 0 && c + 1 < c_end) issue_loads(p, bh, c + 1, false, false, true, sm, &bar_ld, &bar_v);
    }

    if (seg == p.P - 1 && p.final_state) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint32_t rs[16];
            const int cb = 32 * ch + 16 * hh;
            tmem_ld16(tbase + TM_S + lane_off + cb, rs);
            tmem_ld_wait();
            if (key_lane) {
                float *dst = p.final_state + (size_t)bh * 4096 + row16 * 64 + cb;
#pragma unroll
                for (int e = 0; e < 16; e += 4)
                    *reinterpret_cast<float4 *>(dst + e) =
                        make_float4(__uint_as_float(rs[e]), __uint_as_float(rs[e + 1]),
                                    __uint_as_float(rs[e + 2]), __uint_as_float(rs[e + 3]));
            }
        }
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
    size_t agg, aggg, incl, flag, ctr, total;
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
    w.incl = up(w.aggg + slots * 64 * 4);
    w.total = up(w.incl + slots * 4096 * 4);
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
    const CUtensorMapDataType t16 =
        pr.dtype == GTR_GLA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const uint64_t rows = (uint64_t)pr.B * pr.H * pr.n;
    int rc = 0;
    rc |= encode_rows_map(&p.tm_q, pr.q, t16, 2, rows, 64, true);
    rc |= encode_rows_map(&p.tm_k, pr.k, t16, 2, rows, 64, true);
    rc |= encode_rows_map(&p.tm_v, pr.v, t16, 2, rows, 64, true);
    rc |= encode_rows_map(&p.tm_la, pr.la, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, rows, 64, false);
    if (rc) return GTR_GLA_ERR_CUDA;
    char *w = static_cast<char *>(ws);
    p.out = pr.out;
    p.final_state = pr.final_state;
    p.agg = reinterpret_cast<float *>(w + wl.agg);
    p.aggg = reinterpret_cast<float *>(w + wl.aggg);
    p.incl = reinterpret_cast<float *>(w + wl.incl);
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
