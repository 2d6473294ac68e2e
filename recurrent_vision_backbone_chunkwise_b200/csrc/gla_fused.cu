// gla_fused.cu -- single-kernel chunkwise GLA forward on sm_100a tensor cores
// (fp16 / bf16 I/O, chunk 64, 64-wide key and value tiles), warp-specialised.
//
// The chunkwise reorganisation of "GTR: Gated Token Recurrence for Efficient
// Dense Prediction" (x-techcon article, section 算子): every chunk computes
// its own contribution to the state in parallel, a light sequential scan
// carries the boundary states, every chunk's output is produced in parallel,
// and the attention scores never leave the chip.  Mapped onto one launch of
// 576-thread CTAs, one per SM:
//
//   * a CTA owns a segment of L consecutive 64-token chunks of one (b,h);
//     CTAs take their segment from a ticket counter, so a segment only ever
//     waits for segments that were started before it;
//   * pre-pass (every segment but the last of its (b,h)): the segment's
//     aggregate state contribution, transposed,
//       A_seg^T = sum_c V_c^T (k_c . e^{G_after(c) + g_c - b_c}),
//     accumulates in TMEM (every factor <= 1) and is published with the
//     segment's log-gate totals (one release store of a flag on its own line);
//   * boundary: the incoming state is the fold of every earlier segment's
//     aggregate, nearest first, S_in = sum_j diag(e^{G(j..seg)}) A_j, in a
//     fixed order (results are bitwise reproducible);
//   * main pass, chunk by chunk (b: in-chunk inclusive log-gate sums, g: the
//     chunk total, m: a per-key-dimension reference inside [g, 0]):
//       [scores | o] = Q' [K~ ; S~^T]^T   Q' = q e^{b-m}, K~ = k e^{m-b},
//                                         S~ = e^{m} S   (one N = 128 MMA)
//       dS'^T        = V^T K~             (the state contribution is
//                                         dS = diag(e^{g-m}) dS', as K^ = k e^{g-b})
//       A            = causal mask of the scores
//       o           += A V
//       S           <- diag(e^{g}) S + dS (fp32, registers of the state warps)
//     Every operand is in the I/O dtype (fp16 or bf16) with fp32
//     accumulation.  The reference m balances the magnitudes of Q' and K~
//     (each is at most sqrt(max|q| max|k|) e^{-g/2}), so fp16 covers the
//     in-chunk gate spans of the long-memory workloads; a chunk whose span
//     would overflow the operand type takes exact scores from CUDA cores
//     (every factor <= 1) and m = 0.
//
// Roles (warps).  Each product is issued by one thread of the role that makes
// its last input, right after a barrier of that role (no hand-off to a
// separate MMA thread on the main path):
//   0       producer: row tables and TMA tile loads (row scans: one box per
//           tensor; column scans: column slabs, or four-row gathers) of q,
//           k, v, log_alpha into a 4-stage ring, so every scan direction
//           reads the row-major grid in place; TMEM allocation; the
//           pre-pass MMAs (in item order);
//   1..8    two operand warp quads; quad q prepares the chunks of stages q
//           and q + 2 (each lane owns two key dimensions, each warp 16 stage
//           rows) and issues their dS products;
//   9..12   state warps (one per TMEM lane quadrant): the boundary state in
//           fp32 registers, its fp16 copy per chunk and the chunk's
//           [scores | q S] product, the segment aggregate's publication and
//           the fold, the final state;
//   13..16  epilogue warps (one per TMEM lane quadrant): causal mask of the
//           scores and the A V product, then the output through a
//           shared-memory staging tile with coalesced 16-byte stores at the
//           tokens' raster rows.
#include <type_traits>

#include "gla_common.cuh"
#include "gla_internal.h"
#include "sm100.cuh"

namespace gtr {
using namespace sm100;

namespace {

constexpr int FC = 64;  // tokens per chunk
constexpr int FD = 64;  // key / value tile width
constexpr int kStages = 4;
constexpr int kWarpLoad = 0, kWarpOp0 = 1, kWarpSt0 = 9, kWarpEpi0 = 13;
constexpr int kThreads = 17 * 32;
constexpr int kGroupThreads = 128;
constexpr int kBarEpi = 1, kBarSt = 2, kBarQuad0 = 3;  // named barrier ids (operand quad q: 3 + q)
constexpr int kMaxSegments = 32;                       // segments per (b,h): bounds the fold
constexpr float kLog2e = 1.4426950408889634f;

// One pipeline stage (byte offsets from the stage base, every tile 1024-aligned,
// 128-byte rows with the 128-byte swizzle).
constexpr uint32_t ST_Q = 0;       // q -> Q' (K-major A) -> output staging
constexpr uint32_t ST_V = 8192;    // v (MN-major operand)
constexpr uint32_t ST_K = 16384;   // k -> K~ (K-major B of the scores, MN-major B of dS)
constexpr uint32_t ST_S = 24576;   // S~^T (K-major B of q S); exact scores A of flagged chunks
constexpr uint32_t ST_LA = 32768;  // log_alpha [64][256 B] fp32 -> pre-pass K^seg, or the
                                   // masked scores A (flagged chunks: S~^T)
constexpr uint32_t ST_BYTES = 49152;
constexpr uint32_t OFF_GT = kStages * ST_BYTES;  // fold: earlier segments' log2 gate totals
constexpr uint32_t OFF_MISC = OFF_GT + kMaxSegments * 64 * 4;
constexpr int kRing = 8;           // per-chunk gate factors, by main-pass chunk index mod 8
constexpr uint32_t M_ROWS = 0;     // int   [kStages][64] raster row of each stage row
constexpr uint32_t M_LEN = 1024;   // int   [kStages] tokens in the chunk
constexpr uint32_t M_FLAG = 1040;  // int   [kStages] exact-score chunk
constexpr uint32_t M_GAM = 1536;   // float [kRing][64] 2^{g2}
constexpr uint32_t M_EM = M_GAM + kRing * 256;   // float [kRing][64] 2^{m2}
constexpr uint32_t M_CGM = M_EM + kRing * 256;   // float [kRing][64] 2^{g2 - m2}
constexpr uint32_t M_XCH = M_CGM + kRing * 256;  // float [2 quads][4 warps][3][64] pass-1 partials
constexpr uint32_t M_GA = M_XCH + 2 * 4 * 3 * 64 * 4;  // float [4][64] pre-pass gate suffix ring
constexpr uint32_t MISC_BYTES = M_GA + 4 * 64 * 4;
constexpr uint32_t SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory");

// TMEM (512 columns; M = 64 results sit in lanes 32 q + 0..15 of quadrant q):
// three regions of 128 columns [scores | o], chunk j in region j % 3; two
// 64-column dS^T buffers; the pre-pass aggregate borrows region 2 until it
// has been read out.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t TM_DS = 384, TM_PRE = 256;

struct FusedParams {
    // Tiled views of q, k, v, log_alpha.  Row scans (L->R, R->L): [BH][n][64],
    // one 64-row box per chunk.  Column scans (T->B, B->T): [BH][gh][gw][64],
    // boxes of `boxh` consecutive grid rows of one column (boxh: the largest
    // power of two <= 64 that divides grid_h); boxh = 0: four-row gathers.
    CUtensorMap tm_q, tm_k, tm_v, tm_la;
    void *out;
    float *final_state;
    float *agg;     // [BH*P][8][128][4] segment aggregates, in state-thread order
    float *aggg;    // [BH*P][64]    segment log2 gate totals
    int *flag;      // [BH*P] (stride kWsFlagStride) 0 empty, 1 published
    unsigned *ctr;  // [0] ticket, [1] finished CTAs
    int *err;
    int n, gh, gw, dir, nc, P, L, BH;
    // Head sizes of 128 run as 64-wide sub-problems: `out` and `final_state`
    // point at the sub-problem's corner, ldo is the output row stride in
    // elements, acc_out adds to what is already in `out`, fs_bh / fs_ld are
    // the final state's (b,h) and row strides.
    int ldo, acc_out, fs_bh, fs_ld;
    int boxh;
    float logf2;  // log2 of the largest operand magnitude the factorised scores may reach
};

__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(int *p, int v) {
    asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded wait (about 2 s) for a non-zero flag; false if it never came.
__device__ bool wait_flag(const int *f) {
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (ld_acquire(f) != 0) return true;
        if (global_timer_ns() - t0 > 2000000000ull) return false;
        __nanosleep(64);
    }
}

// Bounded wait on an mbarrier phase (about 2 s): the first wait that gives up
// raises `abort`, after which every wait returns at once, so all threads reach
// the end of the kernel.  The waiting thread sleeps in hardware (try_wait with
// a suspend hint) until the phase completes, waking at least every 20 us to
// look at the abort flag and the clock.  False when aborted.
__device__ bool pwait(uint64_t *bar, uint32_t parity, volatile int *abort, int *err) {
    if (mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait_hint(bar, parity, 20000)) return true;
        if (*abort) return false;
        if (global_timer_ns() - t0 > 2000000000ull) {
            *abort = 1;
            latch_error(err, kDevErrTimeout);
            return false;
        }
    }
}

// A warp waits through its lane 0; false when aborted.
__device__ __forceinline__ bool wwait(uint64_t *bar, uint32_t parity, volatile int *abort, int *err) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = pwait(bar, parity, abort, err);
    return __shfl_sync(0xffffffffu, ok, 0);
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

// Element-wise max of magnitudes of two packed 16-bit pairs.
__device__ __forceinline__ uint32_t absmax2(uint32_t a, uint32_t b, __half *) {
    __half2 r = __hmax2(__habs2(*reinterpret_cast<__half2 *>(&a)), __habs2(*reinterpret_cast<__half2 *>(&b)));
    return *reinterpret_cast<uint32_t *>(&r);
}
__device__ __forceinline__ uint32_t absmax2(uint32_t a, uint32_t b, __nv_bfloat16 *) {
    __nv_bfloat162 r = __hmax2(__habs2(*reinterpret_cast<__nv_bfloat162 *>(&a)),
                               __habs2(*reinterpret_cast<__nv_bfloat162 *>(&b)));
    return *reinterpret_cast<uint32_t *>(&r);
}

// A shared-memory descriptor advanced by `bytes` (the start address field
// holds addr >> 4 in its low 14 bits; smem addresses stay far below 256 KiB).
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t bytes) {
    return d + (uint64_t)(bytes >> 4);
}

__device__ __forceinline__ float2 ld2(const float *p) { return *reinterpret_cast<const float2 *>(p); }
__device__ __forceinline__ void st2(float *p, float2 v) { *reinterpret_cast<float2 *>(p) = v; }
__device__ __forceinline__ float2 ex2_2(float2 x) { return make_float2(fast_exp2(x.x), fast_exp2(x.y)); }
__device__ __forceinline__ float fast_log2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 16-bit element pair (2 l, 2 l + 1) of row r in a 128B-swizzled tile.
__device__ __forceinline__ uint32_t pair_off(int r, int l) { return sw128(r, l >> 2) + (l & 3) * 4; }

// The balanced reference of one key dimension (log2 domain): m2 in [g2, 0]
// equalises the bounds max|q| 2^{-m2} and max|k| 2^{m2-g2} of Q' and K~.
__device__ __forceinline__ float ref_m2(float g2, float mq, float mk) {
    float m = 0.5f * g2;
    if (mq > 0.f && mk > 0.f) m = 0.5f * (g2 + fast_log2(mq) - fast_log2(mk));
    return fminf(0.f, fmaxf(g2, m));
}

// Does the factorised form overflow the operand type in this key dimension?
__device__ __forceinline__ bool span_unsafe(float g2, float mq, float mk, float logf2) {
    if (mq <= 0.f || mk <= 0.f) return false;
    return fast_log2(mq) + fast_log2(mk) - g2 > 2.f * logf2;
}

template <bool BF16, bool REV>
__global__ void __launch_bounds__(kThreads, 1) gla_fused_kernel(const __grid_constant__ FusedParams p) {
    using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    int *sRows = reinterpret_cast<int *>(sm + OFF_MISC + M_ROWS);
    float *sGam = reinterpret_cast<float *>(sm + OFF_MISC + M_GAM);
    float *sEm = reinterpret_cast<float *>(sm + OFF_MISC + M_EM);
    float *sCgm = reinterpret_cast<float *>(sm + OFF_MISC + M_CGM);
    int *sLen = reinterpret_cast<int *>(sm + OFF_MISC + M_LEN);
    int *sFlag = reinterpret_cast<int *>(sm + OFF_MISC + M_FLAG);
    float *sXch = reinterpret_cast<float *>(sm + OFF_MISC + M_XCH);
    float *sGA = reinterpret_cast<float *>(sm + OFF_MISC + M_GA);
    float *sGt = reinterpret_cast<float *>(sm + OFF_GT);

    __shared__ uint64_t bar_full[kStages], bar_empty[kStages], bar_op[kStages], bar_ga[kStages];
    __shared__ uint64_t bar_sc[3], bar_o[3], bar_rf[3], bar_ds[2], bar_dsf[2];
    __shared__ uint64_t bar_pre, bar_gtot, bar_fin;
    __shared__ uint32_t s_tmem;
    __shared__ int s_ticket, s_last;
    __shared__ volatile int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bar_full[s], 1);  // producer lane 0 (with the stage's TMA bytes)
            mbar_init(&bar_empty[s], 1);
            mbar_init(&bar_op[s], 4);  // one lane per warp of the quad
            mbar_init(&bar_ga[s], 4);
        }
        for (int b = 0; b < 3; ++b) {
            mbar_init(&bar_sc[b], 1);
            mbar_init(&bar_o[b], 1);
            mbar_init(&bar_rf[b], kGroupThreads);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar_ds[b], 1);
            mbar_init(&bar_dsf[b], kGroupThreads);
        }
        mbar_init(&bar_pre, 1);
        mbar_init(&bar_gtot, 4);
        mbar_init(&bar_fin, 1);
        fence_mbar_init();
        s_ticket = (int)atomicAdd(&p.ctr[0], 1u);
        s_abort = 0;
    }
    if (warp == kWarpLoad) {
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
    const int L = c_end - c_begin;
    const int npre = (seg < p.P - 1) ? L : 0;  // the last segment needs no aggregate
    const int n_items = npre + L;
    const size_t slot = (size_t)bh * p.P + seg;
    constexpr uint32_t kFmt = BF16 ? 1u : 0u;
    constexpr bool rev = REV;  // reversed scans: token u sits in stage row 63 - u
    volatile int *abort = &s_abort;

    if ((unsigned)ticket >= (unsigned)(p.BH * p.P)) {
        // A ticket past the last segment means the workspace header was not
        // zero at launch (two calls sharing it overlapped, or it was never
        // zeroed): this CTA does no work and reports it; the counters and
        // flags are still reset below, so the next call starts clean.
        if (tid == 0) latch_error(p.err, kDevErrWorkspace);
    } else if (warp == kWarpLoad) {
        // ------------------------------------------- producer and pre-pass MMA
        // TMA loads of whole chunks into the 4-stage ring.  Before a stage that
        // held a pre-pass chunk is refilled, lane 0 issues that chunk's
        // aggregate MMA (in item order, so the accumulation order is fixed);
        // the MMA's completion releases the stage.  The main pass issues its
        // products where their inputs are made (dS and the scores by the
        // operand warps, q S by the state warps, A V by the mask warps).
        const uint64_t pol_keep = l2_policy_evict_last();  // pre-pass data is read again
        const uint64_t pol_once = l2_policy_evict_first();
        if (lane == 0) {
            tma_prefetch_desc(&p.tm_q);
            tma_prefetch_desc(&p.tm_k);
            tma_prefetch_desc(&p.tm_v);
            tma_prefetch_desc(&p.tm_la);
        }
        const uint32_t sbase = smem_u32(sm);
        // K^seg: MN-major with 8-row groups 2048 bytes apart (see the operand warps)
        const uint32_t kh_base = ST_LA + (rev ? 1024u : 0u);
        auto issue_pre = [&](int ip) -> bool {  // lane 0: A_seg^T += V^T K^seg of pre-pass item ip
            const int s = ip % kStages;
            if (!pwait(&bar_op[s], (ip / kStages) & 1, abort, p.err)) return false;
            tc_fence_after_sync();
            fence_proxy_async_smem();
            const uint64_t dv = sdesc_sw128(sbase + s * ST_BYTES + ST_V, 8192, 1024);
            const uint64_t dh = sdesc_sw128(sbase + s * ST_BYTES + kh_base, 8192, 2048);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_f16(tbase + TM_PRE, desc_add(dv, ks * 2048), desc_add(dh, ks * 4096), idesc(kFmt, 64, 64, 1, 1),
                        (ip > 0 || ks > 0) ? 1u : 0u);
            mma_commit(&bar_empty[s]);
            if (ip == npre - 1) mma_commit(&bar_pre);
            return true;
        };
        bool ok = true;
        uint32_t issued = 0;  // bit s: the last use of stage s had its copies issued
        for (int it = 0; it < n_items; ++it) {
            const int s = it % kStages;
            const bool pre = it < npre;
            const int c = pre ? (c_end - 1 - it) : (c_begin + it - npre);
            if (it >= kStages) {
                if (it - kStages < npre) {
                    bool w = true;
                    if (lane == 0) w = issue_pre(it - kStages);
                    ok = __shfl_sync(0xffffffffu, w, 0) && ok;
                }
                ok = wwait(&bar_empty[s], ((it / kStages) - 1) & 1, abort, p.err) && ok;
            }
            issued = ok ? (issued | (1u << s)) : (issued & ~(1u << s));
            // During the pre-pass, the main pass's q tiles of the same chunks
            // go to L2 ahead of time (k, v, log_alpha are left there by the
            // pre-pass loads themselves).
            if (pre && p.dir < 2 && lane == 0 && it < L) {
                const int cm = c_begin + it;
                tma_prefetch_l2_3d(&p.tm_q, 0, rev ? (p.n - FC - cm * FC) : cm * FC, bh);
            }
            // The chunk's tokens, in stage-row order: row scans load raster
            // rows [p0, p0 + 64) of the plane, column scans the column-major
            // positions [p0, p0 + 64); reversed scans read the same range
            // (token u sits in stage row 63 - u).  Rows outside the grid read
            // as zero.  Row table: raster row of every stage row (-1: none).
            const int p0 = rev ? (p.n - FC - c * FC) : c * FC;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int r = lane + 32 * e, pp = p0 + r;
                int row = -1;
                if (pp >= 0 && pp < p.n) row = bh * p.n + (p.dir < 2 ? pp : (pp % p.gh) * p.gw + pp / p.gh);
                sRows[s * 64 + r] = row;
            }
            if (lane == 0) sLen[s] = min(FC, p.n - c * FC);
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(&bar_full[s], pre ? 32768u : 40960u);
            __syncwarp();
            if (ok) {
                uint8_t *st = sm + s * ST_BYTES;
                const uint64_t pol = pre ? pol_keep : pol_once;
                if (p.dir < 2) {
                    if (lane == 0) {
                        tma_load_3d_pol(st + ST_K, &p.tm_k, &bar_full[s], 0, p0, bh, pol);
                        tma_load_3d_pol(st + ST_V, &p.tm_v, &bar_full[s], 0, p0, bh, pol);
                        tma_load_3d_pol(st + ST_LA, &p.tm_la, &bar_full[s], 0, p0, bh, pol);
                        if (!pre) tma_load_3d_pol(st + ST_Q, &p.tm_q, &bar_full[s], 0, p0, bh, pol_once);
                    }
                } else if (p.boxh == 0) {
                    if (lane < 16) {  // stage rows 4 lane .. 4 lane + 3, as row gathers
                        int r[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int u = rev ? 63 - (4 * lane + e) : 4 * lane + e;
                            r[e] = bh * p.n + scan_to_raster(min(c * FC + u, p.n - 1), p.n, p.gh, p.gw, p.dir);
                        }
                        const int m = 4 * lane;
                        tma_gather4_pol(st + ST_K + m * 128, &p.tm_k, &bar_full[s], 0, r[0], r[1], r[2], r[3], pol);
                        tma_gather4_pol(st + ST_V + m * 128, &p.tm_v, &bar_full[s], 0, r[0], r[1], r[2], r[3], pol);
                        tma_gather4_pol(st + ST_LA + m * 256, &p.tm_la, &bar_full[s], 0, r[0], r[1], r[2], r[3], pol);
                        if (!pre)
                            tma_gather4_pol(st + ST_Q + m * 128, &p.tm_q, &bar_full[s], 0, r[0], r[1], r[2], r[3],
                                            pol_once);
                    }
                } else {
                    const int h = p.boxh;
                    for (int bx = lane; bx < FC / h; bx += 32) {
                        const int pp = p0 + bx * h;  // a multiple of h: the box stays in one column
                        const int x = pp >= 0 ? pp / p.gh : -1, y = pp >= 0 ? pp % p.gh : 0;
                        const int r = bx * h;
                        tma_load_4d_pol(st + ST_K + r * 128, &p.tm_k, &bar_full[s], 0, x, y, bh, pol);
                        tma_load_4d_pol(st + ST_V + r * 128, &p.tm_v, &bar_full[s], 0, x, y, bh, pol);
                        tma_load_4d_pol(st + ST_LA + r * 256, &p.tm_la, &bar_full[s], 0, x, y, bh, pol);
                        if (!pre)
                            tma_load_4d_pol(st + ST_Q + r * 128, &p.tm_q, &bar_full[s], 0, x, y, bh, pol_once);
                    }
                }
            }
        }
        // the pre-pass chunks whose stage was not refilled
        if (lane == 0)
            for (int ip = (n_items > kStages ? n_items - kStages : 0); ip < npre; ++ip) ok = issue_pre(ip) && ok;
        // no copy may still be landing when the CTA exits (after an abort the
        // consumers may not have waited for them): bounded wait on the last
        // issued phase of every stage; and every pre-pass MMA completes
        if (lane == 0) {
            for (int it = (n_items > kStages ? n_items - kStages : 0); it < n_items; ++it) {
                const int s = it % kStages;
                if (issued & (1u << s)) mbar_wait(&bar_full[s], (it / kStages) & 1, 200000000ull);
            }
            mma_commit(&bar_fin);
            mbar_wait(&bar_fin, 0, 200000000ull);
        }
        __syncwarp();
    } else if (warp < kWarpSt0) {
        // ------------------------------------------------- operand warp quads
        // Quad q (warps 2 + 4 q .. 5 + 4 q) prepares the chunks of stages q
        // and q + 2.  Warp w of the quad owns stage rows [16 w, 16 w + 16)
        // and visits them in token order (ascending rows; descending for
        // reversed scans); lane l owns key dimensions 2 l, 2 l + 1.  Every
        // operand is written in place over data this warp has already read:
        // Q' over q, K~ over k, and (pre-pass) K^ into the log_alpha rows
        // through a tile whose 8-row groups are 2048 bytes apart (rows
        // 8 g .. 8 g + 3 of log_alpha for L->R order, 8 g + 4 .. 8 g + 7 for
        // reversed order: always a row the warp has passed).
        const int quad = (warp - kWarpOp0) >> 2, qw = (warp - kWarpOp0) & 3;
        const int bar_id = kBarQuad0 + quad;
        const int r0 = 16 * qw + (rev ? 15 : 0), rstep = rev ? -1 : 1;  // first row, step
        const int rank = rev ? 3 - qw : qw;  // this warp's 16 tokens are tokens 16 rank .. 16 rank + 15
        const uint32_t kh_base = ST_LA + (rev ? 1024u : 0u);
        auto kh_off = [&](int r) { return kh_base + (uint32_t)(r >> 3) * 2048u + pair_off(r & 7, lane); };
        const float2 kL2 = make_float2(kLog2e, kLog2e);
        for (int it = quad; it < n_items; it += 2) {
            const int s = it % kStages;
            uint8_t *st = sm + s * ST_BYTES;
            const float *lat = reinterpret_cast<const float *>(st + ST_LA);
            if (!wwait(&bar_full[s], (it / kStages) & 1, abort, p.err)) break;
            const bool pre = it < npre;
            const int len = sLen[s];
            if (len < FC) {
                // the plane's last chunk: rows of tokens past the end become
                // zero (box loads already read them as zero; row gathers
                // repeat the last row), so no later step needs to test them
                for (int i = 0; i < 16; ++i) {
                    const int r = r0 + rstep * i, u = rev ? 63 - r : r;
                    if (u >= len) {
                        st2(reinterpret_cast<float *>(st + ST_LA) + r * 64 + 2 * lane, make_float2(0.f, 0.f));
                        *reinterpret_cast<uint32_t *>(st + ST_K + pair_off(r, lane)) = 0u;
                        *reinterpret_cast<uint32_t *>(st + ST_Q + pair_off(r, lane)) = 0u;
                    }
                }
            }
            // pass 1: log-gate sum over this warp's rows, and (main pass) the
            // magnitudes of q and k
            float2 sum = make_float2(0.f, 0.f);
            uint32_t aq = 0u, ak = 0u;
            if (pre) {
#pragma unroll
                for (int i = 0; i < 16; ++i) sum = fadd2(sum, ld2(lat + (r0 + rstep * i) * 64 + 2 * lane));
            } else {
#pragma unroll 8
                for (int i = 0; i < 16; ++i) {
                    const int r = r0 + rstep * i;
                    sum = fadd2(sum, ld2(lat + r * 64 + 2 * lane));
                    aq = absmax2(aq, *reinterpret_cast<const uint32_t *>(st + ST_Q + pair_off(r, lane)), (T *)nullptr);
                    ak = absmax2(ak, *reinterpret_cast<const uint32_t *>(st + ST_K + pair_off(r, lane)), (T *)nullptr);
                }
            }
            float *xw = sXch + (quad * 4 + rank) * 192;
            st2(xw + 2 * lane, sum);
            *reinterpret_cast<uint32_t *>(xw + 64 + lane) = aq;
            *reinterpret_cast<uint32_t *>(xw + 128 + lane) = ak;
            named_bar_sync(bar_id, 128);
            // chunk total, the sum before this warp's first token, the magnitudes
            float2 g = make_float2(0.f, 0.f), before = make_float2(0.f, 0.f);
#pragma unroll
            for (int o = 0; o < 4; ++o) {
                const float *xo = sXch + (quad * 4 + o) * 192;
                const float2 so = ld2(xo + 2 * lane);
                g = fadd2(g, so);
                if (o < rank) before = fadd2(before, so);
                aq = absmax2(aq, *reinterpret_cast<const uint32_t *>(xo + 64 + lane), (T *)nullptr);
                ak = absmax2(ak, *reinterpret_cast<const uint32_t *>(xo + 128 + lane), (T *)nullptr);
            }
            const float2 g2 = fmul2(g, kL2);
            float2 b2 = fmul2(before, kL2);  // log2 gate sum before this warp's first token
            const float2 mq = Pack2<T>::unpack(aq), mk = Pack2<T>::unpack(ak);
            named_bar_sync(bar_id, 128);  // the exchange area is free for the next item
            if (pre) {
                // gate suffix: log2 sum of the segment's chunks after this one
                float2 ga = make_float2(0.f, 0.f);
                if (it > 0) {
                    if (!wwait(&bar_ga[(it - 1) % kStages], ((it - 1) / kStages) & 1, abort, p.err)) break;
                    ga = ld2(sGA + ((it - 1) % kStages) * 64 + 2 * lane);
                }
                if (qw == 0) st2(sGA + (it % kStages) * 64 + 2 * lane, fadd2(ga, g2));
                __syncwarp();  // the warp's stores precede its lane 0's arrive
                if (lane == 0) mbar_arrive(&bar_ga[it % kStages]);
                if (it == npre - 1) {  // the segment's gate totals, for the other segments' folds
                    if (qw == 0) st2(p.aggg + slot * 64 + 2 * lane, fadd2(ga, g2));
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bar_gtot);
                }
                // K^seg = k 2^{GA + g2 - b2}: every factor <= 1.  Rows go in
                // aligned groups of 8: all loads of a group first, then its
                // stores (which only touch rows of the same group).
                const float2 base = fadd2(ga, g2);
#pragma unroll 1
                for (int bq = 0; bq < 4; ++bq) {
                    float2 x[4];
                    uint32_t kw[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int r = r0 + rstep * (4 * bq + e);
                        x[e] = ld2(lat + r * 64 + 2 * lane);
                        kw[e] = *reinterpret_cast<const uint32_t *>(st + ST_K + pair_off(r, lane));
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int r = r0 + rstep * (4 * bq + e);
                        b2 = ffma2(x[e], kL2, b2);
                        const float2 kh = fmul2(Pack2<T>::unpack(kw[e]), ex2_2(fsub2(base, b2)));
                        *reinterpret_cast<uint32_t *>(st + kh_off(r)) = Pack2<T>::pack(kh.x, kh.y);
                    }
                }
            } else {
                bool unsafe = span_unsafe(g2.x, mq.x, mk.x, p.logf2) || span_unsafe(g2.y, mq.y, mk.y, p.logf2);
                unsafe = __any_sync(0xffffffffu, unsafe);  // every warp of the quad sees the same values
                if (!unsafe) {
                    const float2 m2 = make_float2(ref_m2(g2.x, mq.x, mk.x), ref_m2(g2.y, mq.y, mk.y));
                    // pass 2: Q' = q 2^{b2 - m2}, K~ = k 2^{m2 - b2}, in aligned
                    // groups of 8 rows (loads first, then the group's stores).
                    // The state contribution needs K^ = K~ 2^{g2 - m2}: the MMA
                    // reads K~ and the state warps apply the column factor.
#pragma unroll 1
                    for (int bq = 0; bq < 2; ++bq) {
                        float2 x[8];
                        uint32_t qv[8], kv[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int r = r0 + rstep * (8 * bq + e);
                            x[e] = ld2(lat + r * 64 + 2 * lane);
                            qv[e] = *reinterpret_cast<const uint32_t *>(st + ST_Q + pair_off(r, lane));
                            kv[e] = *reinterpret_cast<const uint32_t *>(st + ST_K + pair_off(r, lane));
                        }
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int r = r0 + rstep * (8 * bq + e);
                            b2 = ffma2(x[e], kL2, b2);
                            const float2 d = fsub2(b2, m2);
                            const float2 e1 = ex2_2(d);
                            const float2 e2 = make_float2(fast_exp2(-d.x), fast_exp2(-d.y));
                            const float2 qh = fmul2(Pack2<T>::unpack(qv[e]), e1);
                            const float2 kt = fmul2(Pack2<T>::unpack(kv[e]), e2);
                            *reinterpret_cast<uint32_t *>(st + ST_Q + pair_off(r, lane)) = Pack2<T>::pack(qh.x, qh.y);
                            *reinterpret_cast<uint32_t *>(st + ST_K + pair_off(r, lane)) = Pack2<T>::pack(kt.x, kt.y);
                        }
                    }
                    if (qw == 0) {
                        const int ring = ((it - npre) % kRing) * 64 + 2 * lane;
                        st2(sGam + ring, ex2_2(g2));
                        st2(sEm + ring, ex2_2(m2));
                        st2(sCgm + ring, ex2_2(fsub2(g2, m2)));
                        if (lane == 0) sFlag[s] = 0;
                    }
                } else {
                    // exact scores: b2 (inclusive, log2) in place of log_alpha,
                    // then A[t][s] = sum_i q_ti k_si 2^{b2_ti - b2_si} for token
                    // s <= token t, written straight into the A tile;
                    // Q = q 2^{b2} and K^ = k 2^{g2 - b2} (reference m = 0, K^
                    // in the K~ tile, column factor 1); the state copy S~^T
                    // of these chunks goes to the log_alpha area
                    float *lw = reinterpret_cast<float *>(st + ST_LA);
                    float2 cb = b2;
                    for (int i = 0; i < 16; ++i) {
                        const int r = r0 + rstep * i;
                        cb = ffma2(ld2(lw + r * 64 + 2 * lane), kL2, cb);
                        st2(lw + r * 64 + 2 * lane, cb);
                    }
                    named_bar_sync(bar_id, 128);
                    const int tr = 16 * qw + (lane >> 1), half = lane & 1;  // row t, columns 32 half ..
                    const int tu = rev ? 63 - tr : tr;
                    {
                        float acc[32];
#pragma unroll
                        for (int e = 0; e < 32; ++e) acc[e] = 0.f;
#pragma unroll 1
                        for (int i = 0; i < FD; ++i) {
                            const float qt = to_f32(*reinterpret_cast<const T *>(st + ST_Q + sw128(tr, i >> 3) + (i & 7) * 2));
                            const float bt = lw[tr * 64 + i];
#pragma unroll
                            for (int e = 0; e < 32; ++e) {
                                const int sr = 32 * half + e;
                                const float ks = to_f32(*reinterpret_cast<const T *>(st + ST_K + sw128(sr, i >> 3) + (i & 7) * 2));
                                acc[e] = fmaf(qt * ks, fast_exp2(fminf(bt - lw[sr * 64 + i], 0.f)), acc[e]);
                            }
                        }
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            uint32_t w[4];
#pragma unroll
                            for (int e2 = 0; e2 < 4; ++e2) {
                                const int e = 8 * c + 2 * e2, sr = 32 * half + e;
                                const int su0 = rev ? 63 - sr : sr, su1 = rev ? 62 - sr : sr + 1;
                                const float a0 = (su0 <= tu && tu < len) ? acc[e] : 0.f;
                                const float a1 = (su1 <= tu && tu < len) ? acc[e + 1] : 0.f;
                                w[e2] = Pack2<T>::pack(a0, a1);
                            }
                            *reinterpret_cast<uint4 *>(st + ST_S + sw128(tr, 4 * half + c)) =
                                make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                    named_bar_sync(bar_id, 128);  // every b2, q, k has been read: Q and K^ may overwrite
                    for (int i = 0; i < 16; ++i) {
                        const int r = r0 + rstep * i;
                        const float2 bb = ld2(lw + r * 64 + 2 * lane);
                        uint32_t *qp = reinterpret_cast<uint32_t *>(st + ST_Q + pair_off(r, lane));
                        const uint32_t kw = *reinterpret_cast<const uint32_t *>(st + ST_K + pair_off(r, lane));
                        const float2 qh = fmul2(Pack2<T>::unpack(*qp), ex2_2(bb));
                        const float2 kh = fmul2(Pack2<T>::unpack(kw), ex2_2(fsub2(g2, bb)));
                        *qp = Pack2<T>::pack(qh.x, qh.y);
                        *reinterpret_cast<uint32_t *>(st + ST_K + pair_off(r, lane)) = Pack2<T>::pack(kh.x, kh.y);
                    }
                    if (qw == 0) {
                        const int ring = ((it - npre) % kRing) * 64 + 2 * lane;
                        st2(sGam + ring, ex2_2(g2));
                        st2(sEm + ring, make_float2(1.f, 1.f));
                        st2(sCgm + ring, make_float2(1.f, 1.f));
                        if (lane == 0) sFlag[s] = 1;
                    }
                }
            }
            fence_proxy_async_smem();
            if (!pre) {
                // dS'^T(j) = V^T K~ (the K~ tile read as an MN-major operand),
                // issued by one thread of the quad once every warp's operands
                // are in place and the state warps have read dS buffer j % 2
                named_bar_sync(bar_id, 128);
                if (qw == 0 && lane == 0) {
                    const int j = it - npre;
                    bool ok2 = true;
                    if (j >= 2) ok2 = pwait(&bar_dsf[j & 1], ((j - 2) >> 1) & 1, abort, p.err);
                    if (ok2) {
                        tc_fence_after_sync();
                        const uint32_t sb0 = smem_u32(st);
                        const uint64_t dv = sdesc_sw128(sb0 + ST_V, 8192, 1024), dkt = sdesc_sw128(sb0 + ST_K, 8192, 1024);
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            mma_f16(tbase + TM_DS + 64 * (j & 1), desc_add(dv, ks * 2048), desc_add(dkt, ks * 2048),
                                    idesc(kFmt, 64, 64, 1, 1), ks > 0 ? 1u : 0u);
                        mma_commit(&bar_ds[j & 1]);
                    }
                }
            }
            __syncwarp();  // the warp's operand stores precede its lane 0's arrive
            if (lane == 0) mbar_arrive(&bar_op[s]);
        }
    } else if (warp < kWarpEpi0) {
        // -------------------------------------------------------- state warps
        // Thread element x = 16 half + 4 c + 2 h + e of the M = 64 results in
        // lanes 32 qd + 0..15: row (value dim) v = 16 qd + lane / 4 + 8 h,
        // column (key dim) i = 32 half + 8 c + 2 (lane % 4) + e.
        const int qd = warp & 3, gt = tid - 32 * kWarpSt0;
        const uint32_t lo = (uint32_t)(32 * qd) << 16;
        const int v0 = 16 * qd + (lane >> 2), cq = 2 * (lane & 3);
        bool ok = true;
        float S[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) S[x] = 0.f;
        auto tld = [&](uint32_t col, uint32_t *r) {
            tmem_ld16x256_x4(tbase + lo + col, r);
            tmem_ld16x256_x4(tbase + lo + col + 32, r + 16);
            tmem_ld_wait();
        };
        if (npre > 0) {  // publish the aggregate A_seg^T and raise this segment's flag
            ok = wwait(&bar_pre, 0, abort, p.err) && ok;
            tc_fence_after_sync();
            uint32_t r[32];
            tld(TM_PRE, r);
            tc_fence_before_sync();  // region 2 is read out before the main pass writes it
            float4 *dst = reinterpret_cast<float4 *>(p.agg + slot * 4096);
#pragma unroll
            for (int kb = 0; kb < 8; ++kb)
                dst[kb * 128 + gt] = make_float4(__uint_as_float(r[4 * kb]), __uint_as_float(r[4 * kb + 1]),
                                                 __uint_as_float(r[4 * kb + 2]), __uint_as_float(r[4 * kb + 3]));
            ok = wwait(&bar_gtot, 0, abort, p.err) && ok;
            // One release store publishes everything: the stores above (and the
            // operand warps' gate totals, seen through bar_gtot) precede it
            // through the group barrier, and release is cumulative.
            named_bar_sync(kBarSt, kGroupThreads);
            if (gt == 0 && ok) st_release(p.flag + kWsFlagStride * slot, 1);
        }
        if (seg > 0) {  // fold the earlier segments' aggregates, nearest first
            if (warp == kWarpSt0) {
                bool got = true;
                for (int j = lane; j < seg; j += 32)
                    got = wait_flag(p.flag + kWsFlagStride * ((size_t)bh * p.P + j)) && got;
                if (!__all_sync(0xffffffffu, got) && lane == 0) {
                    *abort = 1;
                    latch_error(p.err, kDevErrTimeout);
                }
            }
            named_bar_sync(kBarSt, kGroupThreads);
            if (*abort) ok = false;
            // sGt[d][i]: log2 gate sum, per key dim, of the segments between
            // segment seg - 1 - d and this one (the decay of that aggregate)
            if (ok && gt < 64) {
                float a = 0.f;
                for (int d = 0; d < seg; ++d) {
                    sGt[d * 64 + gt] = a;
                    a += __ldcg(p.aggg + ((size_t)bh * p.P + (seg - 1 - d)) * 64 + gt);
                }
            }
            named_bar_sync(kBarSt, kGroupThreads);
            // half an aggregate in flight while the previous half is folded:
            // each 16-byte piece is reloaded with the next half's as soon as it
            // has been read
            auto agg_at = [&](int d) {
                return reinterpret_cast<const float4 *>(p.agg + ((size_t)bh * p.P + (seg - 1 - d)) * 4096) + gt;
            };
            float4 va[4];
            if (ok) {
                const float4 *ag = agg_at(0);
#pragma unroll
                for (int kb = 0; kb < 4; ++kb) va[kb] = __ldcg(ag + kb * 128);
            }
            for (int d = 0; d < seg && ok; ++d) {
                const float *dec = sGt + d * 64;
                const float4 *nx1 = agg_at(d) + 4 * 128;                  // this aggregate, blocks 4..7
                const float4 *nx0 = agg_at(d + 1 < seg ? d + 1 : d);     // the next one, blocks 0..3
#pragma unroll
                for (int kb = 0; kb < 8; ++kb) {
                    // block kb = 4 half + c: columns i0, i0 + 1 of rows v0 and v0 + 8
                    const int c = kb & 3;
                    const float4 x = va[c];
                    if (kb < 4) va[c] = __ldcg(nx1 + c * 128);
                    else if (d + 1 < seg) va[c] = __ldcg(nx0 + c * 128);
                    const int i0 = 8 * kb + cq;
                    const float2 f = ex2_2(ld2(dec + i0));
                    S[4 * kb] = fmaf(f.x, x.x, S[4 * kb]);
                    S[4 * kb + 1] = fmaf(f.y, x.y, S[4 * kb + 1]);
                    S[4 * kb + 2] = fmaf(f.x, x.z, S[4 * kb + 2]);
                    S[4 * kb + 3] = fmaf(f.y, x.w, S[4 * kb + 3]);
                }
            }
        }
        // Main pass: S~_j = e^{m_j} S_j into the B tile of chunk j's stage,
        // then S_{j+1} = diag(e^{g_j}) S_j + diag(e^{g_j - m_j}) dS'_j (dS'
        // from the MMA on K~; the factors of chunk j sit in ring slot j % 8).
        bool range_ok = true;
        auto update = [&](int jp) {  // S <- diag(gam) S + diag(cgm) dS'(jp)
            ok = wwait(&bar_ds[jp & 1], (jp >> 1) & 1, abort, p.err) && ok;
            tc_fence_after_sync();
            const float *gm = sGam + (jp % kRing) * 64, *cg = sCgm + (jp % kRing) * 64;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {  // 32 columns at a time
                uint32_t r[16];
                tmem_ld16x256_x4(tbase + lo + TM_DS + 64 * (jp & 1) + 32 * hf, r);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int kb = 4 * hf + c, i0 = 8 * kb + cq;
                    const float2 ga = ld2(gm + i0), cf = ld2(cg + i0);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int x = 4 * kb + 2 * h, y = 4 * c + 2 * h;
                        S[x] = fmaf(ga.x, S[x], cf.x * __uint_as_float(r[y]));
                        S[x + 1] = fmaf(ga.y, S[x + 1], cf.y * __uint_as_float(r[y + 1]));
                    }
                }
            }
            tc_fence_before_sync();
            mbar_arrive(&bar_dsf[jp & 1]);
        };
        for (int j = 0; j < L; ++j) {
            const int it = npre + j, s = it % kStages;
            if (j > 0) update(j - 1);
            ok = wwait(&bar_op[s], (it / kStages) & 1, abort, p.err) && ok;
            uint8_t *sb = sm + s * ST_BYTES + (sFlag[s] ? ST_LA : ST_S);
            const float *emr = sEm + (j % kRing) * 64;
#pragma unroll
            for (int kb = 0; kb < 8; ++kb) {
                const int i0 = 8 * kb + cq;
                const float2 em = ld2(emr + i0);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float a0 = em.x * S[4 * kb + 2 * h], a1 = em.y * S[4 * kb + 2 * h + 1];
                    if (!BF16) range_ok = range_ok && fabsf(a0) <= 65504.f && fabsf(a1) <= 65504.f;
                    *reinterpret_cast<uint32_t *>(sb + sw128(v0 + 8 * h, i0 >> 3) + (i0 & 7) * 2) =
                        Pack2<T>::pack(a0, a1);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            named_bar_sync(kBarSt, kGroupThreads);
            // [scores | o] = Q' [K~ ; S~^T]^T into TMEM region j % 3 (free once
            // the epilogue has read the output of chunk j - 3), issued by one
            // thread of the group; exact-score chunks: only o = Q S~ (S~^T
            // in the log_alpha area)
            if (gt == 0) {
                const int rg = j % 3;
                if (j >= 3) ok = pwait(&bar_rf[rg], ((j - 3) / 3) & 1, abort, p.err) && ok;
                if (ok) {
                    tc_fence_after_sync();
                    const uint32_t sb0 = smem_u32(sm + s * ST_BYTES);
                    const uint64_t dq = sdesc_sw128(sb0 + ST_Q, 16, 1024);
                    if (!sFlag[s]) {
                        const uint64_t db = sdesc_sw128(sb0 + ST_K, 16, 1024);  // K~ rows, then S~^T rows
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            mma_f16(tbase + 128 * rg, desc_add(dq, ks * 32), desc_add(db, ks * 32),
                                    idesc(kFmt, 64, 128, 0, 0), ks > 0 ? 1u : 0u);
                    } else {
                        const uint64_t dsq = sdesc_sw128(sb0 + ST_LA, 16, 1024);
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            mma_f16(tbase + 128 * rg + 64, desc_add(dq, ks * 32), desc_add(dsq, ks * 32),
                                    idesc(kFmt, 64, 64, 0, 0), ks > 0 ? 1u : 0u);
                    }
                    mma_commit(&bar_sc[rg]);
                }
            }
        }
        if (L > 0 && !(seg == p.P - 1 && p.final_state)) {
            // no final state wanted: still wait for the last dS product
            ok = wwait(&bar_ds[(L - 1) & 1], ((L - 1) >> 1) & 1, abort, p.err) && ok;
        }
        if (L > 0 && seg == p.P - 1 && p.final_state) {
            update(L - 1);
            if (ok) {
                float *fs = p.final_state + (size_t)bh * p.fs_bh;
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                    const int i = 32 * (x >> 4) + 8 * ((x >> 2) & 3) + cq + (x & 1);
                    const int v = v0 + 8 * ((x >> 1) & 1);
                    fs[(size_t)i * p.fs_ld + v] = S[x];
                }
            }
        }
    } else {
        // ----------------------------------------------------- epilogue warps
        // Thread element x = 16 half + 4 c + 2 h + e: row (token's stage row)
        // t = 16 qd + lane / 4 + 8 h, column 32 half + 8 c + 2 (lane % 4) + e.
        // Per chunk: causal mask of the scores and the A V product (onto the
        // q S columns), then the output staged through the (by then unused)
        // Q' tile in 128-byte swizzled rows and stored with coalesced 16-byte
        // stores (8 threads per 128-byte output row) at the raster rows.
        const int qd = warp & 3, et = tid - 32 * kWarpEpi0;
        const uint32_t lo = (uint32_t)(32 * qd) << 16;
        const int t0r = 16 * qd + (lane >> 2), cq = 2 * (lane & 3);
        bool ok = true;
        for (int j = 0; j < L; ++j) {
            const int it = npre + j, s = it % kStages, rg = j % 3;
            ok = wwait(&bar_op[s], (it / kStages) & 1, abort, p.err) && ok;  // row table, flag
            ok = wwait(&bar_sc[rg], (j / 3) & 1, abort, p.err) && ok;
            tc_fence_after_sync();
            if (!sFlag[s]) {
                uint8_t *sa = sm + s * ST_BYTES + ST_LA;  // free once the operands are made
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {  // 32 columns at a time
                    uint32_t r[16];
                    tmem_ld16x256_x4(tbase + lo + 128 * rg + 32 * hf, r);
                    tmem_ld_wait();
                    // causal mask in stage-row coordinates: token s <= token t
#pragma unroll
                    for (int x = 0; x < 16; x += 2) {
                        const int t = t0r + 8 * ((x >> 1) & 1), sx = 32 * hf + 8 * (x >> 2) + cq;
                        const bool k0 = rev ? (sx >= t) : (sx <= t), k1 = rev ? (sx + 1 >= t) : (sx + 1 <= t);
                        const float a0 = k0 ? __uint_as_float(r[x]) : 0.f, a1 = k1 ? __uint_as_float(r[x + 1]) : 0.f;
                        *reinterpret_cast<uint32_t *>(sa + sw128(t, sx >> 3) + (sx & 7) * 2) = Pack2<T>::pack(a0, a1);
                    }
                }
                fence_proxy_async_smem();
            }  // exact-score chunks: the operand warps wrote A before releasing the stage
            tc_fence_before_sync();
            named_bar_sync(kBarEpi, kGroupThreads);
            if (et == 0 && ok) {  // o += A V, issued by one thread of the group
                tc_fence_after_sync();
                const uint32_t sb0 = smem_u32(sm + s * ST_BYTES);
                const uint64_t da = sdesc_sw128(sb0 + (sFlag[s] ? ST_S : ST_LA), 16, 1024);
                const uint64_t dv = sdesc_sw128(sb0 + ST_V, 8192, 1024);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(tbase + 128 * rg + 64, desc_add(da, ks * 32), desc_add(dv, ks * 2048),
                            idesc(kFmt, 64, 64, 0, 1), 1u);
                mma_commit(&bar_o[rg]);
            }
            // output of chunk j
            ok = wwait(&bar_o[rg], (j / 3) & 1, abort, p.err) && ok;
            tc_fence_after_sync();
            uint8_t *sq = sm + s * ST_BYTES + ST_Q;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t r[16];
                tmem_ld16x256_x4(tbase + lo + 128 * rg + 64 + 32 * hf, r);
                tmem_ld_wait();
#pragma unroll
                for (int x = 0; x < 16; x += 2) {
                    const int t = t0r + 8 * ((x >> 1) & 1), col = 32 * hf + 8 * (x >> 2) + cq;
                    *reinterpret_cast<uint32_t *>(sq + sw128(t, col >> 3) + (col & 7) * 2) =
                        Pack2<T>::pack(__uint_as_float(r[x]), __uint_as_float(r[x + 1]));
                }
            }
            tc_fence_before_sync();
            mbar_arrive(&bar_rf[rg]);
            named_bar_sync(kBarEpi, kGroupThreads);
            const int *rows = sRows + s * 64;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int idx = e * kGroupThreads + et, t = idx >> 3, c = idx & 7;
                const int row = rows[t];
                if (ok && row >= 0) {
                    uint4 w = *reinterpret_cast<const uint4 *>(sq + sw128(t, c));
                    uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<T *>(p.out) + (size_t)row * p.ldo + 8 * c);
                    if (p.acc_out) {  // second key half: add to the first half's output
                        const uint4 o = *dst;
                        const float2 a0 = Pack2<T>::unpack(o.x), a1 = Pack2<T>::unpack(o.y),
                                     a2 = Pack2<T>::unpack(o.z), a3 = Pack2<T>::unpack(o.w);
                        const float2 b0 = Pack2<T>::unpack(w.x), b1 = Pack2<T>::unpack(w.y),
                                     b2 = Pack2<T>::unpack(w.z), b3 = Pack2<T>::unpack(w.w);
                        w = make_uint4(Pack2<T>::pack(a0.x + b0.x, a0.y + b0.y), Pack2<T>::pack(a1.x + b1.x, a1.y + b1.y),
                                       Pack2<T>::pack(a2.x + b2.x, a2.y + b2.y), Pack2<T>::pack(a3.x + b3.x, a3.y + b3.y));
                    }
                    *dst = w;
                }
            }
            named_bar_sync(kBarEpi, kGroupThreads);
            if (et == 0) mbar_arrive(&bar_empty[s]);
        }
    }

    // ------------------------------------------------------------- teardown
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == kWarpLoad) tmem_dealloc(tbase, kTmemCols);
    if (tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&p.ctr[1], 1u);
        s_last = (prev == gridDim.x - 1) ? 1 : 0;
    }
    __syncthreads();
    if (s_last) {  // last CTA to finish: leave the workspace ready for the next call
        if (p.P > 1)
            for (int idx = tid; idx < p.BH * p.P; idx += kThreads) p.flag[kWsFlagStride * idx] = 0;
        if (tid == 0) {
            p.ctr[0] = 0;
            p.ctr[1] = 0;
        }
        __threadfence();
    }
}

constexpr int kSMs = 148;

struct Plan {
    int nc, P, L;
};

// Segments per (b,h).  More segments put more SMs to work and shorten each
// CTA's serial chain of chunks, but every segment except the last adds a
// pre-pass over its chunks and every segment folds all earlier aggregates.
// The choice minimises a time model of this kernel on B200 (microseconds):
// a main-pass chunk, a pre-pass chunk, one folded aggregate, and the fixed
// cost of publishing and waiting for flags; CTAs beyond one per SM run in
// further waves.
Plan make_plan(const Problem &pr) {
    constexpr double kMain = 0.9, kPre = 0.5, kFold = 0.35, kFlag = 2.0;
    Plan best{0, 1, 1};
    const int nc = (pr.n + FC - 1) / FC;
    const int bh = pr.B * pr.H;
    double tbest = 1e30;
    const int pmax = nc < kMaxSegments ? nc : kMaxSegments;
    for (int P = 1; P <= pmax; ++P) {
        const int L = (nc + P - 1) / P;
        if ((nc + L - 1) / L != P) continue;
        if (P > 1 && (long long)bh * P > kWsMaxFlags) break;
        const long long waves = ((long long)bh * P + kSMs - 1) / kSMs;
        const double t = waves * L * (kMain + (P > 1 ? kPre : 0.0)) + (P - 1) * kFold + (P > 1 ? kFlag : 0.0);
        if (t < tbest) {
            tbest = t;
            best = Plan{nc, P, L};
        }
    }
    best.nc = nc;
    return best;
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
    if ((pr.dk != 64 && pr.dk != 128) || (pr.dv != 64 && pr.dv != 128) || pr.chunk != 64) return false;
    if ((long long)pr.B * pr.H * pr.n >= (1LL << 31)) return false;
    return true;
}

size_t fused_workspace_bytes(const Problem &pr) { return ws_layout(pr, make_plan(pr)).total; }

// One launch for the 64-wide sub-problem (key half kh, value half vh).
static int launch_fused_part(const Problem &pr, const Plan &pl, const WsLayout &wl, void *ws,
                             int kh, int vh, cudaStream_t st) {
    FusedParams p;
    memset(&p, 0, sizeof(p));
    char *w = static_cast<char *>(ws);
    const CUtensorMapDataType dt16 =
        pr.dtype == GTR_GLA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const uint64_t bh = (uint64_t)pr.B * pr.H;
    int boxh = FC;
    if (pr.dir >= 2) {
        boxh = 1;
        while (boxh < FC && pr.gh % (2 * boxh) == 0) boxh *= 2;
        if (boxh < 8) boxh = 0;
    }
    // views of the 64 columns starting at col0 of a [BH][n][ld] tensor
    auto enc = [&](CUtensorMap *m, const void *base0, int ld, int col0, CUtensorMapDataType dt, uint64_t es,
                   bool sw) {
        const void *base = static_cast<const char *>(base0) + (size_t)col0 * es;
        const uint64_t row = (uint64_t)ld * es;
        if (boxh == 0) {  // [BH*n][64], one row per box (gathers)
            const uint64_t dims[2] = {FD, bh * pr.n};
            const uint64_t str[1] = {row};
            const uint32_t box[2] = {FD, 1};
            return encode_tile_map(m, base, dt, 2, dims, str, box, sw);
        }
        if (pr.dir < 2) {  // [BH][n][64]
            const uint64_t dims[3] = {FD, (uint64_t)pr.n, bh};
            const uint64_t str[2] = {row, (uint64_t)pr.n * row};
            const uint32_t box[3] = {FD, FC, 1};
            return encode_tile_map(m, base, dt, 3, dims, str, box, sw);
        }
        // [BH][gh][gw][64]
        const uint64_t dims[4] = {FD, (uint64_t)pr.gw, (uint64_t)pr.gh, bh};
        const uint64_t str[3] = {row, (uint64_t)pr.gw * row, (uint64_t)pr.n * row};
        const uint32_t box[4] = {FD, 1, (uint32_t)boxh, 1};
        return encode_tile_map(m, base, dt, 4, dims, str, box, sw);
    };
    if (enc(&p.tm_q, pr.q, pr.dk, FD * kh, dt16, 2, true) || enc(&p.tm_k, pr.k, pr.dk, FD * kh, dt16, 2, true) ||
        enc(&p.tm_v, pr.v, pr.dv, FD * vh, dt16, 2, true) ||
        enc(&p.tm_la, pr.la, pr.dk, FD * kh, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, false))
        return GTR_GLA_ERR_CUDA;
    p.boxh = boxh;
    p.out = static_cast<char *>(pr.out) + (size_t)FD * vh * 2;
    p.ldo = pr.dv;
    p.acc_out = kh > 0;
    p.final_state = pr.final_state ? pr.final_state + (size_t)FD * kh * pr.dv + FD * vh : nullptr;
    p.fs_bh = pr.dk * pr.dv;
    p.fs_ld = pr.dv;
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
    // fp16 operands stay below 2^15 (half the type's range, for the sums
    // inside a product); bf16 has fp32's exponent range
    p.logf2 = pr.dtype == GTR_GLA_BF16 ? 100.f : 15.f;
    const dim3 grid(p.BH * p.P);
    // one instantiation per I/O dtype and scan sense (reversed scans walk the
    // stage rows backwards, which fixes every shared-memory offset at compile time)
    const void *fn = nullptr;
    const bool rev = pr.dir & 1;
    if (pr.dtype == GTR_GLA_BF16)
        fn = rev ? (const void *)gla_fused_kernel<true, true> : (const void *)gla_fused_kernel<true, false>;
    else
        fn = rev ? (const void *)gla_fused_kernel<false, true> : (const void *)gla_fused_kernel<false, false>;
    if (ensure_smem(fn, SMEM_BYTES)) return GTR_GLA_ERR_CUDA;
    if (pr.dtype == GTR_GLA_BF16) {
        if (rev)
            gla_fused_kernel<true, true><<<grid, kThreads, SMEM_BYTES, st>>>(p);
        else
            gla_fused_kernel<true, false><<<grid, kThreads, SMEM_BYTES, st>>>(p);
    } else {
        if (rev)
            gla_fused_kernel<false, true><<<grid, kThreads, SMEM_BYTES, st>>>(p);
        else
            gla_fused_kernel<false, false><<<grid, kThreads, SMEM_BYTES, st>>>(p);
    }
    note_launch();
    return cudaPeekAtLastError() == cudaSuccess ? GTR_GLA_OK : GTR_GLA_ERR_CUDA;
}

// Head sizes of 128 run as 64-wide sub-problems, one launch each, in stream
// order: first every value half of key half 0 (which writes the output),
// then key half 1 (which adds to it).  The launches share the workspace; each
// leaves its header zeroed for the next.
int launch_fused(const Problem &pr, void *ws, cudaStream_t st) {
    const Plan pl = make_plan(pr);
    const WsLayout wl = ws_layout(pr, pl);
    for (int kh = 0; kh < pr.dk / FD; ++kh)
        for (int vh = 0; vh < pr.dv / FD; ++vh) {
            const int rc = launch_fused_part(pr, pl, wl, ws, kh, vh, st);
            if (rc != GTR_GLA_OK) return rc;
        }
    return GTR_GLA_OK;
}

}  // namespace gtr
