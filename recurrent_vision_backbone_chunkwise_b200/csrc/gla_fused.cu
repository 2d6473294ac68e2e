// gla_fused.cu -- single-kernel chunkwise GLA forward on sm_100a tensor cores
// (fp16 / bf16 I/O, d_k = d_v = 64, chunk 64), warp-specialised.
//
// The chunkwise reorganisation of "GTR: Gated Token Recurrence for Efficient
// Dense Prediction" (x-techcon article, section 算子) -- chunks compute their
// own state contribution in parallel, boundary states are passed along, each
// chunk's output is produced in parallel, scores stay on chip -- mapped onto
// one launch of 576-thread CTAs, one per SM (head sizes of 128 run as one
// launch per 64-wide key half, both value halves in it, see launch_fused):
//
//   * a CTA owns a segment of consecutive 64-token chunks of one (b,h); when
//     the CTAs may run in several waves they take their segment from a
//     ticket counter, so a segment only ever waits for segments that were
//     started before it; one-wave plans run as a cooperative launch;
//   * pre-pass (every segment but the last of its (b,h)): the segment's
//     aggregate state contribution, transposed,
//       A_seg^T = sum_c V_c^T (k_c . e^{G_after(c) + g_c - b_c}),
//     accumulates in TMEM (chunks visited last to first, every factor <= 1)
//     and is published with the segment's gate totals (one release store of
//     a flag with a cache line of its own);
//   * boundary: the incoming state S_in = sum_j diag(e^{G(j..seg)}) A_j over
//     the earlier segments' aggregates, by a transposed scan across the
//     plane's CTAs (cooperative launches: each CTA scans a slice of the state
//     elements through all segments) or by each segment folding the earlier
//     aggregates, nearest first (a fixed order either way: results are
//     bitwise reproducible);
//   * main pass, chunk by chunk:
//       scores = Q^ K~^T        (tf32 MMA; Q^ = q . e^{b}, K~ = k . e^{-b},
//                                b: in-chunk inclusive log-gate sums)
//       dS^T   = V^T K^         (f16/bf16 MMA; K^ = k . e^{g - b})
//       A      = causal mask of the scores, re-quantised to the I/O dtype
//       o      = Q^ S_in + A V  (tf32 + f16/bf16 MMAs into one accumulator)
//       S      <- diag(e^{g}) S + dS   (fp32, registers of the epilogue warps)
//
// Roles (warps):
//   0       producer: row tables and TMA tile loads (row scans: one box per
//           tensor; column scans: column slabs, or four-row gathers) of q,
//           k, v, log_alpha into a 3-stage ring, in scan order, so every
//           direction reads and writes the row-major grid in place;
//   1       MMA issue (one lane) and TMEM allocation;
//   2..9    operand warps, 8 token rows each: gate factors (one exponential
//           per element, running products), Q^ / K~ (tf32, written over
//           log_alpha / q,k in place) and K^ (f16/bf16);
//   10..17  epilogue warps, two per TMEM lane quadrant (32 columns each):
//           state update (state in registers, a tf32 copy in shared memory
//           as the next chunk's MMA operand), causal mask, output stores,
//           the fold, the aggregate's publication.
// Per chunk k the MMA warp issues A V of chunk k-1 as soon as its mask is in
// shared memory (this releases that chunk's stage early), then dS of chunk
// k, then the scores of chunk k once state k is in its stage; the epilogue
// updates the state, masks chunk k and stores chunk k-1's output.
//
// Chunks whose in-chunk gate span exceeds kSpanLimit (e^{-b} would leave fp32
// range) get their scores from an exact CUDA-core evaluation by the operand
// warps (every factor <= 1), stored straight into TMEM.
#include <algorithm>
#include <cstring>
#include <map>
#include <mutex>
#include <type_traits>

#include "gla_common.cuh"
#include "gla_internal.h"
#include "sm100.cuh"

namespace gtr {
using namespace sm100;

namespace {

constexpr int FC = 64;  // tokens per chunk
constexpr int FD = 64;  // d_k = d_v
constexpr int kStages = 3;
constexpr int kOpWarps = 8, kEpiWarps = 8;
constexpr int kWarpLoad = 0, kWarpMma = 1, kWarpOp0 = 2, kWarpEpi0 = kWarpOp0 + kOpWarps;
constexpr int kThreads = 32 * (kWarpEpi0 + kEpiWarps);
constexpr int kOpThreads = 32 * kOpWarps, kEpiThreads = 32 * kEpiWarps;
constexpr int kBarOp = 1, kBarEpi = 2;  // named barrier ids
constexpr int kMaxSegments = 64;        // segments per (b,h): bounds the fold
constexpr int kFoldDepth = 3;           // aggregates in flight during the fold
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kSpanLimit = 80.f;  // max -g (natural log) for the factorised scores

// One pipeline stage (byte offsets from the stage base, every tile 1024-aligned).
// Bytes [0, 32K) are the B operand of the merged product [scores | q S]: a
// tf32 K-major tile [2 blocks of 32 K][128 rows][128 B], rows 0-63 K~
// (tokens, written over q and k) and rows 64-127 S^T (value dims: the state
// entering this chunk, written by the epilogue warps).
constexpr uint32_t ST_Q = 0;       // q  [64 tok][128 B] plain rows -> K~, first 32 K
constexpr uint32_t ST_K = 16384;   // k  [64 tok][128 B] plain rows -> K~, second 32 K
constexpr uint32_t ST_LA = 32768;  // log_alpha [64 tok][256 B] fp32 -> Q^ (tf32, 16 KB)
constexpr uint32_t ST_V = 49152;   // v  [64 tok][128 B] SW128 (MN-major MMA operand)
constexpr uint32_t ST_KH = 57344;  // K^ [64 i][128 B] SW128 K-major
constexpr uint32_t ST_BYTES = 65536;
constexpr uint32_t ST_B1 = 0, ST_QH = ST_LA;
constexpr uint32_t OFF_A = kStages * ST_BYTES;  // A f16/bf16 K-major [2][8 KB]
constexpr uint32_t OFF_MISC = OFF_A + 2 * 8192;
constexpr uint32_t MISC_ROWS = 0;     // int   [kStages][64] global row of each token
constexpr uint32_t MISC_GAM = 768;    // float [kStages][64] e^{g}
constexpr uint32_t MISC_LEN = 1536;   // int   [kStages] tokens in the chunk
constexpr uint32_t MISC_FLAG = 1552;  // int   [kStages] exact-score chunk
constexpr uint32_t MISC_TOT = 2048;   // float [2][kOpWarps][64] operand warps' row-block log sums
constexpr uint32_t MISC_TAIL = 6144;  // float [2][2][64] output tail: half-row sums of squares
constexpr uint32_t MISC_BYTES = 8192;
// gate totals of the plane's segments, staged for the transposed scan
constexpr uint32_t OFF_SCAN = OFF_MISC + MISC_BYTES;
constexpr uint32_t SCAN_BYTES = 8192;
constexpr int kMaxScanSegments = 33;  // (P - 1) * 64 gate totals fit SCAN_BYTES
constexpr uint32_t SMEM_BYTES = OFF_SCAN + SCAN_BYTES + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory");
static_assert(MISC_TOT + 2 * kOpWarps * 64 * 4 <= MISC_TAIL && MISC_TAIL + 1024 <= MISC_BYTES, "misc area");
static_assert(kMaxSegments * 64 * 4 <= 2 * 8192, "the fold stages every gate total in the A buffers");
static_assert((kMaxScanSegments - 1) * 64 * 4 <= SCAN_BYTES, "scan gate totals");
// the scan stages its slice of every aggregate, (2048 / P + 1) (P - 1) pairs,
// in the A buffers
static_assert((2048 / kMaxScanSegments + 1) * (kMaxScanSegments - 1) * 8 <= 2 * 8192, "scan slice");
static_assert((kMaxScanSegments - 1) * 64 <= 8 * 256 && (2048 / kMaxScanSegments + 1) * (kMaxScanSegments - 1) <= 8 * 256,
              "the scan's loads take one pass of the 256 epilogue threads");
static_assert(FC % kOpWarps == 0 && FC / kOpWarps == 8, "operand warps own 8 tokens each");

constexpr uint32_t kTmemCols = 512;
// TMEM columns (M = 64 results, lanes 32 q + 0..15): three regions of 128
// columns, [scores | o] of chunk k in region k % 3; dS^T in two buffers by
// chunk parity; the pre-pass aggregate borrows region 2 (free until main
// chunk 2, which is issued only after the aggregate has been published).
constexpr uint32_t TM_R = 0, TM_DS = 384, TM_PRE = 256;

struct FusedParams {
    // Tiled views of q, k, v, log_alpha.  Row scans (L->R, R->L): [BH][n][64],
    // one 64-row box per chunk.  Column scans (T->B, B->T): [BH][gh][gw][64],
    // boxes of `boxh` consecutive grid rows of one column (boxh: the largest
    // power of two <= 64 that divides grid_h, so no box crosses a column).
    CUtensorMap tm_q, tm_k, tm_v, tm_la;
    // head sizes d_v = 128: the second value half's tile view (the launch's
    // planes are (value half, b, h), value half slowest)
    CUtensorMap tm_v2;
    const void *q, *k, *v;
    const float *la;
    void *out;
    float *final_state;
    float *agg;     // [BH*P][64*64] segment aggregate states, transposed ([j][i])
    float *aggg;    // [BH*P][64]    segment log-gate totals
    int *flag;      // [BH*P] 0 empty, 1 aggregate published
    float *sin;     // [BH*P][64*64] incoming states S_in^T of the segments (coop)
    int *flag2;     // [BH*P] 1: this CTA's slice of every S_in is written (coop)
    unsigned *ctr;  // [0] ticket, [1] finished CTAs
    int *err;
    int n, gh, gw, dir, nc, P, L;
    int BH;   // planes of this launch: BHt x nvh
    int BHt;  // planes of the tensors (B H)
    int nvh;  // value halves processed by this launch (1, or 2 when d_v = 128)
    // coop: every CTA is resident at once (cooperative launch) and the
    // boundary states come from the transposed scan; otherwise each segment
    // folds the earlier aggregates itself
    int coop;
    // the segment that holds the chunks left over, nc - (P - 1) L of them:
    // the last (0) or the first (1; it starts its main pass without waiting
    // for the scan's second round, its incoming state being zero)
    int rem_first;
    // Head sizes of 128 run as 64-wide sub-problems (every key row of the
    // state evolves on its own and every value column too; the output is
    // the sum over the key halves): `out` is the output, `final_state` the
    // key half's first row of it (each value half adds 64 columns), ldo the
    // output row stride in elements, acc_out adds to what is already in
    // `out`, fs_bh / fs_ld the final state's (b,h) and row strides.
    int ldo, acc_out, fs_bh, fs_ld;
    int boxh;  // rows per box (64 for row scans); 0: four-row gathers (column
               // scans whose grid_h is not a multiple of 8, where a box of V
               // could not start on its 128-byte swizzle atom)
    // Output tail (TAIL kernels, d_k = d_v = 64): y[b, r, h, :] = o / sqrt(mean
    // o^2 + eps) * wn[h] * SiLU(z[b, r, h, :]) with z and y [B, n, H, 64] in
    // the I/O dtype and wn [H, 64] fp32; `out` is not written.
    const void *z;
    const float *wn;
    void *y;
    float eps;
    int H;
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

// Polling side of a pipeline wait, bounded (about 2 s): the first wait that
// gives up raises `abort`, after which every wait returns at once, so all
// threads reach the end of the kernel.  It spins on try_wait for about a
// microsecond, then backs off with short sleeps (from the start when
// `sleep_ns` is set): a waiting warp must not take issue slots from the
// warps doing the work.  Returns false when aborted.
__device__ bool pwait(uint64_t *bar, uint32_t parity, volatile int *abort, int *err,
                      uint32_t sleep_ns = 0) {
    if (mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t n = 0;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 7) == 7) {
            if (*abort) return false;
            const uint64_t dt = global_timer_ns() - t0;
            if (dt > 2000000000ull) {
                *abort = 1;
                latch_error(err, kDevErrTimeout);
                return false;
            }
            if (sleep_ns || dt > 1000) __nanosleep(sleep_ns ? sleep_ns : 64);
        }
    }
}

// A group of warps waits through one polling thread; the group's named
// barrier (id, count threads) releases the others.  Returns false when aborted.
__device__ __forceinline__ bool gwait(bool leader, int id, int count, uint64_t *bar, uint32_t parity,
                                      volatile int *abort, int *err, uint32_t sleep_ns = 0) {
    if (leader) pwait(bar, parity, abort, err, sleep_ns);
    named_bar_sync(id, count);
    return *abort == 0;
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

template <typename T>
__device__ __forceinline__ uint4 pack8(const float *x) {
    uint4 w;
    w.x = Pack2<T>::pack(x[0], x[1]);
    w.y = Pack2<T>::pack(x[2], x[3]);
    w.z = Pack2<T>::pack(x[4], x[5]);
    w.w = Pack2<T>::pack(x[6], x[7]);
    return w;
}

// byte offset of tf32 element (row, k) in a K-major [2 blocks of 32][64 rows][128 B] tile
__device__ __forceinline__ uint32_t tf32_kmaj(int row, int k) {
    return (k >> 5) * 8192 + sw128(row, (k & 31) >> 2) + (k & 3) * 4;
}

// the same for the stage's 128-row B tile (rows 0-63 K~, 64-127 S^T)
__device__ __forceinline__ uint32_t b1_off(int row, int k) {
    return (k >> 5) * 16384 + sw128(row, (k & 31) >> 2) + (k & 3) * 4;
}

// A shared-memory descriptor advanced by `bytes` (the start address field
// holds addr >> 4 in its low 14 bits; smem addresses stay far below 256 KiB).
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t bytes) {
    return d + (uint64_t)(bytes >> 4);
}

__device__ __forceinline__ float2 ld2(const float *p) { return *reinterpret_cast<const float2 *>(p); }
__device__ __forceinline__ void st2(float *p, float2 v) { *reinterpret_cast<float2 *>(p) = v; }
__device__ __forceinline__ float2 ex2_2(float2 x) {
    return make_float2(fast_exp2(x.x * kLog2e), fast_exp2(x.y * kLog2e));
}

template <bool BF16, bool TAIL>
__global__ void __launch_bounds__(kThreads, 1) gla_fused_kernel(const __grid_constant__ FusedParams p) {
    using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
    extern __shared__ uint8_t smem_raw[];
    // 1024-aligned base; offset arithmetic on the array keeps shared-memory
    // accesses in the shared state space (no generic loads)
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    int *sRows = reinterpret_cast<int *>(sm + OFF_MISC + MISC_ROWS);
    float *sGam = reinterpret_cast<float *>(sm + OFF_MISC + MISC_GAM);
    float *sTot = reinterpret_cast<float *>(sm + OFF_MISC + MISC_TOT);
    int *sLen = reinterpret_cast<int *>(sm + OFF_MISC + MISC_LEN);
    int *sFlag = reinterpret_cast<int *>(sm + OFF_MISC + MISC_FLAG);

    __shared__ uint64_t bar_full[kStages], bar_empty[kStages], bar_op[kStages];
    __shared__ uint64_t bar_sc[2], bar_o[2], bar_a[2], bar_s[2], bar_ds[2];
    __shared__ uint64_t bar_pre, bar_owpre, bar_fin, bar_pub;
    __shared__ uint32_t s_tmem;
    __shared__ int s_ticket, s_last;
    __shared__ volatile int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    unsigned arrival = 0;  // coop: this CTA's place in the arrival count (header check)
    // (no descriptor prefetch: on B200 each prefetch.tensormap held the issuing
    // thread for about 0.45 us; the first copy of each map fetches it anyway)
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bar_full[s], 1);  // producer lane 0 (with the stage's TMA bytes)
            mbar_init(&bar_empty[s], 1);
            mbar_init(&bar_op[s], kOpThreads);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar_sc[b], 1);
            mbar_init(&bar_o[b], 1);
            mbar_init(&bar_ds[b], 1);
            mbar_init(&bar_a[b], kEpiThreads);
            mbar_init(&bar_s[b], kEpiThreads);
        }
        mbar_init(&bar_pre, 1);
        mbar_init(&bar_owpre, kOpThreads);
        mbar_init(&bar_fin, 1);
        mbar_init(&bar_pub, kEpiThreads);
        fence_mbar_init();
        // A cooperative launch has every CTA resident, so the block index can
        // name the segment; the arrival count is still kept (its value is
        // only checked at the end, off the critical path).  Otherwise the
        // ticket order guarantees that a CTA only waits for earlier ones.
        if (p.coop) {
            arrival = atomicAdd(&p.ctr[0], 1u);
            s_ticket = (int)blockIdx.x;
        } else {
            s_ticket = (int)atomicAdd(&p.ctr[0], 1u);
        }
        s_abort = 0;
    }
    for (int e = tid; e < kStages * 64; e += kThreads) sRows[e] = 0;
    if (warp == kWarpMma) {
        tmem_alloc(&s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tbase = s_tmem;
    const int ticket = s_ticket;
    // launch plane bhf = (value half, tensor plane bh), segment seg
    const int bhf = ticket / p.P, seg = ticket % p.P;
    const int vpart = bhf / p.BHt, bh = bhf - vpart * p.BHt;
    // every segment has L chunks but one, which has the rest (possibly more):
    // the last, or with rem_first the first
    const int rem = p.nc - (p.P - 1) * p.L;
    const int c_begin = p.rem_first ? (seg == 0 ? 0 : rem + (seg - 1) * p.L) : seg * p.L;
    const int c_end = p.rem_first ? (seg == 0 ? rem : c_begin + p.L)
                                  : ((seg == p.P - 1) ? p.nc : min(c_begin + p.L, p.nc));
    const int L = c_end - c_begin;
    const int npre = (seg < p.P - 1) ? L : 0;  // the last segment needs no aggregate
    const int n_items = npre + L;
    const size_t slot = (size_t)bhf * p.P + seg;
    constexpr uint32_t kFmt = BF16 ? 1u : 0u;

    if ((unsigned)ticket >= (unsigned)(p.BH * p.P)) {
        // A ticket past the last segment means the workspace header was not
        // zero at launch (two calls sharing it overlapped, or it was never
        // zeroed): this CTA does no work and reports it; the counters and
        // flags are still reset below, so the next call starts clean.
        if (tid == 0) latch_error(p.err, kDevErrWorkspace);
    } else if (warp == kWarpLoad) {
        // ------------------------------------------------------------ producer
        // TMA tile loads of whole chunks: one box per tensor for row scans,
        // FC / boxh column slabs per tensor for column scans.
        const uint64_t pol_keep = l2_policy_evict_last();  // pre-pass data is read again
        const uint64_t pol_once = l2_policy_evict_first();
        bool ok = true;
        uint32_t issued = 0;  // bit s: the last use of stage s had its copies issued
        const CUtensorMap *vmap = vpart ? &p.tm_v2 : &p.tm_v;
        for (int it = 0; it < n_items; ++it) {
            const int s = it % kStages;
            const bool pre = it < npre;
            const int c = pre ? (c_end - 1 - it) : (c_begin + it - npre);
            if (it >= kStages) {
                bool w = true;
                if (lane == 0) w = pwait(&bar_empty[s], ((it / kStages) - 1) & 1, &s_abort, p.err, 64);
                ok = __shfl_sync(0xffffffffu, w, 0) && ok;
            }
            issued = ok ? (issued | (1u << s)) : (issued & ~(1u << s));
            // row table (for the output stores): global row of every token
            int *rows = sRows + s * 64;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int u = lane + 32 * e;
                const int rr = scan_to_raster(min(c * FC + u, p.n - 1), p.n, p.gh, p.gw, p.dir);
                rows[u] = index_ok(rr >= 0 && rr < p.n && c >= 0 && c < p.nc, p.err) ? bh * p.n + rr : 0;
            }
            if (lane == 0) sLen[s] = min(FC, p.n - c * FC);
#ifdef GTR_CHECKED
            {  // every box / gather of this chunk inside the tensor maps
                const int p0 = (p.dir & 1) ? (p.n - FC - c * FC) : c * FC;
                bool cok = bh < p.BHt && vpart < p.nvh;
                if (p.dir < 2) {
                    cok = cok && p0 > -FC && p0 < p.n;
                } else if (p.boxh == 0) {
                    if (lane < 16)
                        for (int e = 0; e < 4; ++e) {
                            const int u = (p.dir & 1) ? 63 - (4 * lane + e) : 4 * lane + e;
                            const int rr = scan_to_raster(min(c * FC + u, p.n - 1), p.n, p.gh, p.gw, p.dir);
                            cok = cok && rr >= 0 && rr < p.n;
                        }
                } else {
                    for (int bx = lane; bx < FC / p.boxh; bx += 32) {
                        const int pp = p0 + bx * p.boxh;
                        const int x = pp >= 0 ? pp / p.gh : -1, y = pp >= 0 ? pp % p.gh : 0;
                        cok = cok && pp < p.n && x >= -1 && x < p.gw && y >= 0 && y + p.boxh <= p.gh;
                    }
                }
                cok = __all_sync(0xffffffffu, cok);
                if (lane == 0) index_ok(cok, p.err);
                ok = ok && cok;  // a chunk with a bad coordinate loads nothing
                issued = ok ? issued : (issued & ~(1u << s));
            }
#endif
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(&bar_full[s], ok ? (pre ? 32768u : 40960u) : 0u);
            __syncwarp();
            // The chunk's tokens, in stage-row order: row scans load raster rows
            // [y0, y0+64) of the plane, column scans the column-major positions
            // [p0, p0+64); reversed scans take the same range read backwards
            // (token u sits in stage row 63 - u).  Rows outside the grid read
            // as zero.
            if (ok) {
                uint8_t *st = sm + s * ST_BYTES;
                const uint64_t pol = pre ? pol_keep : pol_once;
                const int p0 = (p.dir & 1) ? (p.n - FC - c * FC) : c * FC;
                if (p.dir < 2) {
                    if (lane == 0) {
                        tma_load_3d_pol(st + ST_K, &p.tm_k, &bar_full[s], 0, p0, bh, pol);
                        tma_load_3d_pol(st + ST_V, vmap, &bar_full[s], 0, p0, bh, pol);
                        tma_load_3d_pol(st + ST_LA, &p.tm_la, &bar_full[s], 0, p0, bh, pol);
                        if (!pre) tma_load_3d_pol(st + ST_Q, &p.tm_q, &bar_full[s], 0, p0, bh, pol_once);
                    }
                } else if (p.boxh == 0) {
                    if (lane < 16) {  // stage rows 4 lane .. 4 lane + 3, as row gathers
                        int r[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int u = (p.dir & 1) ? 63 - (4 * lane + e) : 4 * lane + e;
                            r[e] = bh * p.n + scan_to_raster(min(c * FC + u, p.n - 1), p.n, p.gh, p.gw, p.dir);
                        }
                        const int m = 4 * lane;
                        tma_gather4_pol(st + ST_K + m * 128, &p.tm_k, &bar_full[s], 0, r[0], r[1], r[2], r[3], pol);
                        tma_gather4_pol(st + ST_V + m * 128, vmap, &bar_full[s], 0, r[0], r[1], r[2], r[3], pol);
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
                        tma_load_4d_pol(st + ST_V + r * 128, vmap, &bar_full[s], 0, x, y, bh, pol);
                        tma_load_4d_pol(st + ST_LA + r * 256, &p.tm_la, &bar_full[s], 0, x, y, bh, pol);
                        if (!pre)
                            tma_load_4d_pol(st + ST_Q + r * 128, &p.tm_q, &bar_full[s], 0, x, y, bh, pol_once);
                    }
                }
            }
        }
        // no copy may still be landing when the CTA exits (after an abort the
        // consumers may not have waited for them): bounded wait on the last
        // issued phase of every stage
        if (lane == 0) {
            for (int it = (n_items > kStages ? n_items - kStages : 0); it < n_items; ++it) {
                const int s = it % kStages;
                if (issued & (1u << s)) mbar_wait(&bar_full[s], (it / kStages) & 1, 200000000ull);
            }
        }
        __syncwarp();
    } else if (warp == kWarpMma) {
        // ---------------------------------------------------------- MMA issue
        if (lane == 0) {
            const uint32_t id_tf = idesc(2, 64, 128, 0, 0);    // tf32, both K-major, N = 128
            const uint32_t id_tf64 = idesc(2, 64, 64, 0, 0);   // the same, N = 64
            const uint32_t id_av = idesc(kFmt, 64, 64, 0, 1);  // A K-major, V as B (MN-major)
            const uint32_t id_vk = idesc(kFmt, 64, 64, 1, 0);  // V^T as A (MN-major), K^ as B
            // descriptors of stage 0 / buffer 0; stage s adds s * ST_BYTES (the
            // start field holds address >> 4, far from overflowing)
            const uint32_t sbase = smem_u32(sm);
            const uint64_t d_qh = sdesc_sw128(sbase + ST_QH, 16, 1024);
            const uint64_t d_b1 = sdesc_sw128(sbase + ST_B1, 16, 1024);
            const uint64_t d_v = sdesc_sw128(sbase + ST_V, 8192, 1024);
            const uint64_t d_kh = sdesc_sw128(sbase + ST_KH, 16, 1024);
            const uint64_t d_a = sdesc_sw128(sbase + OFF_A, 16, 1024);
            auto st_desc = [](uint64_t d, int s) { return d + (uint64_t)(s * (ST_BYTES >> 4)); };
            for (int it = 0; it < npre; ++it) {  // pre-pass: A_seg^T += V^T K^
                const int s = it % kStages;
                pwait(&bar_op[s], (it / kStages) & 1, &s_abort, p.err);
                tc_fence_after_sync();
                fence_proxy_async_smem();
                const uint64_t dv = st_desc(d_v, s), dk = st_desc(d_kh, s);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(tbase + TM_PRE, desc_add(dv, ks * 2048), desc_add(dk, ks * 32), id_vk,
                            (it > 0 || ks > 0) ? 1u : 0u);
                mma_commit(&bar_empty[s]);
            }
            if (npre > 0) mma_commit(&bar_pre);
            // o(k) += A_k V_k, then release chunk k's stage
            auto issue_av = [&](int k) {
                const int s = (npre + k) % kStages;
                pwait(&bar_a[k & 1], (k >> 1) & 1, &s_abort, p.err);
                tc_fence_after_sync();
                fence_proxy_async_smem();
                const uint64_t dv = st_desc(d_v, s), da = d_a + (uint64_t)((k & 1) * (8192 >> 4));
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(tbase + TM_R + 128 * (k % 3) + 64, desc_add(da, ks * 32), desc_add(dv, ks * 2048),
                            id_av, 1u);
                mma_commit(&bar_o[k & 1]);
                mma_commit(&bar_empty[s]);
            };
            for (int k = 0; k < L; ++k) {
                const int it = npre + k, s = it % kStages;
                // the previous chunk's A V first: it releases that chunk's stage
                // as soon as its mask is done
                if (k > 0) issue_av(k - 1);
                // dS^T(k) = V^T K^ as soon as the operands are ready (the
                // epilogue's state recursion only needs these)
                pwait(&bar_op[s], (it / kStages) & 1, &s_abort, p.err);
                tc_fence_after_sync();
                fence_proxy_async_smem();
                {
                    const uint64_t dv = st_desc(d_v, s), dk = st_desc(d_kh, s);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_f16(tbase + TM_DS + 64 * (k & 1), desc_add(dv, ks * 2048), desc_add(dk, ks * 32),
                                id_vk, ks > 0 ? 1u : 0u);
                    mma_commit(&bar_ds[k & 1]);
                }
                // [scores | o] = Q^ [K~ ; S_k^T]^T once state k is in the stage
                pwait(&bar_s[k & 1], (k >> 1) & 1, &s_abort, p.err);
                tc_fence_after_sync();
                fence_proxy_async_smem();
                {
                    const uint64_t dq = st_desc(d_qh, s), db = st_desc(d_b1, s);
                    if (!sFlag[s]) {
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks)
                            mma_tf32(tbase + TM_R + 128 * (k % 3), desc_add(dq, (ks >> 2) * 8192 + (ks & 3) * 32),
                                     desc_add(db, (ks >> 2) * 16384 + (ks & 3) * 32), id_tf, ks > 0 ? 1u : 0u);
                    } else {  // exact scores are already in TMEM: only o = Q^ S (B rows 64-127)
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks)
                            mma_tf32(tbase + TM_R + 128 * (k % 3) + 64,
                                     desc_add(dq, (ks >> 2) * 8192 + (ks & 3) * 32),
                                     desc_add(db, (ks >> 2) * 16384 + 8192 + (ks & 3) * 32), id_tf64,
                                     ks > 0 ? 1u : 0u);
                    }
                    mma_commit(&bar_sc[k & 1]);
                }
            }
            if (L > 0) issue_av(L - 1);
            mma_commit(&bar_fin);
            pwait(&bar_fin, 0, &s_abort, p.err);
        }
        __syncwarp();
    } else if (warp < kWarpEpi0) {
        // ------------------------------------------------------ operand warps
        constexpr int RW = FC / kOpWarps;  // tokens per thread
        const int ow = warp - kWarpOp0;    // tokens RW ow .. RW ow + RW - 1
        const int p2 = 2 * lane;           // key dims p2, p2 + 1
        const bool rev = p.dir & 1;        // token u sits in stage row 63 - u
        const bool opl = (warp == kWarpOp0 && lane == 0);  // the group's polling thread
        const int row0 = rev ? 63 - RW * ow : RW * ow;    // stage row of token RW ow
        const int rstep = rev ? -1 : 1;                    // stage-row step per token
        // K^ (the K index of V^T K^ follows V's stage rows): this thread's RW
        // tokens fill the 16-byte chunk kc0 of rows p2, p2 + 1
        const int kc0 = rev ? 7 - ow : ow;
        auto store_kh = [&](uint8_t *kh, float *kh0, float *kh1) {
            if (rev) {  // stage-row order is reversed token order
#pragma unroll
                for (int j = 0; j < RW / 2; ++j) {
                    const float t0 = kh0[j], t1 = kh1[j];
                    kh0[j] = kh0[RW - 1 - j];
                    kh0[RW - 1 - j] = t0;
                    kh1[j] = kh1[RW - 1 - j];
                    kh1[RW - 1 - j] = t1;
                }
            }
            *reinterpret_cast<uint4 *>(kh + sw128(p2, kc0)) = pack8<T>(kh0);
            *reinterpret_cast<uint4 *>(kh + sw128(p2 + 1, kc0)) = pack8<T>(kh1);
        };
        float2 gafter = make_float2(0.f, 0.f);
        for (int it = 0; it < n_items; ++it) {
            const int s = it % kStages;
            const bool pre = it < npre;
            const int k = it - npre;
            gwait(opl, kBarOp, kOpThreads, &bar_full[s], (it / kStages) & 1, &s_abort, p.err);
            uint8_t *st = sm + s * ST_BYTES;
            const int len = sLen[s];
            // 1. this thread's gates, q and k (everything is read before the
            //    in-place overwrites below).  Loads are unconditional (every
            //    stage row is valid memory) and tokens past the end are zeroed
            //    afterwards: no branch between the loads, all in flight at once.
            float2 a[RW];
            uint32_t qw[RW], kw[RW];
            float2 l = make_float2(0.f, 0.f);
            const int nin = len - RW * ow;  // this thread's tokens kk < nin are real
            {
                const float *lr = reinterpret_cast<const float *>(st + ST_LA) + row0 * 64 + p2;
                const uint8_t *kr = st + ST_K + row0 * 128 + p2 * 2;
                const uint8_t *qr = st + ST_Q + row0 * 128 + p2 * 2;
                float2 x[RW];
#pragma unroll
                for (int kk = 0; kk < RW; ++kk) {
                    x[kk] = ld2(lr + kk * rstep * 64);
                    kw[kk] = *reinterpret_cast<const uint32_t *>(kr + kk * rstep * 128);
                    qw[kk] = *reinterpret_cast<const uint32_t *>(qr + kk * rstep * 128);
                }
#pragma unroll
                for (int kk = 0; kk < RW; ++kk) {
                    const bool in = kk < nin;
                    x[kk] = in ? x[kk] : make_float2(0.f, 0.f);
                    kw[kk] = in ? kw[kk] : 0u;
                    qw[kk] = in ? qw[kk] : 0u;
                    l.x += x[kk].x;
                    l.y += x[kk].y;
                    a[kk] = ex2_2(x[kk]);
                }
            }
            float *tot = sTot + (it & 1) * (kOpWarps * 64);
            st2(tot + ow * 64 + p2, l);
            named_bar_sync(kBarOp, kOpThreads);
            // 2. where this thread's rows sit in the chunk
            float2 before = make_float2(0.f, 0.f), g = make_float2(0.f, 0.f);
#pragma unroll
            for (int o = 0; o < kOpWarps; ++o) {
                const float2 t = ld2(tot + o * 64 + p2);
                if (o < ow) {
                    before.x += t.x;
                    before.y += t.y;
                }
                g.x += t.x;
                g.y += t.y;
            }
            const float2 after = make_float2(g.x - before.x - l.x, g.y - before.y - l.y);
            if (pre) {
                // K^ relative to the segment end: k . e^{G_after + (gates after u in the chunk)}
                float2 f = ex2_2(make_float2(gafter.x + after.x, gafter.y + after.y));
                float kh0[RW], kh1[RW];
#pragma unroll
                for (int kk = RW - 1; kk >= 0; --kk) {
                    const float2 h = fmul2(Pack2<T>::unpack(kw[kk]), f);
                    kh0[kk] = h.x;
                    kh1[kk] = h.y;
                    f = fmul2(f, a[kk]);
                }
                store_kh(st + ST_KH, kh0, kh1);
                gafter.x += g.x;
                gafter.y += g.y;
                if (it == npre - 1) {  // the segment's gate totals
                    // no fence of its own: the arrive (release, CTA scope) orders
                    // the store before the epilogue's release of the flag
                    if (ow == 0) st2(p.aggg + slot * 64 + p2, gafter);
                    mbar_arrive(&bar_owpre);
                }
            } else {
                const bool unsafe = __any_sync(0xffffffffu, (-g.x > kSpanLimit) || (-g.y > kSpanLimit));
                if (unsafe) {
                    // exact scores: b (log2 domain) in place of log_alpha, then
                    // A[t,s] = sum_i q_ti k_si 2^{b_ti - b_si} for s <= t
                    float2 cb = before;
                    float *lat = reinterpret_cast<float *>(st + ST_LA);
#pragma unroll
                    for (int kk = 0; kk < RW; ++kk) {
                        const int u = RW * ow + kk, pr = rev ? 63 - u : u;
                        const float2 x = (u < len) ? ld2(lat + pr * 64 + p2) : make_float2(0.f, 0.f);
                        cb.x += x.x;
                        cb.y += x.y;
                        st2(lat + pr * 64 + p2, make_float2(cb.x * kLog2e, cb.y * kLog2e));
                    }
                    named_bar_sync(kBarOp, kOpThreads);
                    // TMEM region k % 3 is free: its last chunk (k - 3) was masked
                    // before this stage could be refilled; only region 2 during the
                    // pre-pass's publication needs a wait
                    if (k == 2 && npre > 0) gwait(opl, kBarOp, kOpThreads, &bar_pub, 0, &s_abort, p.err);
                    // this warp's part of the M = 64 score tile: its lane quadrant,
                    // one half of the columns
                    const int qd = warp & 3, hc = (ow >> 2) * 32;
                    const int r0 = 16 * qd + (lane >> 2), cq = 2 * (lane & 3);
                    uint32_t sc[16];
#pragma unroll 1
                    for (int e = 0; e < 16; ++e) {
                        const int t = r0 + 8 * ((e >> 1) & 1), sx = hc + 8 * (e >> 2) + cq + (e & 1);
                        float acc = 0.f;
                        if (sx <= t && t < len) {
                            const int pt = rev ? 63 - t : t, ps = rev ? 63 - sx : sx;
                            const T *qr = reinterpret_cast<const T *>(st + ST_Q + pt * 128);
                            const T *kr = reinterpret_cast<const T *>(st + ST_K + ps * 128);
                            for (int i = 0; i < FD; ++i)
                                acc = fmaf(to_f32(qr[i]) * to_f32(kr[i]),
                                           fast_exp2(lat[pt * 64 + i] - lat[ps * 64 + i]), acc);
                        }
                        sc[e] = __float_as_uint(acc);
                    }
                    tmem_st16x256_x4(tbase + TM_R + 128 * (k % 3) + hc + ((uint32_t)(32 * qd) << 16), sc);
                    tmem_st_wait();
                    named_bar_sync(kBarOp, kOpThreads);  // b is no longer read: Q^ may overwrite it
                }
                // Q^ = q . e^{b_u} (running product of the alphas up to u)
                float2 e = ex2_2(before);
                uint8_t *qh = st + ST_QH;
#pragma unroll
                for (int kk = 0; kk < RW; ++kk) {
                    const int u = RW * ow + kk;
                    e = fmul2(e, a[kk]);
                    const float2 v = fmul2(Pack2<T>::unpack(qw[kk]), e);
                    *reinterpret_cast<uint2 *>(qh + tf32_kmaj(u, p2)) = make_uint2(tf32_rn(v.x), tf32_rn(v.y));
                }
                // K^ = k . e^{g - b_u} (product of the alphas after u), K~ = K^ . e^{-g}
                float2 f = ex2_2(after);
                const float2 m = unsafe ? make_float2(0.f, 0.f) : ex2_2(make_float2(-g.x, -g.y));
                uint8_t *kt = st + ST_B1;
                float kh0[RW], kh1[RW];
#pragma unroll
                for (int kk = RW - 1; kk >= 0; --kk) {
                    const int u = RW * ow + kk;
                    const float2 h = fmul2(Pack2<T>::unpack(kw[kk]), f);
                    kh0[kk] = h.x;
                    kh1[kk] = h.y;
                    const float2 t2 = fmul2(h, m);
                    *reinterpret_cast<uint2 *>(kt + b1_off(u, p2)) = make_uint2(tf32_rn(t2.x), tf32_rn(t2.y));
                    f = fmul2(f, a[kk]);
                }
                store_kh(st + ST_KH, kh0, kh1);
                if (ow == 0) {
                    st2(sGam + s * 64 + p2, ex2_2(g));
                    if (lane == 0) sFlag[s] = unsafe ? 1 : 0;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            mbar_arrive(&bar_op[s]);
        }
    } else {
        // ----------------------------------------------------- epilogue warps
        // Two warps per TMEM lane quadrant, one per half of the columns; a
        // thread holds rows r0, r0 + 8 and columns hc + 8 c + cq + {0, 1}
        // (c = 0..3) of every M = 64 result: element x <-> row r0 + 8 ((x >> 1) & 1),
        // column hc + 8 (x >> 2) + cq + (x & 1).
        const int qd = warp & 3;
        const int hc = ((warp - kWarpEpi0) >> 2) * 32;
        const uint32_t lo = ((uint32_t)(32 * qd) << 16) + hc;
        const int r0 = 16 * qd + (lane >> 2);
        const int cq = 2 * (lane & 3);
        const bool rev = p.dir & 1;
        const bool epl = (warp == kWarpEpi0 && lane == 0);  // the group's polling thread
        bool ok = true;
        float S[16];  // S^T[j][i] of this thread's elements
#pragma unroll
        for (int x = 0; x < 16; ++x) S[x] = 0.f;

        if (npre > 0) {  // publish the aggregate A_seg^T and raise this segment's flag
            ok = gwait(epl, kBarEpi, kEpiThreads, &bar_pre, 0, &s_abort, p.err, 256) && ok;
            tc_fence_after_sync();
            uint32_t r[16];
            tmem_ld16x256_x4(tbase + TM_PRE + lo, r);
            tmem_ld_wait();
            tc_fence_before_sync();
            mbar_arrive(&bar_pub);  // TMEM region 2 is free for the main pass
            float *dst = p.agg + slot * 4096;
            const bool pub_ok = index_ok(slot < (size_t)p.BH * p.P, p.err);
#pragma unroll
            for (int x = 0; x < 16 && pub_ok; x += 2) {
                const int j = r0 + 8 * ((x >> 1) & 1), i = hc + 8 * (x >> 2) + cq;
                st2(dst + j * 64 + i, make_float2(__uint_as_float(r[x]), __uint_as_float(r[x + 1])));
            }
            ok = gwait(epl, kBarEpi, kEpiThreads, &bar_owpre, 0, &s_abort, p.err) && ok;
            // One release store publishes everything: the stores above (and the
            // operand warps' gate totals, seen through bar_owpre) precede it
            // through the CTA barrier, and release is cumulative, so no
            // per-thread fence is needed.
            named_bar_sync(kBarEpi, kEpiThreads);
            if (epl && ok && pub_ok) st_release(p.flag + kWsFlagStride * slot, 1);
        }
        if (p.coop) {
            // Transposed boundary scan: every CTA of the plane is resident, so
            // each one takes a slice of the 64x64 state elements (pairs u0 ..
            // u1 - 1) through every segment boundary,
            //     S_in(s+1) = diag(e^{g_s}) S_in(s) + A_s,   S_in(0) = 0
            // (g_s: segment s's gate totals, A_s its aggregate), writes that
            // slice of every S_in and raises flag2; then it reads its own S_in,
            // whose slices all CTAs of the plane wrote.  Each aggregate is read
            // once per plane instead of once per later segment.
            const int et = tid - 32 * kWarpEpi0;
            if (warp == kWarpEpi0) {
                bool got = true;
                for (int j = lane; j < p.P - 1; j += 32)
                    got = wait_flag(p.flag + kWsFlagStride * ((size_t)bhf * p.P + j)) && got;
                if (!__all_sync(0xffffffffu, got) && lane == 0) {
                    s_abort = 1;
                    latch_error(p.err, kDevErrTimeout);
                }
            }
            named_bar_sync(kBarEpi, kEpiThreads);
            if (s_abort) ok = false;
            // stage this CTA's slice of every aggregate (A buffers, unused until
            // the first mask) and the plane's gate totals, every load in
            // flight at once, then scan the slice's pairs through the segments
            const float2 *agp = reinterpret_cast<const float2 *>(p.agg + (size_t)bhf * p.P * 4096);
            float2 *sinp = reinterpret_cast<float2 *>(p.sin + (size_t)bhf * p.P * 4096);
            float2 *sA = reinterpret_cast<float2 *>(sm + OFF_A);
            float *sG = reinterpret_cast<float *>(sm + OFF_SCAN);
            const int u0 = seg * 2048 / p.P, u1 = (seg + 1) * 2048 / p.P;
            const int m = u1 - u0, nA = (p.P - 1) * m;
            if (ok && !index_ok(bhf < p.BH && seg < p.P && p.P <= kMaxScanSegments && u1 <= 2048, p.err)) ok = false;
            if (ok) {
                float gt[8];  // (P - 1) * 64 <= 8 * kEpiThreads gate totals
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int e = et + j * kEpiThreads;
                    if (e < (p.P - 1) * 64) gt[j] = __ldcg(p.aggg + (size_t)bhf * p.P * 64 + e);
                }
                for (int e0 = et; e0 < nA; e0 += 8 * kEpiThreads) {  // one pass: nA <= 8 * kEpiThreads
                    float2 t[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int e = e0 + j * kEpiThreads, s2 = e / m;
                        if (e < nA) t[j] = __ldcg(agp + (size_t)s2 * 2048 + u0 + (e - s2 * m));
                    }
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (e0 + j * kEpiThreads < nA) sA[e0 + j * kEpiThreads] = t[j];
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int e = et + j * kEpiThreads;
                    if (e < (p.P - 1) * 64) sG[e] = gt[j];
                }
            }
            named_bar_sync(kBarEpi, kEpiThreads);
            if (ok) {
                for (int uu = et; uu < m; uu += kEpiThreads) {
                    const int u = u0 + uu, i = (2 * u) & 63;  // key dim of the pair's first element
                    float2 R = make_float2(0.f, 0.f);
                    for (int s2 = 0; s2 < p.P - 1; ++s2) {
                        R = ffma2(ex2_2(ld2(sG + s2 * 64 + i)), R, sA[s2 * m + uu]);
                        __stcg(sinp + (size_t)(s2 + 1) * 2048 + u, R);
                    }
                }
            }
            named_bar_sync(kBarEpi, kEpiThreads);
            if (epl && ok) st_release(p.flag2 + kWsFlagStride * slot, 1);
            if (seg > 0) {
                if (warp == kWarpEpi0) {
                    bool got = true;
                    for (int j = lane; j < p.P; j += 32)
                        got = wait_flag(p.flag2 + kWsFlagStride * ((size_t)bhf * p.P + j)) && got;
                    if (!__all_sync(0xffffffffu, got) && lane == 0) {
                        s_abort = 1;
                        latch_error(p.err, kDevErrTimeout);
                    }
                }
                named_bar_sync(kBarEpi, kEpiThreads);
                if (s_abort) ok = false;
                if (ok && index_ok(slot < (size_t)p.BH * p.P, p.err)) {
                    const float *sn = p.sin + slot * 4096;
#pragma unroll
                    for (int x = 0; x < 16; x += 2) {
                        const int j = r0 + 8 * ((x >> 1) & 1), i = hc + 8 * (x >> 2) + cq;
                        const float2 t = __ldcg(reinterpret_cast<const float2 *>(sn + j * 64 + i));
                        S[x] = t.x;
                        S[x + 1] = t.y;
                    }
                }
            }
        } else if (seg > 0) {  // fold the earlier segments' aggregates, nearest first
            if (warp == kWarpEpi0) {
                bool got = true;
                for (int j = lane; j < seg; j += 32) got = wait_flag(p.flag + kWsFlagStride * ((size_t)bhf * p.P + j)) && got;
                if (!__all_sync(0xffffffffu, got) && lane == 0) {
                    s_abort = 1;
                    latch_error(p.err, kDevErrTimeout);
                }
            }
            named_bar_sync(kBarEpi, kEpiThreads);
            if (s_abort) ok = false;
            // The earlier segments' gate totals, copied once (coalesced) into
            // the A buffers, which stay unused until the first mask.
            float *sGt = reinterpret_cast<float *>(sm + OFF_A);
            if (ok && !index_ok(bhf < p.BH && seg < p.P && seg <= kMaxSegments, p.err)) ok = false;
            if (ok)
                for (int e = tid - 32 * kWarpEpi0; e < seg * 64; e += kEpiThreads)
                    sGt[e] = __ldcg(p.aggg + (size_t)bhf * p.P * 64 + e);
            named_bar_sync(kBarEpi, kEpiThreads);
            float2 acc[4];  // log-gate sums of the segments between the source and this one
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[c] = make_float2(0.f, 0.f);
            // software-pipelined: the next kFoldDepth - 1 aggregates' loads are
            // in flight while one is folded (same summation order as a plain loop)
            float2 vb[kFoldDepth][8];
            auto load = [&](int d, float2 *vv) {
                const float *ag = p.agg + ((size_t)bhf * p.P + (seg - 1 - d)) * 4096;
#pragma unroll
                for (int x = 0; x < 16; x += 2) {
                    const int j = r0 + 8 * ((x >> 1) & 1), i = hc + 8 * (x >> 2) + cq;
                    vv[x >> 1] = __ldcg(reinterpret_cast<const float2 *>(ag + j * 64 + i));
                }
            };
#pragma unroll
            for (int e = 0; e < kFoldDepth; ++e)
                if (ok && e < seg) load(e, vb[e]);
            for (int d0 = 0; d0 < seg && ok; d0 += kFoldDepth) {
#pragma unroll
                for (int e = 0; e < kFoldDepth; ++e) {
                    const int d = d0 + e;
                    if (d < seg) {
                        const float *gt = sGt + (seg - 1 - d) * 64 + hc + cq;
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const float2 sc = ex2_2(acc[c]);
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const int x = 4 * c + 2 * h;
                                const float2 t = ffma2(sc, vb[e][x >> 1], make_float2(S[x], S[x + 1]));
                                S[x] = t.x;
                                S[x + 1] = t.y;
                            }
                            const float2 g2 = ld2(gt + 8 * c);
                            acc[c].x += g2.x;
                            acc[c].y += g2.y;
                        }
                        if (d + kFoldDepth < seg) load(d + kFoldDepth, vb[e]);
                    }
                }
            }
        }
        // state k^T (tf32) -> rows 64-127 of the B tile of the stage holding chunk k
        auto store_state = [&](int stage) {
            uint8_t *sb = sm + stage * ST_BYTES + ST_B1;
#pragma unroll
            for (int x = 0; x < 16; x += 2) {
                const int j = r0 + 8 * ((x >> 1) & 1), i = hc + 8 * (x >> 2) + cq;
                *reinterpret_cast<uint2 *>(sb + b1_off(64 + j, i)) = make_uint2(tf32_rn(S[x]), tf32_rn(S[x + 1]));
            }
            fence_proxy_async_smem();
        };
        if (L > 0) store_state(npre % kStages);  // state 0: the incoming state
        tc_fence_before_sync();
        mbar_arrive(&bar_s[0]);

        // Output tail: this thread's 8 norm weights (columns hc + 8 c + cq, +1),
        // and where its head sits in the merged [B, n, H, 64] layout.
        float wnv[8];
        const int t_head = TAIL ? bh % p.H : 0;
        const size_t t_img = TAIL ? (size_t)(bh / p.H) : 0;
        if constexpr (TAIL) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float2 w2 = __ldg(reinterpret_cast<const float2 *>(p.wn + t_head * 64 + hc + 8 * c + cq));
                wnv[2 * c] = w2.x;
                wnv[2 * c + 1] = w2.y;
            }
        }
        float *sTail = reinterpret_cast<float *>(sm + OFF_MISC + MISC_TAIL);

        // output of chunk kp (its o is complete once bar_o says so)
        int prow[2] = {0, 0}, plen = 0;
        auto emit = [&](int kp) {
            // tail: the gate z at this thread's elements (rows r0, r0 + 8;
            // columns hc + 8 c + cq, +1), loaded before the wait
            uint32_t zr[2][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
            size_t yoff[2] = {0, 0};
            if constexpr (TAIL) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const size_t raster = (size_t)(prow[h] - bh * p.n);
                    yoff[h] = ((t_img * p.n + raster) * p.H + t_head) * 64 + hc + cq;
                    if (r0 + 8 * h < plen && index_ok(yoff[h] + 26 <= (size_t)p.BHt * p.n * 64, p.err)) {
                        const uint32_t *zp = reinterpret_cast<const uint32_t *>(reinterpret_cast<const T *>(p.z) +
                                                                                yoff[h]);
#pragma unroll
                        for (int c = 0; c < 4; ++c) zr[h][c] = __ldcs(zp + 4 * c);
                    }
                }
            }
            ok = gwait(epl, kBarEpi, kEpiThreads, &bar_o[kp & 1], (kp >> 1) & 1, &s_abort, p.err) && ok;
            tc_fence_after_sync();
            uint32_t r[16];
            tmem_ld16x256_x4(tbase + TM_R + 128 * (kp % 3) + 64 + lo, r);
            tmem_ld_wait();
            if constexpr (TAIL) {
                // the row's sum of squares: this quad's 32 columns (shuffles),
                // then the other half from the partner warp through shared memory
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float ss = 0.f;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float a = __uint_as_float(r[4 * c + 2 * h]), b = __uint_as_float(r[4 * c + 2 * h + 1]);
                        ss = fmaf(a, a, fmaf(b, b, ss));
                    }
                    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
                    if ((lane & 3) == 0) sTail[(kp & 1) * 128 + (hc >> 5) * 64 + r0 + 8 * h] = ss;
                }
                named_bar_sync(kBarEpi, kEpiThreads);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int row = r0 + 8 * h;
                    const float ss = sTail[(kp & 1) * 128 + row] + sTail[(kp & 1) * 128 + 64 + row];
                    const float rs = rsqrtf(fmaf(ss, 1.f / 64.f, p.eps));
                    if (ok && row < plen && index_ok(yoff[h] + 26 <= (size_t)p.BHt * p.n * 64, p.err)) {
                        uint32_t *yp = reinterpret_cast<uint32_t *>(reinterpret_cast<T *>(p.y) + yoff[h]);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const float2 zf = Pack2<T>::unpack(zr[h][c]);
                            yp[4 * c] = Pack2<T>::pack(
                                __uint_as_float(r[4 * c + 2 * h]) * rs * wnv[2 * c] * silu_f32(zf.x),
                                __uint_as_float(r[4 * c + 2 * h + 1]) * rs * wnv[2 * c + 1] * silu_f32(zf.y));
                        }
                    }
                }
            } else if (ok) {
                // 4-byte stores of each thread's column pairs: a warp's store
                // covers 16 bytes of 8 rows, four of them a row's 64 bytes.
                // (16-byte stores need a transpose inside each quad first;
                // on the epilogue's per-chunk critical path that measured
                // slower than the extra store instructions.)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (r0 + 8 * h < plen && index_ok(prow[h] >= 0 && prow[h] < p.BHt * p.n, p.err)) {
                        uint32_t *dst = reinterpret_cast<uint32_t *>(reinterpret_cast<T *>(p.out) +
                                                                     (size_t)prow[h] * p.ldo + 64 * vpart + hc + cq);
                        if (p.acc_out) {  // second key half: add to the first half's output
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const float2 o = Pack2<T>::unpack(dst[4 * c]);
                                dst[4 * c] = Pack2<T>::pack(o.x + __uint_as_float(r[4 * c + 2 * h]),
                                                            o.y + __uint_as_float(r[4 * c + 2 * h + 1]));
                            }
                        } else {
#pragma unroll
                            for (int c = 0; c < 4; ++c)
                                dst[4 * c] = Pack2<T>::pack(__uint_as_float(r[4 * c + 2 * h]),
                                                            __uint_as_float(r[4 * c + 2 * h + 1]));
                        }
                    }
                }
            }
        };

        uint8_t *const sAbuf = sm + OFF_A;
        for (int k = 0; k < L; ++k) {
            const int it = npre + k, s = it % kStages, b = k & 1;
            // the operand warps' release of this stage makes its row table,
            // length and gate factors visible here
            ok = gwait(epl, kBarEpi, kEpiThreads, &bar_op[s], (it / kStages) & 1, &s_abort, p.err) && ok;
            // stage-local values, read before the stage can be recycled
            const int *rows = sRows + s * 64;
            const int len = sLen[s];
            const int row0 = rows[r0], row1 = rows[r0 + 8];
            float2 gam[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) gam[c] = ld2(sGam + s * 64 + hc + 8 * c + cq);
            // 1. state update S_{k+1} = diag(e^{g}) S_k + dS_k  (S^T: scale column i),
            //    written into the next chunk's stage (its previous chunk's
            //    product, which read that spot, completed before bar_sc of
            //    chunk k-2 was seen)
            ok = gwait(epl, kBarEpi, kEpiThreads, &bar_ds[b], (k >> 1) & 1, &s_abort, p.err) && ok;
            tc_fence_after_sync();
            {
                uint32_t r[16];
                tmem_ld16x256_x4(tbase + TM_DS + 64 * b + lo, r);
                tmem_ld_wait();
#pragma unroll
                for (int x = 0; x < 16; x += 2) {
                    const float2 t = ffma2(gam[x >> 2], make_float2(S[x], S[x + 1]),
                                           make_float2(__uint_as_float(r[x]), __uint_as_float(r[x + 1])));
                    S[x] = t.x;
                    S[x + 1] = t.y;
                }
            }
            if (k + 1 < L) store_state((it + 1) % kStages);
            tc_fence_before_sync();
            mbar_arrive(&bar_s[(k + 1) & 1]);
            // 2. causal mask of the scores -> A[b] (rows t, K = s)
            ok = gwait(epl, kBarEpi, kEpiThreads, &bar_sc[b], (k >> 1) & 1, &s_abort, p.err) && ok;
            tc_fence_after_sync();
            {
                uint32_t r[16];
                tmem_ld16x256_x4(tbase + TM_R + 128 * (k % 3) + lo, r);
                tmem_ld_wait();
                uint8_t *sa = sAbuf + 8192 * b;
                // columns follow V's stage rows: token s at column s, or 63 - s
                // for reversed scans (16-byte chunk 7 ^ c, element 6 ^ cq, the
                // pair swapped)
                const int cx = rev ? 7 : 0, ex = rev ? 6 : 0;
#pragma unroll
                for (int x = 0; x < 16; x += 2) {
                    const int t = r0 + 8 * ((x >> 1) & 1), c = (hc >> 3) + (x >> 2), sx = 8 * c + cq;
                    const float v0 = (sx <= t) ? __uint_as_float(r[x]) : 0.f;
                    const float v1 = (sx + 1 <= t) ? __uint_as_float(r[x + 1]) : 0.f;
                    *reinterpret_cast<uint32_t *>(sa + sw128(t, c ^ cx) + (cq ^ ex) * 2) =
                        rev ? Pack2<T>::pack(v1, v0) : Pack2<T>::pack(v0, v1);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            mbar_arrive(&bar_a[b]);
            // 3. output of the previous chunk
            if (k > 0) emit(k - 1);
            prow[0] = row0;
            prow[1] = row1;
            plen = len;
        }
        if (L > 0) emit(L - 1);
        if (seg == p.P - 1 && p.final_state && ok && index_ok(bhf < p.BH, p.err)) {
            float *fs = p.final_state + (size_t)bh * p.fs_bh + 64 * vpart;
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                const int j = r0 + 8 * ((x >> 1) & 1), i = hc + 8 * (x >> 2) + cq + (x & 1);
                fs[(size_t)i * p.fs_ld + j] = S[x];
            }
        }
    }

    // ------------------------------------------------------------- teardown
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == kWarpMma) tmem_dealloc(tbase, kTmemCols);
    // coop: more arrivals than CTAs means the header was not zero at launch
    if (tid == 0 && p.coop && arrival >= (unsigned)(p.BH * p.P)) latch_error(p.err, kDevErrWorkspace);
    if (tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&p.ctr[1], 1u);
        s_last = (prev == gridDim.x - 1) ? 1 : 0;
    }
    __syncthreads();
    if (s_last) {  // last CTA to finish: leave the workspace ready for the next call
        if (p.P > 1)
            for (int idx = tid; idx < p.BH * p.P; idx += kThreads) {
                p.flag[kWsFlagStride * idx] = 0;
                if (p.coop) p.flag2[kWsFlagStride * idx] = 0;
            }
        if (tid == 0) {
            p.ctr[0] = 0;
            p.ctr[1] = 0;
        }
        __threadfence();
    }
}

constexpr int kSMs = 148;

struct Plan {
    int nc, P, L, coop, rem_first;
};

// Segments per (b,h).  More segments put more SMs to work and shorten each
// CTA's serial chain of chunks, but every segment except the last adds a
// pre-pass over its chunks.  When all segments fit on the SMs at once
// (coop) the boundary states come from the transposed scan, whose cost does
// not grow with the number of segments, and the last segment may be longer
// than the others (it runs no pre-pass); otherwise every segment folds all
// earlier aggregates itself and CTAs beyond one per SM run in further waves.
// The choice minimises a time model built from this kernel's measured costs
// on B200 (microseconds): a main-pass chunk, a pre-pass chunk, one folded
// aggregate, the transposed scan, and the fixed cost of publishing and
// waiting for flags.
// Planes of one launch: every (b, h), twice when d_v = 128 (both value halves
// of a key half in one launch).
int launch_planes(const Problem &pr) { return pr.B * pr.H * (pr.dv / FD); }

Plan make_plan(const Problem &pr) {
    // kFlag: publishing and the flag round of the fold; the cooperative plans
    // split it into the aggregates' round (kFlag1) and the scan's (kFlag2)
    constexpr double kMain = 2.2, kPre = 1.2, kFold = 0.5, kFlag = 3.0, kScan = 3.0, kFlag1 = 2.0, kFlag2 = 1.8;
    const int nc = (pr.n + FC - 1) / FC;
    const int bh = launch_planes(pr);
    Plan best{nc, 1, nc, 0, 0};
    double tbest = nc * kMain * (double)((bh + kSMs - 1) / kSMs);
    const int pmax = nc < kMaxSegments ? nc : kMaxSegments;
    for (int P = 2; P <= pmax; ++P) {
        if ((long long)bh * P > kWsMaxFlags) break;
        if ((long long)bh * P <= kSMs && bh * P <= kWsMaxFlags / 2 && P <= kMaxScanSegments) {
            // one wave: the cost falls with L while the last segment is the
            // longest and rises after, so floor and ceil of nc / P bracket it
            for (int L = nc / P; L <= (nc + P - 1) / P; ++L) {
                const int rem = nc - (P - 1) * L;
                if (L < 1 || rem < 1) continue;
                const int lmax = rem > L ? rem : L;
                // the rest in the last segment, or in the first (whose main
                // pass needs no incoming state, but whose pre-pass everyone waits for)
                const double t_last = L * kPre + kFlag1 + kScan + kFlag2 + lmax * kMain;
                const double t_first =
                    lmax * kPre + kFlag1 + kScan + std::max(rem * kMain, kFlag2 + L * kMain);
                if (t_last < tbest) {
                    tbest = t_last;
                    best = Plan{nc, P, L, 1, 0};
                }
                // (row scans only: the column scans' pre-pass, on strided row
                // slabs, is slower, and measured no gain)
                if (pr.dir < 2 && t_first < tbest) {
                    tbest = t_first;
                    best = Plan{nc, P, L, 1, 1};
                }
            }
        }
        const int L = (nc + P - 1) / P;
        if ((nc + L - 1) / L != P) continue;
        const long long waves = ((long long)bh * P + kSMs - 1) / kSMs;
        const double t = waves * L * (kMain + kPre) + (P - 1) * kFold + kFlag;
        if (t < tbest) {
            tbest = t;
            best = Plan{nc, P, L, 0, 0};
        }
    }
    return best;
}

struct WsLayout {
    size_t agg, aggg, sin, flag, flag2, ctr, total;
};

// ctr and both flag arrays live in the shared workspace header (flag2 in its
// second half); the segment states after it.
WsLayout ws_layout(const Problem &pr, const Plan &pl) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t slots = pl.P > 1 ? (size_t)launch_planes(pr) * pl.P : 0;
    WsLayout w;
    w.ctr = 0;
    w.flag = 256;
    w.flag2 = 256 + (size_t)(kWsMaxFlags / 2) * kWsFlagStride * 4;
    w.agg = kWsHeaderBytes;
    w.aggg = up(w.agg + slots * 4096 * 4);
    w.sin = up(w.aggg + slots * 64 * 4);
    w.total = up(w.sin + (pl.coop ? slots * 4096 * 4 : 0));
    return w;
}

// CTAs of this kernel that the current device holds at once (cached per
// kernel and device; 0 if the query fails).
int coresident(const void *func) {
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, int> done;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_pair(func, dev);
    auto it = done.find(key);
    if (it != done.end()) return it->second;
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, func, kThreads, SMEM_BYTES) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    done[key] = per_sm * sms;
    return per_sm * sms;
}

}  // namespace

bool fused_supported(const Problem &pr) {
    if (pr.dtype != GTR_GLA_F16 && pr.dtype != GTR_GLA_BF16) return false;
    if ((pr.dk != 64 && pr.dk != 128) || (pr.dv != 64 && pr.dv != 128) || pr.chunk != 64) return false;
    if ((long long)pr.B * pr.H * pr.n >= (1LL << 31)) return false;
    return true;
}

// The plan may differ between row and column scans; the workspace size covers
// both, so a size queried without the direction fits every call.
size_t fused_workspace_bytes(const Problem &pr) {
    Problem rows = pr, cols = pr;
    rows.dir = 0;
    cols.dir = 2;
    return std::max(ws_layout(rows, make_plan(rows)).total, ws_layout(cols, make_plan(cols)).total);
}

// One launch for key half kh and every value half (its planes are (value
// half, b, h)).
static int launch_fused_part(const Problem &pr, const Plan &pl, const WsLayout &wl, void *ws,
                             int kh, cudaStream_t st) {
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
    const int nvh = pr.dv / FD;
    if (enc(&p.tm_q, pr.q, pr.dk, FD * kh, dt16, 2, false) || enc(&p.tm_k, pr.k, pr.dk, FD * kh, dt16, 2, false) ||
        enc(&p.tm_v, pr.v, pr.dv, 0, dt16, 2, true) ||
        enc(&p.tm_v2, pr.v, pr.dv, FD * (nvh - 1), dt16, 2, true) ||
        enc(&p.tm_la, pr.la, pr.dk, FD * kh, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, false))
        return GTR_GLA_ERR_CUDA;
    p.boxh = boxh;
    p.q = pr.q;
    p.k = pr.k;
    p.v = pr.v;
    p.la = pr.la;
    p.out = pr.out;  // the kernel adds 64 columns per value half
    p.ldo = pr.dv;
    p.acc_out = kh > 0;
    p.final_state = pr.final_state ? pr.final_state + (size_t)FD * kh * pr.dv : nullptr;
    p.fs_bh = pr.dk * pr.dv;
    p.fs_ld = pr.dv;
    p.agg = reinterpret_cast<float *>(w + wl.agg);
    p.aggg = reinterpret_cast<float *>(w + wl.aggg);
    p.flag = reinterpret_cast<int *>(w + wl.flag);
    p.flag2 = reinterpret_cast<int *>(w + wl.flag2);
    p.sin = reinterpret_cast<float *>(w + wl.sin);
    p.ctr = reinterpret_cast<unsigned *>(w + wl.ctr);
    p.err = pr.err;
    p.n = pr.n;
    p.gh = pr.gh;
    p.gw = pr.gw;
    p.dir = pr.dir;
    p.nc = pl.nc;
    p.P = pl.P;
    p.L = pl.L;
    p.BHt = pr.B * pr.H;
    p.nvh = nvh;
    p.BH = p.BHt * nvh;
    const dim3 grid(p.BH * p.P);
    p.z = pr.z;
    p.wn = pr.wn;
    p.y = pr.y;
    p.eps = pr.eps;
    p.H = pr.H;
    const bool bf = pr.dtype == GTR_GLA_BF16, tail = pr.tail != 0;
    auto kern = bf ? (tail ? gla_fused_kernel<true, true> : gla_fused_kernel<true, false>)
                   : (tail ? gla_fused_kernel<false, true> : gla_fused_kernel<false, false>);
    const void *func = (const void *)kern;
    if (ensure_smem(func, SMEM_BYTES)) return GTR_GLA_ERR_CUDA;
    // The transposed scan needs every CTA resident at once: a cooperative
    // launch guarantees it.  If this device holds fewer CTAs (a partitioned
    // GPU), the same plan runs with per-segment folds instead.
    p.coop = (pl.coop && coresident(func) >= (int)grid.x) ? 1 : 0;
    p.rem_first = pl.rem_first;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.coop ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return GTR_GLA_ERR_CUDA;
    note_launch();
    return cudaPeekAtLastError() == cudaSuccess ? GTR_GLA_OK : GTR_GLA_ERR_CUDA;
}

// Head sizes of 128 run as 64-wide sub-problems: one launch per key half, in
// stream order, each covering both value halves when d_v = 128 (its planes
// are (value half, b, h)): key half 0 writes the output, key half 1 adds to
// it.  The launches share the workspace; each leaves its header zeroed for
// the next.
int launch_fused(const Problem &pr, void *ws, cudaStream_t st) {
    const Plan pl = make_plan(pr);
    const WsLayout wl = ws_layout(pr, pl);
    for (int kh = 0; kh < pr.dk / FD; ++kh) {
        const int rc = launch_fused_part(pr, pl, wl, ws, kh, st);
        if (rc != GTR_GLA_OK) return rc;
    }
    return GTR_GLA_OK;
}

}  // namespace gtr
