// tc_gemm.cu -- the dense projections of the backbone layer and of the
// Spatial SwiGLU block on this library's own sm_100a tensor-core GEMM:
//     out[M, N] = in[M, K] . W[N, K]^T (+ bias[N]) (+ resid[M, N])
// fp16 / bf16 operands and output, fp32 accumulation in tensor memory, bias
// and residual added in fp32, one rounding (see include/gtr_gemm.h).
//
// Persistent CTAs (at most one per SM) walk output tiles of 128 rows x BN
// columns (BN = 256, 192, 128 or 64: the fewest waves of tiles, weighted by
// the operand bytes and MMA work of a tile).  Per
// tile, K runs in blocks of 64 through a 4-stage shared-memory ring filled by
// TMA (both operands K-major with the 128-byte swizzle) and drained by
// tcgen05.mma M128 x BN x K16 into one of two TMEM accumulators.  Four
// epilogue warps (one per TMEM lane quadrant, one output row per thread) read
// the other accumulator, so a tile's epilogue overlaps the next tile's MMAs.
//   warp 0     TMA producer (one lane)
//   warp 1     TMEM allocation and MMA issue (one lane)
//   warps 2-5  epilogue
// Every wait is bounded: a wait that gives up latches a timeout in the
// library's error word and the CTA runs to its end without further work.
#include "../../include/gtr_gemm.h"
#include "gla_common.cuh"
#include "gla_internal.h"
#include "io_pack.cuh"
#include "sm100.cuh"

#include <cstring>
#include <map>
#include <mutex>
#include <type_traits>

namespace gtr {
using namespace sm100;

namespace {

constexpr int GM = 128, GK = 64, kGStages = 4;
constexpr int kGThreads = 192;
constexpr uint32_t kGABytes = GM * GK * 2;  // A tile: 128 rows x 128 B

constexpr uint32_t kOutChunk = 32 * 64;  // one warp's 32 rows x 32 columns of output, 2 B each

template <int BN> struct GemmCfg {
    static constexpr uint32_t kStage = kGABytes + BN * GK * 2;
    static constexpr uint32_t kOffOut = kGStages * kStage;  // 4 warps x 2 output staging buffers
    static constexpr uint32_t kSmem = kOffOut + 8 * kOutChunk + 1024;  // + alignment slack
    // two accumulators (at columns 0 and BN), allocated as a power of two
    static constexpr uint32_t kTmemCols = 2 * BN <= 128 ? 128 : 2 * BN <= 256 ? 256 : 512;
};
static_assert(GemmCfg<256>::kSmem <= 232448, "shared memory");

struct GemmParams {
    CUtensorMap tm_a, tm_b;  // in [M][K], W [N][K]: boxes of 64 K x 128 / BN rows
    CUtensorMap tm_c;        // out [M][N]: boxes of 32 x 32, 64-byte swizzle
    const void *bias, *resid;
    void *out;
    int *err;
    int M, N, K, num_m, tiles;
};

// Bounded wait (about 2 s): try_wait, then short sleeps.  After the first wait
// of the CTA that gives up, every later wait returns false at once.
__device__ bool gwait(uint64_t *bar, uint32_t parity, volatile int *abort, int *err) {
    if (mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t n = 0;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 15) == 15) {
            if (*abort) return false;
            const uint64_t dt = global_timer_ns() - t0;
            if (dt > 2000000000ull) {
                *abort = 1;
                latch_error(err, kDevErrTimeout);
                return false;
            }
            if (dt > 2000) __nanosleep(64);
        }
    }
}

template <typename T, int BN>
__global__ void __launch_bounds__(kGThreads, 1) tc_gemm_kernel(const __grid_constant__ GemmParams p) {
    using Cfg = GemmCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ uint64_t full[kGStages], empty[kGStages], acc_full[2], acc_empty[2];
    __shared__ uint32_t s_tmem;
    __shared__ volatile int s_abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 128);
        }
        fence_mbar_init();
        s_abort = 0;
    }
    if (warp == 1) {
        tmem_alloc(&s_tmem, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tbase = s_tmem;
    const int nk = (p.K + GK - 1) / GK;

    if (warp == 0) {
        if (lane == 0) {  // ------------------------------------------ producer
            int g = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < p.tiles && ok; t += gridDim.x) {
                const int nt = t / p.num_m, mt = t - nt * p.num_m;
                for (int kb = 0; kb < nk; ++kb, ++g) {
                    const int s = g % kGStages;
                    if (g >= kGStages && !gwait(&empty[s], ((g / kGStages) - 1) & 1, &s_abort, p.err)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = sm + s * Cfg::kStage;
                    mbar_arrive_expect_tx(&full[s], Cfg::kStage);
                    tma_load_2d(st, &p.tm_a, &full[s], kb * GK, mt * GM);
                    tma_load_2d(st + kGABytes, &p.tm_b, &full[s], kb * GK, nt * BN);
                }
            }
            // no copy may still be landing when the CTA exits: bounded wait on
            // the last phase of every stage that was issued
            for (int q = (g > kGStages ? g - kGStages : 0); q < g; ++q)
                mbar_wait(&full[q % kGStages], (q / kGStages) & 1, 200000000ull);
        }
    } else if (warp == 1) {
        if (lane == 0) {  // ---------------------------------------- MMA issue
            const uint32_t id = idesc(std::is_same<T, __nv_bfloat16>::value ? 1u : 0u, GM, BN, 0, 0);
            const uint32_t base = smem_u32(sm);
            const uint64_t da = sdesc_sw128(base, 16, 1024), db = sdesc_sw128(base + kGABytes, 16, 1024);
            int g = 0, lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < p.tiles && ok; t += gridDim.x, ++lt) {
                const int buf = lt & 1;
                if (lt >= 2 && !gwait(&acc_empty[buf], ((lt >> 1) - 1) & 1, &s_abort, p.err)) break;
                tc_fence_after_sync();
                for (int kb = 0; kb < nk; ++kb, ++g) {
                    const int s = g % kGStages;
                    if (!gwait(&full[s], (g / kGStages) & 1, &s_abort, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint64_t off = (uint64_t)((s * Cfg::kStage) >> 4);
#pragma unroll
                    for (int ks = 0; ks < GK / 16; ++ks)  // a K step of 16 is 32 B inside the row
                        mma_f16(tbase + buf * BN, da + off + 2 * ks, db + off + 2 * ks, id, (kb | ks) ? 1u : 0u);
                    mma_commit(&empty[s]);
                }
                if (ok) mma_commit(&acc_full[buf]);
            }
        }
    } else {  // ------------------------------------------------------- epilogue
        // Each 32-column chunk of the warp's 32 rows goes to a shared-memory
        // buffer (row = lane, 64 B per row, 16-byte pieces at piece ^ ((row / 2) % 4):
        // the tensor map's 64-byte swizzle, conflict-free for these stores) and
        // from there to global memory as one TMA store; two buffers per warp,
        // so a chunk is written while the previous one is stored.
        const int q = warp & 3;  // the TMEM lane quadrant this warp may read
        const int r = 32 * q + lane;
        uint8_t *obuf = sm + Cfg::kOffOut + (warp - 2) * 2 * kOutChunk;
        int nst = 0, lt = 0;
        for (int t = blockIdx.x; t < p.tiles; t += gridDim.x, ++lt) {
            const int nt = t / p.num_m, mt = t - nt * p.num_m, buf = lt & 1;
            if (!gwait(&acc_full[buf], (lt >> 1) & 1, &s_abort, p.err)) break;
            tc_fence_after_sync();
            const int row = mt * GM + r;
            const bool row_ok = row < p.M && index_ok(row >= 0, p.err);
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                const int col0 = nt * BN + 32 * c;
                if (col0 >= p.N) break;  // (warp-uniform)
                uint32_t v[32];
                tmem_ld32x32b_x32(tbase + buf * BN + 32 * c + ((uint32_t)(32 * q) << 16), v);
                tmem_ld_wait();
                float f[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(v[e]);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int col = col0 + 8 * j;
                    if (col < p.N && p.bias) {
                        float2 b2[4];
                        unpack8<T>(*reinterpret_cast<const uint4 *>(static_cast<const T *>(p.bias) + col), b2);
#pragma unroll
                        for (int e = 0; e < 4; ++e) f[8 * j + 2 * e] += b2[e].x, f[8 * j + 2 * e + 1] += b2[e].y;
                    }
                    if (col < p.N && row_ok && p.resid) {
                        float2 x2[4];
                        unpack8<T>(*reinterpret_cast<const uint4 *>(static_cast<const T *>(p.resid) +
                                                                     (size_t)row * p.N + col),
                                   x2);
#pragma unroll
                        for (int e = 0; e < 4; ++e) f[8 * j + 2 * e] += x2[e].x, f[8 * j + 2 * e + 1] += x2[e].y;
                    }
                }
                // the buffer's previous store (two stores ago) must have read it
                if (lane == 0 && nst >= 2) tma_store_wait_read<1>();
                __syncwarp();
                uint8_t *ob = obuf + (nst & 1) * kOutChunk;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    *reinterpret_cast<uint4 *>(ob + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
                        make_uint4(Pair<T>::pack(f[8 * j], f[8 * j + 1]), Pair<T>::pack(f[8 * j + 2], f[8 * j + 3]),
                                   Pair<T>::pack(f[8 * j + 4], f[8 * j + 5]),
                                   Pair<T>::pack(f[8 * j + 6], f[8 * j + 7]));
                fence_proxy_async_smem();
                __syncwarp();
                // rows past M and columns past N are clipped by the store
                if (lane == 0) {
                    tma_store_2d(&p.tm_c, ob, col0, mt * GM + 32 * q);
                    tma_store_commit();
                }
                ++nst;
            }
            tc_fence_before_sync();
            mbar_arrive(&acc_empty[buf]);
        }
        if (lane == 0) tma_store_wait_all();  // the stores read shared memory: finish before exit
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 1) tmem_dealloc(tbase, Cfg::kTmemCols);
}

int sm_count_cached() {
    static std::mutex mu;
    static std::map<int, int> cache;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(dev);
    if (it != cache.end()) return it->second;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
    return n;
}

template <typename T, int BN>
int launch(GemmParams &p, const void *in, const void *w, int sms, cudaStream_t st) {
    const CUtensorMapDataType dt =
        std::is_same<T, __nv_bfloat16>::value ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const uint64_t da[2] = {(uint64_t)p.K, (uint64_t)p.M}, db[2] = {(uint64_t)p.K, (uint64_t)p.N};
    const uint64_t stride[1] = {(uint64_t)p.K * 2};
    const uint32_t ba[2] = {GK, GM}, bb[2] = {GK, BN};
    const uint64_t dc[2] = {(uint64_t)p.N, (uint64_t)p.M}, sc[1] = {(uint64_t)p.N * 2};
    const uint32_t bc[2] = {32, 32};
    if (encode_tile_map(&p.tm_a, in, dt, 2, da, stride, ba, true) ||
        encode_tile_map(&p.tm_b, w, dt, 2, db, stride, bb, true) ||
        encode_tile_map_sw(&p.tm_c, p.out, dt, 2, dc, sc, bc, 64))
        return GTR_GLA_ERR_CUDA;
    const int num_n = (p.N + BN - 1) / BN;
    p.tiles = p.num_m * num_n;
    auto kern = tc_gemm_kernel<T, BN>;
    if (ensure_smem((const void *)kern, GemmCfg<BN>::kSmem)) return GTR_GLA_ERR_CUDA;
    const int grid = p.tiles < sms ? p.tiles : sms;
    kern<<<grid, kGThreads, GemmCfg<BN>::kSmem, st>>>(p);
    note_launch();
    return cudaPeekAtLastError() == cudaSuccess ? GTR_GLA_OK : GTR_GLA_ERR_CUDA;
}

}  // namespace

int dense_gemm(int dtype, long long M, int N, int K, const void *in, const void *w, const void *bias,
               const void *resid, void *out, cudaStream_t st) {
    if (M <= 0 || N <= 0 || K <= 0 || M > (1LL << 31) - 128 || N % 8 || K % 8) return GTR_GLA_ERR_SHAPE;
    if (dtype != GTR_GLA_F16 && dtype != GTR_GLA_BF16) return GTR_GLA_ERR_DTYPE;
    const int sms = sm_count_cached();
    if (sms <= 0) return GTR_GLA_ERR_CUDA;
    GemmParams p;
    memset(&p, 0, sizeof(p));
    p.bias = bias;
    p.resid = resid;
    p.out = out;
    p.M = (int)M;
    p.N = N;
    p.K = K;
    p.num_m = (int)((M + GM - 1) / GM);
    int rc = error_word(&p.err);
    if (rc) return rc;
    // tile width (256, 192, 128 or 64 columns): the fewest waves of tiles,
    // each weighted by the operand rows it reads (128 + BN), its MMA work (BN)
    // and a fixed cost (measured on B200: this picks 128 for 1600 x 3072 x 384,
    // 64 for 1600 x 384 x 1536, 256 for 12800 x 6144 x 768, 192 for
    // 12800 x 768 x 3072)
    auto cost = [&](long long bn) {
        const long long tiles = (long long)p.num_m * ((N + bn - 1) / bn);
        return ((tiles + sms - 1) / sms) * (GM + 2 * bn + 64);
    };
    int bn = 256;
    for (int c : {192, 128, 64})
        if (cost(c) < cost(bn)) bn = c;
    if (dtype == GTR_GLA_BF16) {
        switch (bn) {
            case 256: return launch<__nv_bfloat16, 256>(p, in, w, sms, st);
            case 192: return launch<__nv_bfloat16, 192>(p, in, w, sms, st);
            case 128: return launch<__nv_bfloat16, 128>(p, in, w, sms, st);
            default: return launch<__nv_bfloat16, 64>(p, in, w, sms, st);
        }
    }
    switch (bn) {
        case 256: return launch<__half, 256>(p, in, w, sms, st);
        case 192: return launch<__half, 192>(p, in, w, sms, st);
        case 128: return launch<__half, 128>(p, in, w, sms, st);
        default: return launch<__half, 64>(p, in, w, sms, st);
    }
}

}  // namespace gtr

using namespace gtr;

extern "C" int gtr_gemm_fwd(const void *in, const void *w, const void *bias, const void *resid, void *out,
                            long long M, int N, int K, int dtype, cudaStream_t stream) {
    if (!in || !w || !out) return GTR_GLA_ERR_NULL;
    if (M <= 0 || N <= 0 || K <= 0 || M > (1LL << 31) - 128 || N % 8 || K % 8) return GTR_GLA_ERR_SHAPE;
    if (dtype != GTR_GLA_F16 && dtype != GTR_GLA_BF16) return GTR_GLA_ERR_DTYPE;
    const void *ptrs[] = {in, w, bias, resid, out};
    for (const void *q : ptrs)
        if (((uintptr_t)q & 15u) != 0) return GTR_GLA_ERR_ALIGN;
    const size_t no = (size_t)M * N * 2;
    auto overlaps = [](const void *a, size_t na, const void *b, size_t nb) {
        const char *pa = (const char *)a, *pb = (const char *)b;
        return b && pa < pb + nb && pb < pa + na;
    };
    if (overlaps(out, no, in, (size_t)M * K * 2) || overlaps(out, no, w, (size_t)N * K * 2) ||
        overlaps(out, no, bias, (size_t)N * 2) || (resid && resid != out && overlaps(out, no, resid, no)))
        return GTR_GLA_ERR_ALIAS;
    return dense_gemm(dtype, M, N, K, in, w, bias, resid, out, stream);
}
