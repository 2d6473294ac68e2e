// gtr_gla_api.cu -- the C ABI of libgtr_gla.so: argument validation,
// workspace management and dispatch to the kernels.  See include/gtr_gla.h for
// the contract of every entry point.
#include <atomic>
#include <map>
#include <mutex>

#include "../../include/gtr_output_tail.h"
#include "gla_common.cuh"
#include "gla_internal.h"

namespace gtr {

static std::atomic<unsigned long long> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int ensure_smem(const void *func, size_t bytes) {
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, size_t> done;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return GTR_GLA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_pair(func, dev);
    auto it = done.find(key);
    if (it != done.end() && it->second >= bytes) return GTR_GLA_OK;
    if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
        cudaSuccess)
        return GTR_GLA_ERR_CUDA;
    done[key] = bytes;
    return GTR_GLA_OK;
}

// Device-side error word (one per device): kernels latch the first error here.
__device__ int g_dev_err;

constexpr int kMaxDevices = 64;
static std::mutex g_mu;
static int *g_err_ptr[kMaxDevices];
static void *g_ws[kMaxDevices];
static size_t g_ws_bytes[kMaxDevices];

static int current_device(int *dev) {
    if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= kMaxDevices)
        return GTR_GLA_ERR_CUDA;
    return GTR_GLA_OK;
}

// Address of this device's error word (looked up once per device).
static int device_err_ptr(int dev, int **out) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_err_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_dev_err) != cudaSuccess) return GTR_GLA_ERR_CUDA;
        g_err_ptr[dev] = (int *)p;
    }
    *out = g_err_ptr[dev];
    return GTR_GLA_OK;
}

static size_t elem_size(int dtype) { return dtype == GTR_GLA_F32 ? 4 : 2; }

static bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    const char *pa = (const char *)a, *pb = (const char *)b;
    return pa < pb + nb && pb < pa + na;
}

static bool misaligned(const void *p) { return ((uintptr_t)p & 15u) != 0; }

static bool head_dims_ok(int dk, int dv) {
    return (dk == 64 || dk == 128) && (dv == 64 || dv == 128);
}

// Chunk lengths: 32 and 64 for every case; 128 with d_k = 64 (the CUDA-core
// path keeps a chunk's q, k and gates in shared memory, which a 128 x 128
// chunk would overflow).
static bool chunk_ok(int chunk, int dk) {
    return chunk == 32 || chunk == 64 || (chunk == 128 && dk == 64);
}

static int validate_shape(int B, int H, int gh, int gw, int dk, int dv, int dtype, int chunk) {
    if (B <= 0 || H <= 0 || gh <= 0 || gw <= 0) return GTR_GLA_ERR_SHAPE;
    if ((long long)B * H > 65535 || (long long)gh * gw > (1LL << 22)) return GTR_GLA_ERR_SHAPE;
    // token rows of all planes are 32-bit (row tables, TMA coordinates)
    if ((long long)B * H * gh * gw >= (1LL << 31)) return GTR_GLA_ERR_SHAPE;
    if (dtype != GTR_GLA_F16 && dtype != GTR_GLA_BF16 && dtype != GTR_GLA_F32)
        return GTR_GLA_ERR_DTYPE;
    if (!head_dims_ok(dk, dv)) return GTR_GLA_ERR_HEAD_DIM;
    if (!chunk_ok(chunk, dk)) return GTR_GLA_ERR_CHUNK;
    return GTR_GLA_OK;
}

static int validate(const Problem &p) {
    if (!p.q || !p.k || !p.v || !p.la || !p.out) return GTR_GLA_ERR_NULL;
    int rc = validate_shape(p.B, p.H, p.gh, p.gw, p.dk, p.dv, p.dtype, p.chunk);
    if (rc) return rc;
    if (p.dir < 0 || p.dir > 3) return GTR_GLA_ERR_DIRECTION;
    if (misaligned(p.q) || misaligned(p.k) || misaligned(p.v) || misaligned(p.la) ||
        misaligned(p.out) || (p.final_state && misaligned(p.final_state)))
        return GTR_GLA_ERR_ALIGN;
    const size_t es = elem_size(p.dtype);
    const size_t tok = (size_t)p.B * p.H * p.n;
    const size_t nq = tok * p.dk * es, nv = tok * p.dv * es, nla = tok * p.dk * 4;
    const size_t nfs = (size_t)p.B * p.H * p.dk * p.dv * 4;
    if (overlaps(p.out, nv, p.q, nq) || overlaps(p.out, nv, p.k, nq) ||
        overlaps(p.out, nv, p.v, nv) || overlaps(p.out, nv, p.la, nla))
        return GTR_GLA_ERR_ALIAS;
    if (p.final_state &&
        (overlaps(p.final_state, nfs, p.out, nv) || overlaps(p.final_state, nfs, p.q, nq) ||
         overlaps(p.final_state, nfs, p.k, nq) || overlaps(p.final_state, nfs, p.v, nv) ||
         overlaps(p.final_state, nfs, p.la, nla)))
        return GTR_GLA_ERR_ALIAS;
    return GTR_GLA_OK;
}

// The workspace is written by the kernels, so its first `n` bytes may overlap
// no tensor argument of the call (inputs, out or y, final_state).
static bool workspace_touches(const Problem &p, const void *ws, size_t n) {
    if (!ws || n == 0) return false;
    const size_t es = elem_size(p.dtype);
    const size_t tok = (size_t)p.B * p.H * p.n;
    const size_t nq = tok * p.dk * es, nv = tok * p.dv * es, nla = tok * p.dk * 4;
    const size_t nfs = (size_t)p.B * p.H * p.dk * p.dv * 4;
    return overlaps(ws, n, p.q, nq) || overlaps(ws, n, p.k, nq) || overlaps(ws, n, p.v, nv) ||
           overlaps(ws, n, p.la, nla) || overlaps(ws, n, p.out, nv) ||
           (p.final_state && overlaps(ws, n, p.final_state, nfs));
}

// fp16/bf16 with chunk 64 run the fused tensor-core kernel (head sizes of 128
// as one launch per 64-wide key half); everything else (fp32 I/O, other chunk
// lengths) the three-phase CUDA-core path.
static size_t workspace_bytes(const Problem &p) {
    return fused_supported(p) ? fused_workspace_bytes(p) : generic_workspace_bytes(p);
}

static int dispatch(const Problem &p, void *ws, cudaStream_t st) {
    return fused_supported(p) ? launch_fused(p, ws, st) : launch_generic(p, ws, st);
}

static Problem make_problem(const void *q, const void *k, const void *v, const float *la,
                            void *out, float *fs, int B, int H, int gh, int gw, int dk,
                            int dv, int dir, int dtype, int chunk) {
    Problem p;
    p.q = q; p.k = k; p.v = v; p.la = la; p.out = out; p.final_state = fs;
    p.B = B; p.H = H; p.gh = gh; p.gw = gw;
    p.n = (gh > 0 && gw > 0 && (long long)gh * gw <= (1LL << 22)) ? gh * gw : 0;
    p.dk = dk; p.dv = dv; p.dir = dir; p.dtype = dtype; p.chunk = chunk;
    p.err = nullptr;
    return p;
}

int check_problem(const Problem &p) { return validate(p); }

int error_word(int **out) {
    int dev;
    int rc = current_device(&dev);
    if (rc) return rc;
    return device_err_ptr(dev, out);
}

}  // namespace gtr

using namespace gtr;

extern "C" {

int gtr_gla_fwd_ex(const void *q, const void *k, const void *v, const float *log_alpha,
                   void *out, float *final_state, int B, int H, int grid_h, int grid_w,
                   int d_k, int d_v, int direction, int dtype, int chunk, void *workspace,
                   size_t workspace_bytes_, cudaStream_t stream) {
    Problem p = make_problem(q, k, v, log_alpha, out, final_state, B, H, grid_h, grid_w,
                             d_k, d_v, direction, dtype, chunk);
    int rc = validate(p);
    if (rc) return rc;
    const size_t need = workspace_bytes(p);
    if (need > 0 && (!workspace || workspace_bytes_ < need || ((uintptr_t)workspace & 255u)))
        return GTR_GLA_ERR_WORKSPACE;
    if (need > 0 && workspace_touches(p, workspace, need)) return GTR_GLA_ERR_ALIAS;
    int dev;
    if ((rc = current_device(&dev))) return rc;
    if ((rc = device_err_ptr(dev, &p.err))) return rc;
    return dispatch(p, workspace, stream);
}

int gtr_gla_fwd(const void *q, const void *k, const void *v, const float *log_alpha,
                void *out, float *final_state, int B, int H, int grid_h, int grid_w, int d_k,
                int d_v, int direction, cudaStream_t stream) {
    Problem p = make_problem(q, k, v, log_alpha, out, final_state, B, H, grid_h, grid_w,
                             d_k, d_v, direction, GTR_GLA_F16, 64);
    int rc = validate(p);
    if (rc) return rc;
    int dev;
    if ((rc = current_device(&dev))) return rc;
    if ((rc = device_err_ptr(dev, &p.err))) return rc;
    const size_t need = workspace_bytes(p);
    void *ws = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (need > g_ws_bytes[dev]) {
            // Growing: wait for work that may still use the old buffer, then
            // replace it.  The new buffer starts zero-filled.
            if (g_ws[dev]) {
                if (cudaDeviceSynchronize() != cudaSuccess) return GTR_GLA_ERR_CUDA;
                cudaFree(g_ws[dev]);
                g_ws[dev] = nullptr;
                g_ws_bytes[dev] = 0;
            }
            void *nw = nullptr;
            if (cudaMalloc(&nw, need) != cudaSuccess) return GTR_GLA_ERR_CUDA;
            if (cudaMemset(nw, 0, need) != cudaSuccess) {
                cudaFree(nw);
                return GTR_GLA_ERR_CUDA;
            }
            g_ws[dev] = nw;
            g_ws_bytes[dev] = need;
        }
        ws = g_ws[dev];
    }
    return dispatch(p, ws, stream);
}

// Output tail fused into the stores (d_k = d_v = 64), or for head sizes of 128
// the attention into a workspace buffer followed by the tail kernel.
static size_t tail_layout(const Problem &p, size_t *obuf) {
    const size_t gla = workspace_bytes(p);
    if (p.dk == 64 && p.dv == 64) {
        *obuf = 0;
        return gla;
    }
    *obuf = (gla + 255) & ~(size_t)255;
    return *obuf + (size_t)p.B * p.H * p.n * p.dv * 2;
}

size_t gtr_gla_tail_workspace_size(int B, int H, int grid_h, int grid_w, int d_k, int d_v, int dtype) {
    if (dtype != GTR_GLA_F16 && dtype != GTR_GLA_BF16) return 0;
    if (validate_shape(B, H, grid_h, grid_w, d_k, d_v, dtype, 64)) return 0;
    Problem p = make_problem(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, B, H, grid_h, grid_w,
                             d_k, d_v, 0, dtype, 64);
    size_t obuf;
    return tail_layout(p, &obuf);
}

int gtr_gla_fwd_tail(const void *q, const void *k, const void *v, const float *log_alpha, const void *z,
                     const float *w_n, float eps, void *y, float *final_state, int B, int H, int grid_h,
                     int grid_w, int d_k, int d_v, int direction, int dtype, void *workspace,
                     size_t workspace_bytes_, cudaStream_t stream) {
    if (dtype != GTR_GLA_F16 && dtype != GTR_GLA_BF16) return GTR_GLA_ERR_DTYPE;
    // y takes the place of `out` in the checks: the same bytes, the same aliasing rules
    Problem p = make_problem(q, k, v, log_alpha, y, final_state, B, H, grid_h, grid_w, d_k, d_v,
                             direction, dtype, 64);
    if (!z || !w_n) return GTR_GLA_ERR_NULL;
    int rc = validate(p);
    if (rc) return rc;
    if (!(eps >= 0.f) || eps > 3.0e38f) return GTR_GLA_ERR_SHAPE;
    if (misaligned(z) || misaligned(w_n)) return GTR_GLA_ERR_ALIGN;
    const size_t ny = (size_t)p.B * p.H * p.n * p.dv * 2;
    if (overlaps(y, ny, z, ny) || overlaps(y, ny, w_n, (size_t)p.H * p.dv * 4) ||
        (final_state && overlaps(final_state, (size_t)p.B * p.H * p.dk * p.dv * 4, z, ny)))
        return GTR_GLA_ERR_ALIAS;
    size_t obuf;
    const size_t need = tail_layout(p, &obuf);
    if (!workspace || workspace_bytes_ < need || ((uintptr_t)workspace & 255u)) return GTR_GLA_ERR_WORKSPACE;
    if (workspace_touches(p, workspace, need) || overlaps(z, ny, workspace, need) ||
        overlaps(w_n, (size_t)p.H * p.dv * 4, workspace, need))
        return GTR_GLA_ERR_ALIAS;
    int dev;
    if ((rc = current_device(&dev))) return rc;
    if ((rc = device_err_ptr(dev, &p.err))) return rc;
    if (p.dk == 64 && p.dv == 64) {
        p.tail = 1;
        p.z = z;
        p.wn = w_n;
        p.y = y;
        p.eps = eps;
        return launch_fused(p, workspace, stream);
    }
    void *o = static_cast<char *>(workspace) + obuf;
    p.out = o;
    if ((rc = dispatch(p, workspace, stream))) return rc;
    return gtr_output_tail_fwd(o, z, w_n, y, B, H, grid_h, grid_w, d_v, eps, dtype, stream);
}

size_t gtr_gla_workspace_size(int B, int H, int grid_h, int grid_w, int d_k, int d_v,
                              int dtype, int chunk) {
    if (validate_shape(B, H, grid_h, grid_w, d_k, d_v, dtype, chunk)) return 0;
    Problem p = make_problem(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, B, H,
                             grid_h, grid_w, d_k, d_v, 0, dtype, chunk);
    return workspace_bytes(p);
}

int gtr_gla_status(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return GTR_GLA_ERR_CUDA;
    int dev;
    if (current_device(&dev)) return GTR_GLA_ERR_CUDA;
    int *ep;
    if (device_err_ptr(dev, &ep)) return GTR_GLA_ERR_CUDA;
    int host_err = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbol(&host_err, g_dev_err, sizeof(int)) != cudaSuccess)
        return GTR_GLA_ERR_CUDA;
    if (host_err != 0 && cudaMemcpyToSymbol(g_dev_err, &zero, sizeof(int)) != cudaSuccess)
        return GTR_GLA_ERR_CUDA;
    if (host_err == kDevErrTimeout) return GTR_GLA_ERR_TIMEOUT;
    if (host_err == kDevErrWorkspace) return GTR_GLA_ERR_WORKSPACE_STATE;
    if (host_err == kDevErrBounds) return GTR_GLA_ERR_BOUNDS;
    return host_err ? GTR_GLA_ERR_CUDA : GTR_GLA_OK;
}

const char *gtr_gla_strerror(int code) {
    switch (code) {
        case GTR_GLA_OK: return "ok";
        case GTR_GLA_ERR_NULL: return "a required pointer is NULL";
        case GTR_GLA_ERR_SHAPE: return "B, H, grid_h or grid_w out of range";
        case GTR_GLA_ERR_HEAD_DIM: return "unsupported (d_k, d_v)";
        case GTR_GLA_ERR_DIRECTION: return "direction must be 0..3";
        case GTR_GLA_ERR_ALIGN: return "a pointer is not 16-byte aligned";
        case GTR_GLA_ERR_DTYPE: return "unsupported dtype";
        case GTR_GLA_ERR_CHUNK: return "unsupported chunk length";
        case GTR_GLA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case GTR_GLA_ERR_CUDA: return "CUDA runtime error";
        case GTR_GLA_ERR_TIMEOUT: return "a device-side wait timed out";
        case GTR_GLA_ERR_ALIAS: return "output overlaps an input";
        case GTR_GLA_ERR_WORKSPACE_STATE:
            return "workspace header not zero when a call started (overlapping calls sharing it?)";
        case GTR_GLA_ERR_BOUNDS: return "a kernel's index check failed (checked build)";
        default: return "unknown error code";
    }
}

void gtr_gla_release(void) {
    std::lock_guard<std::mutex> lock(g_mu);
    int cur = -1;
    cudaGetDevice(&cur);
    for (int d = 0; d < kMaxDevices; ++d) {
        if (!g_ws[d]) continue;
        if (cudaSetDevice(d) == cudaSuccess) {
            cudaDeviceSynchronize();
            cudaFree(g_ws[d]);
        }
        g_ws[d] = nullptr;
        g_ws_bytes[d] = 0;
    }
    if (cur >= 0) cudaSetDevice(cur);
}

unsigned long long gtr_gla_launch_count(void) { return g_launches.load(); }

}  // extern "C"
