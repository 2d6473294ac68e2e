// gla_noalloc.cu -- gtr_gla_fwd_noalloc: the fused forward pass with its
// scratch in a fixed device array, so the call itself allocates nothing.
//
// Some callers cannot allocate device memory while they run: a deployment
// with a fixed, pre-planned memory budget, or host code that has no device
// allocator of its own and no way to manage a workspace buffer.  For them
// this entry point keeps the fused kernel's scratch (look-back flags,
// counters and per-segment states) in one file-scope device array of
// kNoAllocScratchBytes, which every GPU that loads this library holds until
// the process exits.
#include <mutex>

#include "gla_common.cuh"
#include "gla_internal.h"

namespace gtr {
namespace {

constexpr size_t kNoAllocScratchBytes = 12u << 20;  // 12 MiB
constexpr int kNoAllocMaxDevices = 64;

// Device-side scratch.  In host code this name is only a stand-in for the
// symbol, never a device address: the address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kNoAllocMaxDevices];

// Once per device, with that device current: look up the array's device
// address and zero the part that must start at zero (the fused kernel's
// synchronisation header; every later call leaves it zero again).
int noalloc_setup(int dev, cudaStream_t st, void **out) {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr)
            return GTR_GLA_ERR_CUDA;
        if (cudaMemsetAsync(ptr, 0, kWsHeaderBytes, st) != cudaSuccess) return GTR_GLA_ERR_CUDA;
        g_noalloc_ptr[dev] = ptr;
    }
    *out = g_noalloc_ptr[dev];
    return GTR_GLA_OK;
}

}  // namespace
}  // namespace gtr

using namespace gtr;

extern "C" int gtr_gla_fwd_noalloc(const void *q, const void *k, const void *v,
                                   const float *log_alpha, void *out, float *final_state, int B,
                                   int H, int grid_h, int grid_w, int d_k, int d_v, int direction,
                                   cudaStream_t stream) {
    Problem p;
    p.q = q;
    p.k = k;
    p.v = v;
    p.la = log_alpha;
    p.out = out;
    p.final_state = final_state;
    p.B = B;
    p.H = H;
    p.gh = grid_h;
    p.gw = grid_w;
    p.n = (grid_h > 0 && grid_w > 0 && (long long)grid_h * grid_w <= (1LL << 22)) ? grid_h * grid_w : 0;
    p.dk = d_k;
    p.dv = d_v;
    p.dir = direction;
    p.dtype = GTR_GLA_F16;
    p.chunk = 64;
    p.err = nullptr;
    int rc = check_problem(p);
    if (rc) return rc;
    if (!fused_supported(p) || p.dk != 64 || p.dv != 64) return GTR_GLA_ERR_HEAD_DIM;
    if (fused_workspace_bytes(p) > kNoAllocScratchBytes) return GTR_GLA_ERR_WORKSPACE;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices)
        return GTR_GLA_ERR_CUDA;
    if ((rc = error_word(&p.err))) return rc;
    void *scratch = nullptr;
    if ((rc = noalloc_setup(dev, stream, &scratch))) return rc;
    return launch_fused(p, scratch, stream);
}
