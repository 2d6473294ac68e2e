// gla_internal.h -- host-side declarations shared by the translation units of
// libgtr_gla.so (not part of the public ABI; see include/gtr_gla.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/gtr_gla.h"

namespace gtr {

// One validated forward-pass request.
struct Problem {
    const void *q, *k, *v;
    const float *la;
    void *out;
    float *final_state;  // may be null
    int B, H, gh, gw, n, dk, dv, dir, dtype, chunk;
    int *err;            // device error word of the current device
    // output tail fused into the stores (gtr_gla_fwd_tail): y = RMSNorm(o) w_n
    // * SiLU(z), heads merged [B, N, H d_v]; `out` is then not written
    int tail = 0;
    const void *z = nullptr;
    const float *wn = nullptr;
    void *y = nullptr;
    float eps = 0.f;
};

// Every workspace starts with a fixed header that only the fused kernel uses
// (ticket / completion counters and segment flags).  It is zero before a call
// and zero after it; the data areas of both paths start after it.
// Each segment flag has a 128-byte line of its own (kWsFlagStride ints), so a
// release store never lands on a line that other CTAs are polling for a
// different flag.
constexpr size_t kWsHeaderBytes = 65536;
constexpr int kWsFlagStride = 32;
constexpr int kWsMaxFlags = (int)((kWsHeaderBytes - 256) / (4 * kWsFlagStride));  // 510

// Record that one kernel was launched (feeds gtr_gla_launch_count()).
void note_launch();

// Raise a kernel's dynamic shared-memory limit on the current device, once per
// (kernel, device): later calls (e.g. inside a stream capture) touch no CUDA API.
int ensure_smem(const void *func, size_t bytes);

// Encode a tiled TMA map of rank 2..5 (tensormap.cu); 0 on success.
int encode_tile_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int rank,
                    const uint64_t *dims, const uint64_t *strides, const uint32_t *box,
                    bool swizzle128);
// The same with the shared-memory swizzle span in bytes (0, 32, 64 or 128).
int encode_tile_map_sw(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int rank,
                       const uint64_t *dims, const uint64_t *strides, const uint32_t *box,
                       int swizzle_bytes);

// Single-kernel tensor-core path (gla_fused.cu): fp16/bf16, chunk 64, d_k and d_v
// each 64 or 128 (head sizes of 128 as one launch per 64-wide key half).
bool fused_supported(const Problem &p);
size_t fused_workspace_bytes(const Problem &p);
int launch_fused(const Problem &p, void *ws, cudaStream_t st);

// Argument checks of the public entry points, and the current device's error
// word (gtr_gla_api.cu).
int check_problem(const Problem &p);
int error_word(int **out);

// Three-phase CUDA-core path (gla_generic.cu): all dtypes, chunk 32 or 64.
size_t generic_workspace_bytes(const Problem &p);
int launch_generic(const Problem &p, void *ws, cudaStream_t st);

// The library's tensor-core GEMM after its argument checks (tc_gemm.cu):
// out[M, N] = in[M, K] . W[N, K]^T (+ bias[N]) (+ resid[M, N]), row-major fp16
// or bf16, N and K multiples of 8, resid may be out.
int dense_gemm(int dtype, long long M, int N, int K, const void *in, const void *w, const void *bias,
               const void *resid, void *out, cudaStream_t st);

// Spatial SwiGLU block after its argument checks (swiglu.cu), with an optional
// residual: y = resid + SwiGLU(x) (resid and y may be the same tensor).  The
// workspace holds at least gtr_swiglu_workspace_size bytes.
int swiglu_apply(const void *x, const void *w_gu, const float *b_gu, const float *w_dw, const float *b_dw,
                 const void *w_down, const float *b_down, const void *resid, void *y, int B, int grid_h,
                 int grid_w, int C, int F, int dtype, void *workspace, cudaStream_t stream);

}  // namespace gtr
