// gla_common.cuh -- small device helpers shared by the CUDA kernels of
// libgtr_gla.so (token addressing per scan direction, dtype conversion).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gtr {

// Scan position p -> raster index r = y*grid_w + x of the row-major grid.
// Directions ("GTR: Gated Token Recurrence for Efficient Dense Prediction",
// x-techcon article, section 架构: left->right, right->left, top->bottom,
// bottom->top, one continuous scan over all tokens):
//   0 L->R  r = p
//   1 R->L  r = N-1-p
//   2 T->B  y = p mod grid_h, x = p div grid_h
//   3 B->T  T->B applied to N-1-p
// No token is ever copied into scan order: kernels address the grid in place.
__host__ __device__ __forceinline__ int scan_to_raster(int p, int n, int gh, int gw, int dir) {
    const int pp = (dir & 1) ? (n - 1 - p) : p;
    if (dir < 2) return pp;
    const int y = pp % gh;
    const int x = pp / gh;
    return y * gw + x;
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__half>(__half x) { return __half2float(x); }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// SiLU(z) = z * sigmoid(z) = z/2 * (1 + tanh(z/2)): one hardware tanh (relative
// error about 2^-11, that of an fp16 rounding of the result).
__device__ __forceinline__ float silu_f32(float z) {
    float t;
    const float hz = 0.5f * z;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(hz));
    return fmaf(hz, t, hz);
}

// Device-side error codes latched into the library's error word.
enum : int { kDevErrNone = 0, kDevErrTimeout = 1, kDevErrWorkspace = 2, kDevErrBounds = 3 };

__device__ __forceinline__ void latch_error(int *err, int code) {
    if (err) atomicCAS(err, 0, code);
}

// Index checks of the checked build (-DGTR_CHECKED, libgtr_gla_checked.so):
// every computed global index and TMA coordinate is tested before use; a
// failed test latches kDevErrBounds and the caller skips the access.  In the
// normal build the test compiles away.
#ifdef GTR_CHECKED
__device__ __forceinline__ bool index_ok(bool ok, int *err) {
    if (!ok) latch_error(err, kDevErrBounds);
    return ok;
}
#else
__device__ __forceinline__ bool index_ok(bool, int *) { return true; }
#endif

}  // namespace gtr
