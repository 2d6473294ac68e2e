// io_pack.cuh -- two 16-bit I/O values in one 32-bit word <-> a float2, for
// the elementwise kernels of the library (fp16 and bf16, round to nearest even).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace gtr {

template <typename T> struct Pair;
template <> struct Pair<__half> {
    static __device__ __forceinline__ float2 unpack(uint32_t w) {
        return __half22float2(*reinterpret_cast<__half2 *>(&w));
    }
    static __device__ __forceinline__ uint32_t pack(float a, float b) {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&h);
    }
};
template <> struct Pair<__nv_bfloat16> {
    static __device__ __forceinline__ float2 unpack(uint32_t w) {
        return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&w));
    }
    static __device__ __forceinline__ uint32_t pack(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&h);
    }
};

// Eight 16-bit values (one 16-byte load) as four float2.
template <typename T>
__device__ __forceinline__ void unpack8(const uint4 &w, float2 *f) {
    f[0] = Pair<T>::unpack(w.x);
    f[1] = Pair<T>::unpack(w.y);
    f[2] = Pair<T>::unpack(w.z);
    f[3] = Pair<T>::unpack(w.w);
}

}  // namespace gtr
