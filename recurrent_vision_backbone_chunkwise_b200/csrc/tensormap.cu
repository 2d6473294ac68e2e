// tensormap.cu -- host-side TMA descriptor encoding (cuTensorMapEncodeTiled,
// reached through the runtime's driver entry point so the library does not
// link libcuda directly).
#include <mutex>

#include <cudaTypedefs.h>

#include "gla_internal.h"

namespace gtr {

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// A tiled view of rank 2..5 (dims innermost first, strides in bytes for
// dims 1..rank-1); loads of `box` elements start at any coordinate, elements
// outside the tensor read as zero.
int encode_tile_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int rank,
                    const uint64_t *dims, const uint64_t *strides, const uint32_t *box,
                    bool swizzle128) {
    return encode_tile_map_sw(m, base, dt, rank, dims, strides, box, swizzle128 ? 128 : 0);
}

int encode_tile_map_sw(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int rank,
                       const uint64_t *dims, const uint64_t *strides, const uint32_t *box,
                       int swizzle_bytes) {
    auto fn = encode_fn();
    if (!fn || rank < 2 || rank > 5) return 1;
    cuuint64_t d[5], st[4];
    cuuint32_t b[5], e[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
        e[i] = 1;
    }
    for (int i = 0; i < rank - 1; ++i) st[i] = strides[i];
    CUresult r = fn(m, dt, rank, const_cast<void *>(base), d, st, b, e,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                    : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                    : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                          : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? 0 : 1;
}

}  // namespace gtr
