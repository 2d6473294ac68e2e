// gla_internal.h -- host-side declarations shared by the translation units of
// libgtr_gla.so (not part of the public ABI; see include/gtr_gla.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

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
};

// Record that one kernel was launched (feeds gtr_gla_launch_count()).
void note_launch();

// Raise a kernel's dynamic shared-memory limit on the current device, once per
// (kernel, device): later calls (e.g. inside a stream capture) touch no CUDA API.
int ensure_smem(const void *func, size_t bytes);

// Three-phase CUDA-core path (gla_generic.cu): all dtypes, chunk 32 or 64.
size_t generic_workspace_bytes(const Problem &p);
int launch_generic(const Problem &p, void *ws, cudaStream_t st);

}  // namespace gtr
