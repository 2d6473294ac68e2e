/*
 * gtr_gla.h -- C ABI of the B200 (sm_100a) chunkwise key-gated linear
 * attention forward pass, the token mixer of GTR.
 *
 * Operation ("GTR: Gated Token Recurrence for Efficient Dense Prediction",
 * x-techcon article, section 架构 "architecture"): for every batch b and head
 * h, a state S (d_k x d_v) is carried along a scan of the grid_h x grid_w
 * patch-token grid.  At each token the gate keeps a per-key-dimension
 * fraction alpha = exp(log_alpha) of the state (key-only gating, value-side
 * decay fixed at 1), the token's key/value outer product is added, and the
 * token's query reads the updated state:
 *     S_t = diag(alpha_t) S_{t-1} + k_t^T v_t,   o_t = q_t S_t,   S_{-1} = 0.
 * The scan direction is chosen per call; every direction reads and writes the
 * row-major grid in place and the output is stored at each token's own grid
 * position (the grid order is restored after the scan, same section).
 * The sequence is evaluated chunkwise (same article, section 算子
 * "operator"): chunks compute their own state contribution in parallel, the
 * chunk-boundary states are passed along, and each chunk's output is then
 * produced in parallel; the attention scores never reach global memory.
 *
 * Tensor layout (all device pointers, contiguous, row-major):
 *   q, k        [B, H, grid_h, grid_w, d_k]   I/O dtype
 *   v, out      [B, H, grid_h, grid_w, d_v]   I/O dtype
 *   log_alpha   [B, H, grid_h, grid_w, d_k]   fp32, every value finite and <= 0
 *   final_state [B, H, d_k, d_v]              fp32, row i = key dimension i
 * The library never frees, retains or reallocates caller buffers.  Every
 * base pointer must be 16-byte aligned; out must not overlap any input.
 * No scale is applied inside (pre-scale k by 1/sqrt(d_k) if wanted).
 * log_alpha values outside (-inf, 0] are not checked and give undefined
 * results.
 *
 * Calls are asynchronous and stream-ordered; none synchronises the host
 * except gtr_gla_status() and the allocation done by gtr_gla_fwd() when its
 * internal workspace has to grow (do that first call outside any stream
 * capture).
 */
#ifndef GTR_GLA_H
#define GTR_GLA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#ifndef __CUDA_RUNTIME_API_H__
typedef struct CUstream_st *cudaStream_t;
#endif

/* ---- enums ---------------------------------------------------------- */

/* Scan directions, in the pages' layer-cycle order (section 架构). */
enum {
    GTR_GLA_L2R = 0, /* raster order                                  */
    GTR_GLA_R2L = 1, /* raster order reversed (whole sequence)       */
    GTR_GLA_T2B = 2, /* column-major: columns left->right, top->bottom */
    GTR_GLA_B2T = 3  /* column-major order reversed                  */
};

/* I/O dtypes of q, k, v and out. */
enum { GTR_GLA_F16 = 0, GTR_GLA_BF16 = 1, GTR_GLA_F32 = 2 };

/* Return codes.  Argument errors are reported before anything is launched. */
enum {
    GTR_GLA_OK = 0,
    GTR_GLA_ERR_NULL = -1,        /* a required pointer is NULL                   */
    GTR_GLA_ERR_SHAPE = -2,       /* B, H, grid_h or grid_w <= 0, or too large:
                                     B*H > 65535, grid_h*grid_w > 2^22 or
                                     B*H*grid_h*grid_w >= 2^31                  */
    GTR_GLA_ERR_HEAD_DIM = -3,    /* (d_k, d_v) not supported                     */
    GTR_GLA_ERR_DIRECTION = -4,   /* direction not in [0, 3]                      */
    GTR_GLA_ERR_ALIGN = -5,       /* a pointer is not 16-byte aligned             */
    GTR_GLA_ERR_DTYPE = -6,       /* dtype not one of GTR_GLA_F16/BF16/F32        */
    GTR_GLA_ERR_CHUNK = -7,       /* chunk length not supported for these sizes   */
    GTR_GLA_ERR_WORKSPACE = -8,   /* workspace NULL or smaller than required      */
    GTR_GLA_ERR_CUDA = -9,        /* a CUDA runtime call or launch failed         */
    GTR_GLA_ERR_TIMEOUT = -10,    /* a device-side wait gave up (gtr_gla_status)  */
    GTR_GLA_ERR_ALIAS = -11,      /* out overlaps an input, or a caller workspace
                                     overlaps a tensor argument                   */
    GTR_GLA_ERR_WORKSPACE_STATE = -12 /* a call found the workspace header not zero
                                         (calls sharing a workspace overlapped, or it
                                         was not zero-filled); reported by
                                         gtr_gla_status, the call did no work in the
                                         affected segments and the header is clean
                                         again afterwards                          */,
    GTR_GLA_ERR_BOUNDS = -13      /* checked build (libgtr_gla_checked.so) only,
                                     reported by gtr_gla_status: a kernel's index
                                     check failed; that access was skipped       */
};

/* ---- entry points --------------------------------------------------- */

/*
 * gtr_gla_fwd -- forward pass with fp16 q/k/v/out, chunk length 64 and a
 * workspace owned by the library (one per device, grown on demand, freed by
 * gtr_gla_release).  Calls that share the library workspace must not run
 * concurrently on the GPU (use one stream per device, or gtr_gla_fwd_ex with
 * separate workspaces).
 *   final_state may be NULL (not written).
 *   Supported (d_k, d_v): (64, 64), (128, 128), (64, 128), (128, 64).
 * Returns GTR_GLA_OK or a negative code; nothing is launched on error.
 */
int gtr_gla_fwd(const void *q, const void *k, const void *v, const float *log_alpha,
                void *out, float *final_state, int B, int H, int grid_h, int grid_w,
                int d_k, int d_v, int direction, cudaStream_t stream);

/*
 * gtr_gla_fwd_ex -- as gtr_gla_fwd with the I/O dtype, the chunk length and
 * the workspace chosen by the caller.
 *   dtype:     GTR_GLA_F16, GTR_GLA_BF16 or GTR_GLA_F32.
 *   chunk:     tokens per chunk: 32 or 64, or 128 when d_k = 64 (else
 *              GTR_GLA_ERR_CHUNK).  The result does not depend on it
 *              beyond rounding.  F16/BF16 with chunk 64 run the fused
 *              tensor-core kernel (head sizes of 128 as 64-wide parts, one
 *              launch per key half); every other combination runs the three-phase
 *              CUDA-core path.
 *   workspace: device buffer of at least gtr_gla_workspace_size(...) bytes,
 *              256-byte aligned, zero-filled before its first use.  Every call
 *              leaves it ready for the next one.  Calls that share a workspace
 *              must not overlap on the GPU.  May be NULL only when the
 *              required size is 0.  The bytes it uses must not overlap q, k,
 *              v, log_alpha, out or final_state (GTR_GLA_ERR_ALIAS).
 */
int gtr_gla_fwd_ex(const void *q, const void *k, const void *v, const float *log_alpha,
                   void *out, float *final_state, int B, int H, int grid_h, int grid_w,
                   int d_k, int d_v, int direction, int dtype, int chunk,
                   void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * gtr_gla_fwd_noalloc -- as gtr_gla_fwd, but the call allocates nothing.
 * The paper has no counterpart: this is a library convenience for callers
 * that cannot allocate device memory while they run (a fixed, pre-planned
 * memory budget, or host code with no device allocator of its own).
 *   Scratch: one 12 MiB device array inside this library, held by every GPU
 *   that loads it until the process exits, and shared by every call on that
 *   GPU.  Calls that overlap on the GPU race on it: order them (one stream per
 *   device, or explicit dependencies).  The array keeps the last call's
 *   contents; the part that must start at zero is zeroed once and left zero
 *   by every call.
 *   Set-up: the first call on a device (made with that device current) looks
 *   up the array's address and zeroes that part on `stream`; make that first
 *   call before any stream capture.
 *   Supported: fp16 q/k/v/out, d_k = d_v = 64, chunk 64 (the fused kernel);
 *   other head sizes return GTR_GLA_ERR_HEAD_DIM, and a problem whose scratch
 *   would exceed 12 MiB returns GTR_GLA_ERR_WORKSPACE.  Never calls cudaMalloc,
 *   cudaFree or any allocating routine.
 */
int gtr_gla_fwd_noalloc(const void *q, const void *k, const void *v, const float *log_alpha,
                        void *out, float *final_state, int B, int H, int grid_h, int grid_w,
                        int d_k, int d_v, int direction, cudaStream_t stream);

/*
 * gtr_gla_fwd_tail -- the forward pass followed by the output tail of GTR's
 * token mixer, with the tail fused into the attention's output stores
 * ("GTR: Gated Token Recurrence for Efficient Dense Prediction", x-techcon
 * article, section 算子: the operator's benchmark leaves this fusion out; the
 * pages do not define the tail, and the reading used is the per-token
 * epilogue of gtr_output_tail.h):
 *     y[b, r, h*d_v + j] = o[b, h, r, j] / sqrt(mean_j' o[b, h, r, j']^2 + eps)
 *                          * w_n[h, j] * SiLU(z[b, r, h*d_v + j])
 * with o the attention output of gtr_gla_fwd_ex (never written to memory when
 * d_k = d_v = 64: the norm is taken on its fp32 value and y is rounded once).
 *   z, y:      [B, grid_h, grid_w, H*d_v] in the I/O dtype (heads merged
 *              channels-last); y must not overlap any input.
 *   w_n:       [H, d_v] fp32.  eps: finite, >= 0.
 *   dtype:     GTR_GLA_F16 or GTR_GLA_BF16 (chunk 64).
 *   workspace: gtr_gla_tail_workspace_size(...) bytes, 256-byte aligned,
 *              zero-filled before its first use (as for gtr_gla_fwd_ex).
 *              Head sizes of 128 keep o there and run the tail as a second
 *              launch (gtr_output_tail_fwd).
 * Other arguments, errors and final_state as gtr_gla_fwd_ex; in addition
 * GTR_GLA_ERR_NULL for a NULL z or w_n, _SHAPE for eps < 0 or not finite,
 * _ALIGN for z or w_n, _ALIAS when y overlaps z or w_n, or the workspace
 * overlaps any tensor argument.
 */
int gtr_gla_fwd_tail(const void *q, const void *k, const void *v, const float *log_alpha,
                     const void *z, const float *w_n, float eps, void *y, float *final_state,
                     int B, int H, int grid_h, int grid_w, int d_k, int d_v, int direction,
                     int dtype, void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* Workspace bytes of gtr_gla_fwd_tail (0 for invalid sizes or dtypes). */
size_t gtr_gla_tail_workspace_size(int B, int H, int grid_h, int grid_w, int d_k, int d_v,
                                   int dtype);

/* Workspace bytes gtr_gla_fwd_ex needs for this problem (0 if none). */
size_t gtr_gla_workspace_size(int B, int H, int grid_h, int grid_w, int d_k, int d_v,
                              int dtype, int chunk);

/*
 * gtr_gla_status -- synchronise `stream` and report the first device-side
 * error latched by an earlier call on this device (GTR_GLA_ERR_TIMEOUT when a
 * bounded wait inside a kernel gave up, GTR_GLA_ERR_WORKSPACE_STATE when a
 * call found its workspace header not zero), or GTR_GLA_ERR_CUDA if the stream
 * itself reports an error.  Clears the latched error.  Returns GTR_GLA_OK if
 * all is well.
 */
int gtr_gla_status(cudaStream_t stream);

/* Static, human-readable text for a return code. */
const char *gtr_gla_strerror(int code);

/* Free the library-owned workspaces (all devices).  Synchronises each one. */
void gtr_gla_release(void);

/* Number of kernels this library has launched in this process so far. */
unsigned long long gtr_gla_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* GTR_GLA_H */
