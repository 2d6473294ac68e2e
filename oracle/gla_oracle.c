/*
 * gla_oracle.c -- fp64 CPU oracle for GTR's key-gated linear attention (GLA)
 * forward pass over a 2-D patch-token grid.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: it is used by tests/, by __graft_entry__.smoke() and by the
 * cpu_baseline / reference legs of bench.py.  It shares no code, header,
 * table or helper with the CUDA library; the two meet only through the seeded
 * input generator, which holds none of the method's arithmetic.
 *
 * What it computes (source: "GTR: Gated Token Recurrence for Efficient Dense
 * Prediction", x-techcon article, section 架构 "architecture"): a state matrix
 * S (d_k x d_v) is carried along a scan of the token grid.  At each token the
 * input-dependent gate first keeps a per-key-dimension fraction alpha of the
 * old state (key-only gating, value-side decay fixed at 1), then the token's
 * key/value outer product is written, and the token's query reads the UPDATED
 * state:
 *     S_t = diag(alpha_t) S_{t-1} + k_t^T v_t ,   o_t = q_t S_t ,
 * with alpha_t = exp(log_alpha_t) and S_{-1} = 0.  The article's formula
 * itself was lost in extraction; the recurrence above is the plainest reading
 * of the surrounding prose (the gate retains history per key dimension, then
 * the current key/value is written, then the query reads the updated state).
 *
 * Scan directions (same article, section 架构): consecutive layers scan
 * left->right, right->left, top->bottom, bottom->top, and the grid order is
 * restored after each scan.  Reading taken here: one continuous 1-D scan over
 * all N = grid_h*grid_w tokens (the state is not reset at row/column ends);
 *   0 L->R : raster order (row-major),
 *   1 R->L : raster order reversed,
 *   2 T->B : column-major order (columns left to right, top to bottom inside),
 *   3 B->T : column-major order reversed.
 * This oracle builds the scan-ordered sequence with explicit copies
 * (transpose, then reversal), runs one plain forward scan, and copies the
 * outputs back to raster positions.  Each token keeps its own gate.
 *
 * Chunkwise restatement (same article, section 算子 "operator"): the CUDA
 * operator splits the sequence into 64-token chunks, lets every chunk compute
 * its own contribution to the state in parallel, passes the chunk-boundary
 * states, and then produces every chunk's output in parallel.
 * gla_oracle_chunkwise() writes that reorganisation out literally in fp64,
 * for any chunk length, so tests can check it equals the recurrence before any
 * GPU code exists.
 *
 * Layout: q,k,log_alpha [B,H,grid_h,grid_w,d_k], v,out [B,H,grid_h,grid_w,d_v],
 * final_state [B,H,d_k,d_v] (row-major, d_k rows), all fp64, contiguous.
 * final_state is the state after the last token in scan order; it may be NULL.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- direction handling by explicit copies --------------------------- */

/* Copy one [grid_h, grid_w, d] plane into scan order. */
static void plane_to_scan(const double *src, double *dst, int gh, int gw, int d,
                          int direction)
{
    const int n = gh * gw;
    double *tmp = (double *)malloc((size_t)n * d * sizeof(double));
    if (direction == 2 || direction == 3) {
        /* transpose: scan position x*gh + y holds raster token y*gw + x */
        for (int y = 0; y < gh; ++y)
            for (int x = 0; x < gw; ++x)
                memcpy(tmp + ((size_t)x * gh + y) * d,
                       src + ((size_t)y * gw + x) * d, (size_t)d * sizeof(double));
    } else {
        memcpy(tmp, src, (size_t)n * d * sizeof(double));
    }
    if (direction == 1 || direction == 3) {
        for (int p = 0; p < n; ++p)
            memcpy(dst + (size_t)p * d, tmp + (size_t)(n - 1 - p) * d,
                   (size_t)d * sizeof(double));
    } else {
        memcpy(dst, tmp, (size_t)n * d * sizeof(double));
    }
    free(tmp);
}

/* Inverse of plane_to_scan: scan-ordered rows back to raster positions. */
static void scan_to_plane(const double *src, double *dst, int gh, int gw, int d,
                          int direction)
{
    const int n = gh * gw;
    double *tmp = (double *)malloc((size_t)n * d * sizeof(double));
    if (direction == 1 || direction == 3) {
        for (int p = 0; p < n; ++p)
            memcpy(tmp + (size_t)(n - 1 - p) * d, src + (size_t)p * d,
                   (size_t)d * sizeof(double));
    } else {
        memcpy(tmp, src, (size_t)n * d * sizeof(double));
    }
    if (direction == 2 || direction == 3) {
        for (int y = 0; y < gh; ++y)
            for (int x = 0; x < gw; ++x)
                memcpy(dst + ((size_t)y * gw + x) * d,
                       tmp + ((size_t)x * gh + y) * d, (size_t)d * sizeof(double));
    } else {
        memcpy(dst, tmp, (size_t)n * d * sizeof(double));
    }
    free(tmp);
}

/* ---- token-by-token recurrence (the definition) ---------------------- */

/* One (b,h) plane, already in scan order. */
static void scan_recurrence(const double *q, const double *k, const double *v,
                            const double *la, double *o, double *S, int n,
                            int dk, int dv)
{
    memset(S, 0, (size_t)dk * dv * sizeof(double));
    for (int t = 0; t < n; ++t) {
        const double *qt = q + (size_t)t * dk, *kt = k + (size_t)t * dk;
        const double *vt = v + (size_t)t * dv, *lat = la + (size_t)t * dk;
        /* S <- diag(alpha_t) S + k_t^T v_t */
        for (int i = 0; i < dk; ++i) {
            const double a = exp(lat[i]);
            double *Si = S + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) Si[j] = a * Si[j] + kt[i] * vt[j];
        }
        /* o_t = q_t S (reads the updated state) */
        double *ot = o + (size_t)t * dv;
        for (int j = 0; j < dv; ++j) ot[j] = 0.0;
        for (int i = 0; i < dk; ++i) {
            const double *Si = S + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) ot[j] += qt[i] * Si[j];
        }
    }
}

/* ---- chunkwise restatement ------------------------------------------- */

/* One (b,h) plane in scan order, chunk length C (any C >= 1).
 * Per chunk c covering scan positions [t0, t0+len):
 *   b_t   = sum_{u=t0..t} log_alpha_u            (inclusive, per key dim)
 *   g     = b at the chunk's last token
 *   o_t   = (q_t . e^{b_t}) S_in  +  sum_{s=t0..t} A[t,s] v_s
 *   A[t,s]= sum_i q_ti k_si e^{b_ti - b_si}      (s <= t, diagonal included)
 *   dS    = sum_s (k_s . e^{g - b_s})^T v_s
 *   S_in <- diag(e^{g}) S_in + dS                 (boundary-state pass)
 */
static void scan_chunkwise(const double *q, const double *k, const double *v,
                           const double *la, double *o, double *S, int n,
                           int dk, int dv, int C)
{
    double *b = (double *)malloc((size_t)C * dk * sizeof(double));
    double *dS = (double *)malloc((size_t)dk * dv * sizeof(double));
    memset(S, 0, (size_t)dk * dv * sizeof(double));
    for (int t0 = 0; t0 < n; t0 += C) {
        const int len = (n - t0 < C) ? (n - t0) : C;
        for (int i = 0; i < dk; ++i) {
            double acc = 0.0;
            for (int u = 0; u < len; ++u) {
                acc += la[(size_t)(t0 + u) * dk + i];
                b[(size_t)u * dk + i] = acc;
            }
        }
        const double *g = b + (size_t)(len - 1) * dk;
        for (int u = 0; u < len; ++u) {
            const int t = t0 + u;
            double *ot = o + (size_t)t * dv;
            for (int j = 0; j < dv; ++j) ot[j] = 0.0;
            /* inter-chunk part: (q_t . e^{b_t}) S_in */
            for (int i = 0; i < dk; ++i) {
                const double qi = q[(size_t)t * dk + i] * exp(b[(size_t)u * dk + i]);
                for (int j = 0; j < dv; ++j) ot[j] += qi * S[(size_t)i * dv + j];
            }
            /* intra-chunk part */
            for (int w = 0; w <= u; ++w) {
                const int s = t0 + w;
                double a = 0.0;
                for (int i = 0; i < dk; ++i)
                    a += q[(size_t)t * dk + i] * k[(size_t)s * dk + i] *
                         exp(b[(size_t)u * dk + i] - b[(size_t)w * dk + i]);
                for (int j = 0; j < dv; ++j) ot[j] += a * v[(size_t)s * dv + j];
            }
        }
        /* the chunk's own contribution to the state */
        memset(dS, 0, (size_t)dk * dv * sizeof(double));
        for (int w = 0; w < len; ++w) {
            const int s = t0 + w;
            for (int i = 0; i < dk; ++i) {
                const double kh = k[(size_t)s * dk + i] * exp(g[i] - b[(size_t)w * dk + i]);
                for (int j = 0; j < dv; ++j) dS[(size_t)i * dv + j] += kh * v[(size_t)s * dv + j];
            }
        }
        for (int i = 0; i < dk; ++i) {
            const double gam = exp(g[i]);
            for (int j = 0; j < dv; ++j)
                S[(size_t)i * dv + j] = gam * S[(size_t)i * dv + j] + dS[(size_t)i * dv + j];
        }
    }
    free(b);
    free(dS);
}

/* ---- public entry points (called from oracle/oracle.py via ctypes) ---- */

static int check_args(int B, int H, int gh, int gw, int dk, int dv, int direction)
{
    if (B <= 0 || H <= 0 || gh <= 0 || gw <= 0 || dk <= 0 || dv <= 0) return -1;
    if (direction < 0 || direction > 3) return -2;
    return 0;
}

/* mode 0: recurrence; mode > 0: chunkwise restatement with chunk = mode. */
static int run(const double *q, const double *k, const double *v, const double *la,
               double *out, double *final_state, int B, int H, int gh, int gw,
               int dk, int dv, int direction, int mode, int n_threads)
{
    int rc = check_args(B, H, gh, gw, dk, dv, direction);
    if (rc) return rc;
    const int n = gh * gw;
    const int planes = B * H;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < planes; ++bh) {
        double *qs = (double *)malloc((size_t)n * dk * sizeof(double));
        double *ks = (double *)malloc((size_t)n * dk * sizeof(double));
        double *las = (double *)malloc((size_t)n * dk * sizeof(double));
        double *vs = (double *)malloc((size_t)n * dv * sizeof(double));
        double *os = (double *)malloc((size_t)n * dv * sizeof(double));
        double *S = (double *)malloc((size_t)dk * dv * sizeof(double));
        plane_to_scan(q + (size_t)bh * n * dk, qs, gh, gw, dk, direction);
        plane_to_scan(k + (size_t)bh * n * dk, ks, gh, gw, dk, direction);
        plane_to_scan(la + (size_t)bh * n * dk, las, gh, gw, dk, direction);
        plane_to_scan(v + (size_t)bh * n * dv, vs, gh, gw, dv, direction);
        if (mode == 0)
            scan_recurrence(qs, ks, vs, las, os, S, n, dk, dv);
        else
            scan_chunkwise(qs, ks, vs, las, os, S, n, dk, dv, mode);
        scan_to_plane(os, out + (size_t)bh * n * dv, gh, gw, dv, direction);
        if (final_state)
            memcpy(final_state + (size_t)bh * dk * dv, S, (size_t)dk * dv * sizeof(double));
        free(qs); free(ks); free(las); free(vs); free(os); free(S);
    }
    return 0;
}

int gla_oracle_forward(const double *q, const double *k, const double *v,
                       const double *log_alpha, double *out, double *final_state,
                       int B, int H, int grid_h, int grid_w, int d_k, int d_v,
                       int direction, int n_threads)
{
    return run(q, k, v, log_alpha, out, final_state, B, H, grid_h, grid_w, d_k,
               d_v, direction, 0, n_threads);
}

int gla_oracle_chunkwise(const double *q, const double *k, const double *v,
                         const double *log_alpha, double *out, double *final_state,
                         int B, int H, int grid_h, int grid_w, int d_k, int d_v,
                         int direction, int chunk, int n_threads)
{
    if (chunk <= 0) return -3;
    return run(q, k, v, log_alpha, out, final_state, B, H, grid_h, grid_w, d_k,
               d_v, direction, chunk, n_threads);
}

int gla_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
