/*
 * gla_backward.c -- fp64 CPU oracle for the gradients of GTR's key-gated
 * linear attention over a 2-D patch-token grid.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file; it shares no code with the CUDA library.
 *
 * The forward pass is the recurrence of gla_oracle.c ("GTR: Gated Token
 * Recurrence for Efficient Dense Prediction", x-techcon article, section 架构):
 *     S_t = diag(alpha_t) S_{t-1} + k_t^T v_t,   o_t = q_t S_t,
 * alpha_t = exp(log_alpha_t), S_{-1} = 0, along the scan order of the chosen
 * direction.  (The pages train with the FLA library's kernel and give no
 * backward pass; its gradients follow from the recurrence alone.)
 *
 * Given dO = dL/do for every token and dS = dL/dS_final (may be NULL, read as
 * zero), reverse-mode through the recurrence carries G_t = dL/dS_t backwards:
 *     G_{n-1} = dS + q_{n-1}^T dO_{n-1},
 *     G_{t-1} = diag(alpha_t) G_t + q_{t-1}^T dO_{t-1},
 * and at every token
 *     dq_t          = dO_t S_t^T            (o_t reads S_t)
 *     dk_t[i]       = sum_j G_t[i,j] v_t[j]
 *     dv_t[j]       = sum_i k_t[i] G_t[i,j]
 *     dlog_alpha_t[i] = alpha_t[i] * sum_j G_t[i,j] S_{t-1}[i,j].
 * The forward states are kept (n * d_k * d_v doubles per plane), which is
 * meant for test-sized planes.
 *
 * Directions: the plane is copied into scan order (transpose for the column
 * scans, reversal for the reversed ones), scanned, and the gradients copied
 * back to raster positions, as in gla_oracle.c.
 *
 * Layout: q, k, log_alpha and their gradients [B,H,grid_h,grid_w,d_k]; v, dO,
 * dv [B,H,grid_h,grid_w,d_v]; dS [B,H,d_k,d_v]; all fp64, contiguous.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

static void bw_to_scan(const double *src, double *dst, int gh, int gw, int d, int direction)
{
    const int n = gh * gw;
    for (int p = 0; p < n; ++p) {
        /* scan position p -> position q of the unreversed order -> raster token r
           (column scans visit x * gh + y for raster y * gw + x) */
        const int q = (direction == 1 || direction == 3) ? n - 1 - p : p;
        const int r = (direction == 2 || direction == 3) ? (q % gh) * gw + q / gh : q;
        memcpy(dst + (size_t)p * d, src + (size_t)r * d, (size_t)d * sizeof(double));
    }
}

static void bw_from_scan(const double *src, double *dst, int gh, int gw, int d, int direction)
{
    const int n = gh * gw;
    for (int p = 0; p < n; ++p) {
        const int q = (direction == 1 || direction == 3) ? n - 1 - p : p;
        const int r = (direction == 2 || direction == 3) ? (q % gh) * gw + q / gh : q;
        memcpy(dst + (size_t)r * d, src + (size_t)p * d, (size_t)d * sizeof(double));
    }
}

/* One plane in scan order.  States: n+1 slots of dk*dv (slot t+1 = S_t). */
static void plane_backward(const double *q, const double *k, const double *v, const double *la,
                           const double *dO, const double *dS, double *dq, double *dk_,
                           double *dv_, double *dla, double *states, int n, int dk, int dv)
{
    const size_t SZ = (size_t)dk * dv;
    memset(states, 0, SZ * sizeof(double));
    for (int t = 0; t < n; ++t) {
        const double *Sp = states + (size_t)t * SZ;
        double *St = states + (size_t)(t + 1) * SZ;
        for (int i = 0; i < dk; ++i) {
            const double a = exp(la[(size_t)t * dk + i]);
            for (int j = 0; j < dv; ++j)
                St[(size_t)i * dv + j] = a * Sp[(size_t)i * dv + j] + k[(size_t)t * dk + i] * v[(size_t)t * dv + j];
        }
    }
    double *G = (double *)calloc(SZ, sizeof(double));
    if (dS) memcpy(G, dS, SZ * sizeof(double));
    for (int t = n - 1; t >= 0; --t) {
        const double *qt = q + (size_t)t * dk, *kt = k + (size_t)t * dk, *vt = v + (size_t)t * dv;
        const double *gt = dO + (size_t)t * dv;
        const double *St = states + (size_t)(t + 1) * SZ, *Sp = states + (size_t)t * SZ;
        /* this token's read of S_t */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] += qt[i] * gt[j];
        for (int i = 0; i < dk; ++i) {
            double sq = 0.0, sk = 0.0, sa = 0.0;
            for (int j = 0; j < dv; ++j) {
                sq += gt[j] * St[(size_t)i * dv + j];
                sk += G[(size_t)i * dv + j] * vt[j];
                sa += G[(size_t)i * dv + j] * Sp[(size_t)i * dv + j];
            }
            dq[(size_t)t * dk + i] = sq;
            dk_[(size_t)t * dk + i] = sk;
            dla[(size_t)t * dk + i] = exp(la[(size_t)t * dk + i]) * sa;
        }
        for (int j = 0; j < dv; ++j) {
            double s = 0.0;
            for (int i = 0; i < dk; ++i) s += kt[i] * G[(size_t)i * dv + j];
            dv_[(size_t)t * dv + j] = s;
        }
        /* on to dL/dS_{t-1} */
        for (int i = 0; i < dk; ++i) {
            const double a = exp(la[(size_t)t * dk + i]);
            for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] *= a;
        }
    }
    free(G);
}

int gla_oracle_backward(const double *q, const double *k, const double *v, const double *la,
                        const double *dO, const double *dS, double *dq, double *dk_, double *dv_,
                        double *dla, int B, int H, int gh, int gw, int dk, int dv, int direction)
{
    if (B <= 0 || H <= 0 || gh <= 0 || gw <= 0 || dk <= 0 || dv <= 0) return 1;
    if (direction < 0 || direction > 3) return 2;
    const int n = gh * gw;
    const size_t pk = (size_t)n * dk, pv = (size_t)n * dv;
    /* scan-ordered copies of q, k, log_alpha, v, dO and of the gradients,
       then the n + 1 states */
    double *buf = (double *)malloc((6 * pk + 3 * pv + (size_t)(n + 1) * dk * dv) * sizeof(double));
    if (!buf) return 3;
    double *sq = buf, *sk = sq + pk, *sla = sk + pk, *sdq = sla + pk, *sdk = sdq + pk, *sdla = sdk + pk;
    double *sv = sdla + pk, *sdO = sv + pv, *sdv = sdO + pv;
    double *states = sdv + pv;
    for (int p = 0; p < B * H; ++p) {
        bw_to_scan(q + p * pk, sq, gh, gw, dk, direction);
        bw_to_scan(k + p * pk, sk, gh, gw, dk, direction);
        bw_to_scan(la + p * pk, sla, gh, gw, dk, direction);
        bw_to_scan(v + p * pv, sv, gh, gw, dv, direction);
        bw_to_scan(dO + p * pv, sdO, gh, gw, dv, direction);
        plane_backward(sq, sk, sv, sla, sdO, dS ? dS + (size_t)p * dk * dv : NULL, sdq, sdk, sdv, sdla,
                       states, n, dk, dv);
        bw_from_scan(sdq, dq + p * pk, gh, gw, dk, direction);
        bw_from_scan(sdk, dk_ + p * pk, gh, gw, dk, direction);
        bw_from_scan(sdv, dv_ + p * pv, gh, gw, dv, direction);
        bw_from_scan(sdla, dla + p * pk, gh, gw, dk, direction);
    }
    free(buf);
    return 0;
}
