/*
 * ca2_oracle.c -- plain fp64 CPU oracle for the Ca2-VDM cached attention path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check in __graft_entry__.py and the
 * CPU-baseline leg of bench.py may load this.  The product path (the CUDA library under
 * causal_kv_cache_b200/) never calls it and shares no code with it.
 *
 * Every function here is the textbook definition written out, in double precision, on
 * the exact values of the bf16 inputs.  No blocking, no online softmax, no ring buffer:
 * cached frames are handed in as a list of frame pointers in age order (oldest first).
 * The OpenMP loop only spreads independent output units over threads; the arithmetic
 * of every output element is the same sequential sum whatever the thread count.
 *
 * Sources ("Ca2-VDM" papernotes page = the ICML 2025 note on arXiv 2411.16375):
 *   temporal: section "关键设计 1 因果时序注意力", equation CausalAttn
 *             Softmax(Q K^T / sqrt(C') + M) V with M_ij = -inf for i < j (also the
 *             bohrium arXiv 2411.16375 page, "Formula Representation");
 *             C' read as the per-head dimension D.
 *   spatial:  section "关键设计 3 前缀增强空间注意力": the frame's own K/V concatenated
 *             along the spatial axis with the last P' prefix frames' spatial K/V; clean
 *             prefix frames are aligned by self-repeat; map size (HW) x ((P'+1) HW).
 *             No mask and scale 1/sqrt(D) (the page prints no formula; plain softmax
 *             attention is the reading taken).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf(uint16_t h)
{
    union { uint32_t u; float f; } x;
    x.u = ((uint32_t)h) << 16;
    return (double)x.f;
}

static long long frame_off(int b, int s, int h, int HW, int H, int D)
{
    /* offset of the D-vector of (video b, token s, head h) inside one frame-plane */
    return (((long long)b * HW + s) * H + h) * (long long)D;
}

/*
 * Causal temporal attention over the sequence [prefix frames 0..P-1 || chunk frames 0..n-1].
 *
 *   q, k, v : chunk tensors [B][n][HW][H][D] (bf16 bits)
 *   pk, pv  : P pointers, each to one cached frame-plane [B][HW][H][D], oldest first
 *   units   : if non-NULL, n_units indices u = (b*HW + s)*H + h to compute; else all
 *   out     : [n_units][n][D] doubles, unit-major in the order computed
 *
 * Sequence position of prefix frame p is p; of chunk frame c is P + c.  The query of chunk
 * frame c is row i = P + c; key j (0 <= j < L = P + n) gets logit q_i.k_j / sqrt(D) + M_ij
 * with M_ij = -inf when i < j, else 0.
 */
void oracle_temporal_attn(int B, int HW, int H, int D, int n, int P,
                          const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          const uint16_t *const *pk, const uint16_t *const *pv,
                          const long long *units, long long n_units, double *out)
{
    const long long total = (long long)B * HW * H;
    const long long nu = units ? n_units : total;
    const int L = P + n;
    const double inv_sqrt_d = 1.0 / sqrt((double)D);

#pragma omp parallel for schedule(dynamic, 4)
    for (long long ui = 0; ui < nu; ++ui) {
        const long long u = units ? units[ui] : ui;
        const int h = (int)(u % H);
        const int s = (int)((u / H) % HW);
        const int b = (int)(u / ((long long)H * HW));
        const long long fo = frame_off(b, s, h, HW, H, D);
        double *logit = (double *)malloc(sizeof(double) * (size_t)L);

        for (int c = 0; c < n; ++c) {
            const int i = P + c;
            /* q[b][c][s][h][:] */
            const uint16_t *qi = q + (((long long)b * n + c) * HW + s) * (long long)H * D + (long long)h * D;

            double m = -INFINITY;
            for (int j = 0; j < L; ++j) {
                const uint16_t *kj = (j < P)
                    ? pk[j] + fo
                    : k + (((long long)b * n + (j - P)) * HW + s) * (long long)H * D + (long long)h * D;
                double dot = 0.0;
                for (int d = 0; d < D; ++d) dot += bf(qi[d]) * bf(kj[d]);
                const double mask = (i < j) ? -INFINITY : 0.0;
                logit[j] = dot * inv_sqrt_d + mask;
                if (logit[j] > m) m = logit[j];
            }
            double den = 0.0;
            for (int j = 0; j < L; ++j) {
                logit[j] = exp(logit[j] - m);     /* exp(-inf) = 0 removes masked keys */
                den += logit[j];
            }
            double *o = out + (ui * n + c) * (long long)D;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            for (int j = 0; j < L; ++j) {
                const uint16_t *vj = (j < P)
                    ? pv[j] + fo
                    : v + (((long long)b * n + (j - P)) * HW + s) * (long long)H * D + (long long)h * D;
                const double w = logit[j] / den;
                for (int d = 0; d < D; ++d) o[d] += w * bf(vj[d]);
            }
        }
        free(logit);
    }
}

/*
 * Prefix-enhanced spatial attention, one frame at a time.
 *
 *   q, k, v : chunk tensors [B][n][HW][H][D] (bf16 bits)
 *   sk, sv  : n_sp pointers, each to one spatial-cache frame-plane [B][HW][H][D]
 *   repeat  : 0  -> denoising mode: keys/values = own frame's HW tokens, then each of the
 *                  n_sp prefix frames' HW tokens, concatenated along the spatial axis;
 *             R>0-> self-repeat mode: keys/values = the own frame's HW tokens written out
 *                  R times (R = P'+1 aligns a clean prefix frame with the (P'+1)HW map)
 *   units   : if non-NULL, n_units indices u = (b*n + f)*H + h to compute; else all
 *   out     : [n_units][HW][D] doubles
 */
void oracle_spatial_attn(int B, int HW, int H, int D, int n,
                         const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         const uint16_t *const *sk, const uint16_t *const *sv, int n_sp,
                         int repeat, const long long *units, long long n_units, double *out)
{
    const long long total = (long long)B * n * H;
    const long long nu = units ? n_units : total;
    const int n_blocks = repeat > 0 ? repeat : 1 + n_sp;   /* HW-token blocks in the key list */
    const long long NK = (long long)n_blocks * HW;
    const double inv_sqrt_d = 1.0 / sqrt((double)D);

#pragma omp parallel for schedule(dynamic, 1)
    for (long long ui = 0; ui < nu; ++ui) {
        const long long u = units ? units[ui] : ui;
        const int h = (int)(u % H);
        const int f = (int)((u / H) % n);
        const int b = (int)(u / ((long long)H * n));
        double *logit = (double *)malloc(sizeof(double) * (size_t)NK);
        const uint16_t **krow = (const uint16_t **)malloc(sizeof(uint16_t *) * (size_t)NK);
        const uint16_t **vrow = (const uint16_t **)malloc(sizeof(uint16_t *) * (size_t)NK);

        /* the concatenated key / value list, block by block */
        for (int blk = 0; blk < n_blocks; ++blk) {
            for (int t = 0; t < HW; ++t) {
                const long long j = (long long)blk * HW + t;
                if (repeat > 0 || blk == 0) {
                    const long long off = (((long long)b * n + f) * HW + t) * (long long)H * D + (long long)h * D;
                    krow[j] = k + off;
                    vrow[j] = v + off;
                } else {
                    const long long off = frame_off(b, t, h, HW, H, D);
                    krow[j] = sk[blk - 1] + off;
                    vrow[j] = sv[blk - 1] + off;
                }
            }
        }

        for (int i = 0; i < HW; ++i) {
            const uint16_t *qi = q + (((long long)b * n + f) * HW + i) * (long long)H * D + (long long)h * D;
            double m = -INFINITY;
            for (long long j = 0; j < NK; ++j) {
                double dot = 0.0;
                for (int d = 0; d < D; ++d) dot += bf(qi[d]) * bf(krow[j][d]);
                logit[j] = dot * inv_sqrt_d;
                if (logit[j] > m) m = logit[j];
            }
            double den = 0.0;
            for (long long j = 0; j < NK; ++j) {
                logit[j] = exp(logit[j] - m);
                den += logit[j];
            }
            double *o = out + (ui * HW + i) * (long long)D;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            for (long long j = 0; j < NK; ++j) {
                const double w = logit[j] / den;
                for (int d = 0; d < D; ++d) o[d] += w * bf(vrow[j][d]);
            }
        }
        free(logit);
        free(krow);
        free(vrow);
    }
}

/* Number of OpenMP threads the loops above will use (1 when built without OpenMP). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
