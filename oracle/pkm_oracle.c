/*
 * pkm_oracle.c -- plain, slow, obviously-correct CPU oracle for the
 * product-key memory lookup.  TEST INFRASTRUCTURE ONLY: the tests, the
 * smoke check and the CPU-baseline leg of the benchmark call it; the CUDA
 * library never links, includes or calls anything in this directory, and
 * this file shares no code with it.
 *
 * Every quantity is computed in IEEE double from the exact input values
 * (bf16 and fp32 inputs are decoded exactly), one (token, head) at a time,
 * in the order the method states.  There is no blocking, fusion or
 * reordering.  Sorting uses the C library's qsort (a library primitive).
 *
 * Sources (web pages on the method; cited by title and section):
 *   [MLS]  "Memory Layers at Scale" digest page: sections "Product-key
 *          검색" (keys split in two sub-keys; top-k with 2*sqrt(N)
 *          comparisons instead of N), "Memory+ 블록" (gate
 *          (y ⊙ silu(x W1)) W2 and qk-normalization), "병렬 EmbeddingBag
 *          구현" (the weighted bag gather).
 *   [MEM]  "모델 안의 메모리" explainer page: section "작동 방식" (query split
 *          into front and back halves, each scored against ~1000 half-keys,
 *          best of each combined; a few values read and weight-averaged; a
 *          gate decides how much passes on) and figure D (8+8 comparisons
 *          over 64 cells).
 *
 * Readings where the pages are silent (each also listed in the design
 * notes): L2 normalisation of every query half and sub-key row with the
 * norm clamped at 1e-12; score scale sqrt(d_half); full score
 * S(a,b) = s1[a] + s2[b]; row id a*n_sub + b; softmax over the k selected;
 * per-head sub-key tables, one shared value table, per-head bags summed;
 * order = larger score first, equal scores -> smaller id first, applied at
 * every selection.
 *
 * Parity pins of each function live in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "pkm_oracle.h"

/* ------------------------------------------------------------------ */
/* exact decoding of the input element types                           */
/* ------------------------------------------------------------------ */

static double bf16_to_double(uint16_t h) {
    uint32_t bits = ((uint32_t)h) << 16; /* bf16 is the top half of fp32 */
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* element i of a tensor stored as ORC_F64 / ORC_F32 / ORC_BF16 */
static double ld(const void *p, int dtype, int64_t i) {
    switch (dtype) {
    case ORC_F64: return ((const double *)p)[i];
    case ORC_F32: return (double)((const float *)p)[i];
    default: return bf16_to_double(((const uint16_t *)p)[i]);
    }
}

/* ------------------------------------------------------------------ */
/* qk-normalization [MLS "Memory+ 블록"]                               */
/* ------------------------------------------------------------------ */

/* u = x / max(||x||_2, eps); returns max(||x||_2, eps). */
static double unit_vector(const void *x, int dtype, int64_t off, int d, double *u) {
    double ss = 0.0;
    for (int i = 0; i < d; i++) {
        double v = ld(x, dtype, off + i);
        ss += v * v;
    }
    double nrm = sqrt(ss);
    double den = nrm > ORC_NORM_EPS ? nrm : ORC_NORM_EPS;
    for (int i = 0; i < d; i++) u[i] = ld(x, dtype, off + i) / den;
    return den;
}

/* ------------------------------------------------------------------ */
/* ordering used by every selection                                     */
/* ------------------------------------------------------------------ */

typedef struct {
    double s;   /* score */
    int64_t id; /* position (half) or row id (full key) */
} cand_t;

/* larger score first; equal scores -> smaller id first */
static int cand_cmp(const void *pa, const void *pb) {
    const cand_t *a = (const cand_t *)pa, *b = (const cand_t *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    if (a->id < b->id) return -1;
    if (a->id > b->id) return 1;
    return 0;
}

/* ------------------------------------------------------------------ */
/* half scores                                                          */
/* ------------------------------------------------------------------ */

/*
 * Unit sub-keys kappa[h][c][a][:] for all heads and halves (computed once
 * per call; each row is the same normalisation as in the definition).
 */
static double *unit_subkeys(const void *K, int k_dtype, int H, int n, int dh) {
    double *kap = (double *)malloc(sizeof(double) * (size_t)H * 2 * n * dh);
    if (!kap) return NULL;
    for (int64_t r = 0; r < (int64_t)H * 2 * n; r++)
        unit_vector(K, k_dtype, r * dh, dh, kap + r * dh);
    return kap;
}

/*
 * s_c[a] = sqrt(d_half) * <u_c, kappa_c[a]> for every a < n
 * [MEM "작동 방식": each half of the query is compared with every half-key].
 * Writes u_c (the unit query half) into u.
 */
static void half_scores(const void *q, int q_dtype, int64_t t, int h, int c, int H,
                        int dh, int n, const double *kap, double *u, double *s) {
    int64_t off = (((t * H) + h) * 2 + c) * (int64_t)dh;
    unit_vector(q, q_dtype, off, dh, u);
    const double scale = sqrt((double)dh);
    const double *kc = kap + ((int64_t)(h * 2 + c) * n) * dh;
    for (int a = 0; a < n; a++) {
        double acc = 0.0;
        for (int i = 0; i < dh; i++) acc += u[i] * kc[(int64_t)a * dh + i];
        s[a] = scale * acc;
    }
}

int orc_half_scores(int64_t T, int H, int dh, int n, const void *q, int q_dtype,
                    const void *K, int k_dtype, double *s_out) {
    double *kap = unit_subkeys(K, k_dtype, H, n, dh);
    if (!kap) return -1;
    int err = 0;
#pragma omp parallel
    {
        double *u = (double *)malloc(sizeof(double) * dh);
        if (!u) err = -1;
#pragma omp for schedule(dynamic, 4)
        for (int64_t th = 0; th < T * H; th++) {
            if (!u) continue;
            int64_t t = th / H;
            int h = (int)(th % H);
            for (int c = 0; c < 2; c++)
                half_scores(q, q_dtype, t, h, c, H, dh, n, kap, u,
                            s_out + ((t * H + h) * 2 + c) * (int64_t)n);
        }
        free(u);
    }
    free(kap);
    return err;
}

/* ------------------------------------------------------------------ */
/* product-key selection [MLS "Product-key 검색"], [MEM "작동 방식"]   */
/* ------------------------------------------------------------------ */

/* indices (positions) of the k best entries of s[0..n) in selection order */
static void topk_positions(const double *s, int n, int k, cand_t *work, int *pos) {
    for (int a = 0; a < n; a++) {
        work[a].s = s[a];
        work[a].id = a;
    }
    qsort(work, (size_t)n, sizeof(cand_t), cand_cmp);
    for (int j = 0; j < k; j++) pos[j] = (int)work[j].id;
}

int orc_topk(const double *s, int n, int k, int *pos_out) {
    cand_t *work = (cand_t *)malloc(sizeof(cand_t) * (size_t)n);
    if (!work) return -1;
    topk_positions(s, n, k, work, pos_out);
    free(work);
    return 0;
}

/* softmax over the k selected scores [MEM "작동 방식": weighted average] */
static void softmax(const double *S, int k, double *w) {
    double m = S[0];
    for (int j = 1; j < k; j++) m = S[j] > m ? S[j] : m;
    double z = 0.0;
    for (int j = 0; j < k; j++) {
        w[j] = exp(S[j] - m);
        z += w[j];
    }
    for (int j = 0; j < k; j++) w[j] /= z;
}

int orc_pkm_select(int64_t T, int H, int dh, int n, int k, const void *q, int q_dtype,
                   const void *K, int k_dtype, int64_t *idx_out, double *score_out,
                   double *w_out, int64_t *n_half_dots) {
    if (k < 1 || k > n) return -2;
    double *kap = unit_subkeys(K, k_dtype, H, n, dh);
    if (!kap) return -1;
    int err = 0;
    int64_t dots = 0;
#pragma omp parallel reduction(+ : dots)
    {
        double *u = (double *)malloc(sizeof(double) * dh);
        double *s1 = (double *)malloc(sizeof(double) * n);
        double *s2 = (double *)malloc(sizeof(double) * n);
        cand_t *work = (cand_t *)malloc(sizeof(cand_t) * (size_t)(n > k * k ? n : k * k));
        int *p1 = (int *)malloc(sizeof(int) * k);
        int *p2 = (int *)malloc(sizeof(int) * k);
        int ok = u && s1 && s2 && work && p1 && p2;
        if (!ok) err = -1;
#pragma omp for schedule(dynamic, 4)
        for (int64_t th = 0; th < T * H; th++) {
            if (!ok) continue;
            int64_t t = th / H;
            int h = (int)(th % H);
            /* 1. score each half against its n half-keys: 2n dot products */
            half_scores(q, q_dtype, t, h, 0, H, dh, n, kap, u, s1);
            half_scores(q, q_dtype, t, h, 1, H, dh, n, kap, u, s2);
            dots += 2 * (int64_t)n;
            /* 2. the k best of each half */
            topk_positions(s1, n, k, work, p1);
            topk_positions(s2, n, k, work, p2);
            /* 3. combine the best of each half: k*k candidate full keys */
            for (int i = 0; i < k; i++)
                for (int j = 0; j < k; j++) {
                    work[i * k + j].s = s1[p1[i]] + s2[p2[j]];
                    work[i * k + j].id = (int64_t)p1[i] * n + p2[j];
                }
            /* 4. the k best candidates, in selection order */
            qsort(work, (size_t)k * k, sizeof(cand_t), cand_cmp);
            double *S = score_out + th * k;
            for (int j = 0; j < k; j++) {
                idx_out[th * k + j] = work[j].id;
                S[j] = work[j].s;
            }
            /* 5. softmax weights */
            softmax(S, k, w_out + th * k);
        }
        free(u);
        free(s1);
        free(s2);
        free(work);
        free(p1);
        free(p2);
    }
    free(kap);
    if (n_half_dots) *n_half_dots = dots;
    return err;
}

/*
 * The plain definition: score all N = n*n full keys and keep the k best.
 * The full key of row a*n+b is the concatenation of sub-keys K1[a] and
 * K2[b]; its score is s1[a] + s2[b].
 */
int orc_bruteforce_select(int64_t T, int H, int dh, int n, int k, const void *q,
                          int q_dtype, const void *K, int k_dtype, int64_t *idx_out,
                          double *score_out) {
    int64_t N = (int64_t)n * n;
    if (k < 1 || k > N) return -2;
    double *kap = unit_subkeys(K, k_dtype, H, n, dh);
    if (!kap) return -1;
    int err = 0;
#pragma omp parallel
    {
        double *u = (double *)malloc(sizeof(double) * dh);
        double *s1 = (double *)malloc(sizeof(double) * n);
        double *s2 = (double *)malloc(sizeof(double) * n);
        cand_t *all = (cand_t *)malloc(sizeof(cand_t) * (size_t)N);
        int ok = u && s1 && s2 && all;
        if (!ok) err = -1;
#pragma omp for schedule(dynamic, 1)
        for (int64_t th = 0; th < T * H; th++) {
            if (!ok) continue;
            int64_t t = th / H;
            int h = (int)(th % H);
            half_scores(q, q_dtype, t, h, 0, H, dh, n, kap, u, s1);
            half_scores(q, q_dtype, t, h, 1, H, dh, n, kap, u, s2);
            for (int64_t r = 0; r < N; r++) {
                all[r].s = s1[r / n] + s2[r % n];
                all[r].id = r;
            }
            qsort(all, (size_t)N, sizeof(cand_t), cand_cmp);
            for (int j = 0; j < k; j++) {
                idx_out[th * k + j] = all[j].id;
                score_out[th * k + j] = all[j].s;
            }
        }
        free(u);
        free(s1);
        free(s2);
        free(all);
    }
    free(kap);
    return err;
}

int orc_softmax(const double *S, int64_t rows, int k, double *w_out) {
    for (int64_t r = 0; r < rows; r++) softmax(S + r * k, k, w_out + r * k);
    return 0;
}

/* ------------------------------------------------------------------ */
/* weighted bag gather [MLS "병렬 EmbeddingBag 구현"]                    */
/* ------------------------------------------------------------------ */

int orc_bag(int64_t n_bags, int B, int d, const int64_t *idx, const double *w,
            const void *table, int t_dtype, int64_t n_rows, double *y_out) {
    int err = 0;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n_bags; t++) {
        double *y = y_out + t * d;
        for (int i = 0; i < d; i++) y[i] = 0.0;
        for (int j = 0; j < B; j++) {
            int64_t r = idx[t * B + j];
            if (r < 0 || r >= n_rows) {
                err = -3;
                continue;
            }
            double wj = w[t * B + j];
            for (int i = 0; i < d; i++) y[i] += wj * ld(table, t_dtype, r * d + i);
        }
    }
    return err;
}

/* ------------------------------------------------------------------ */
/* Memory+ gate [MLS "Memory+ 블록"]: out = (y ⊙ silu(x W1)) W2          */
/* ------------------------------------------------------------------ */

static double silu(double z) { return z / (1.0 + exp(-z)); }

int orc_memplus(int64_t T, int dm, int dv, const double *y, const void *x, int x_dtype,
                const void *W1, int w1_dtype, const void *W2, int w2_dtype,
                double *out) {
    int err = 0;
#pragma omp parallel
    {
        double *z = (double *)malloc(sizeof(double) * dv);
        if (!z) err = -1;
#pragma omp for schedule(static)
        for (int64_t t = 0; t < T; t++) {
            if (!z) continue;
            for (int v = 0; v < dv; v++) {
                double a = 0.0;
                for (int m = 0; m < dm; m++)
                    a += ld(x, x_dtype, t * dm + m) * ld(W1, w1_dtype, (int64_t)m * dv + v);
                z[v] = y[t * dv + v] * silu(a);
            }
            for (int m = 0; m < dm; m++) {
                double a = 0.0;
                for (int v = 0; v < dv; v++) a += z[v] * ld(W2, w2_dtype, (int64_t)v * dm + m);
                out[t * dm + m] = a;
            }
        }
        free(z);
    }
    return err;
}

/* ------------------------------------------------------------------ */
/* backward of the lookup (selection held fixed)                        */
/* ------------------------------------------------------------------ */

/*
 * Gradient of y[t] = sum_h sum_j w[t,h,j] V[idx[t,h,j]] with
 * w = softmax(S), S_j = s1[a_j] + s2[b_j], s_c[a] = sqrt(dh) <u_c, kappa_c[a]>,
 * u_c = q_c / max(||q_c||, eps), kappa_c[a] = K_c[a] / max(||K_c[a]||, eps).
 * The selection (idx) is piecewise constant in the inputs and is held fixed.
 *
 *   dw_j   = <dy_t, V[idx_j]>
 *   dS_j   = w_j (dw_j - sum_l w_l dw_l)
 *   dV[r]  = sum over (t,h,j) with idx = r of w_j dy_t
 *   du_c   = sqrt(dh) sum_j dS_j kappa_c[row_c(j)]
 *   dkap_c[a] = sqrt(dh) sum over (t,h,j) with row_c(j) = a of dS_j u_c
 *   dx     = (dv - v <v, dv>) / max(||x||, eps)  for v = x / max(||x||, eps)
 *            when ||x|| > eps, and dv / eps when the clamp is active.
 *
 * idx holds global row ids; vrow[t*H*k + ...] holds, for each selected slot,
 * the position of that row in the compact table `table` (n_rows rows).
 * dV is accumulated per compact row into dv_out [n_rows, d_v] (may be NULL).
 */
int orc_pkm_backward(int64_t T, int H, int dh, int n, int k, int dv,
                     const void *q, int q_dtype, const void *K, int k_dtype,
                     const void *table, int t_dtype, int64_t n_rows,
                     const int64_t *idx, const int64_t *vrow, const double *w,
                     const void *dy, int dy_dtype, double *dw_out, double *dS_out,
                     double *dq_out, double *dK_out, double *dv_out) {
    const double scale = sqrt((double)dh);
    const int64_t TH = T * H;
    double *kap = unit_subkeys(K, k_dtype, H, n, dh);
    double *uq = (double *)malloc(sizeof(double) * (size_t)TH * 2 * dh);
    double *dkap = (double *)calloc((size_t)H * 2 * n * dh, sizeof(double));
    if (!kap || !uq || !dkap) {
        free(kap);
        free(uq);
        free(dkap);
        return -1;
    }
    int err = 0;

    /* per (t,h): dw, dS, du -> dq */
#pragma omp parallel
    {
        double *du = (double *)malloc(sizeof(double) * dh);
        if (!du) err = -1;
#pragma omp for schedule(dynamic, 4)
        for (int64_t th = 0; th < TH; th++) {
            if (!du) continue;
            int64_t t = th / H;
            int h = (int)(th % H);
            const int64_t *ix = idx + th * k;
            const int64_t *vr = vrow + th * k;
            const double *wj = w + th * k;
            double *dw = dw_out + th * k;
            double *dS = dS_out + th * k;
            double qn[2];
            for (int c = 0; c < 2; c++)
                qn[c] = unit_vector(q, q_dtype, ((t * H + h) * 2 + c) * (int64_t)dh, dh,
                                    uq + (th * 2 + c) * dh);
            double wdw = 0.0;
            for (int j = 0; j < k; j++) {
                if (vr[j] < 0 || vr[j] >= n_rows) {
                    err = -3;
                    dw[j] = 0.0;
                    continue;
                }
                double a = 0.0;
                for (int i = 0; i < dv; i++)
                    a += ld(dy, dy_dtype, t * dv + i) * ld(table, t_dtype, vr[j] * dv + i);
                dw[j] = a;
                wdw += wj[j] * a;
            }
            for (int j = 0; j < k; j++) dS[j] = wj[j] * (dw[j] - wdw);
            for (int c = 0; c < 2; c++) {
                const double *u = uq + (th * 2 + c) * dh;
                for (int i = 0; i < dh; i++) du[i] = 0.0;
                for (int j = 0; j < k; j++) {
                    int64_t a = c == 0 ? ix[j] / n : ix[j] % n;
                    const double *kr = kap + ((int64_t)(h * 2 + c) * n + a) * dh;
                    for (int i = 0; i < dh; i++) du[i] += scale * dS[j] * kr[i];
                }
                double ud = 0.0;
                for (int i = 0; i < dh; i++) ud += u[i] * du[i];
                double *dq = dq_out + (th * 2 + c) * dh;
                if (qn[c] > ORC_NORM_EPS)
                    for (int i = 0; i < dh; i++) dq[i] = (du[i] - u[i] * ud) / qn[c];
                else
                    for (int i = 0; i < dh; i++) dq[i] = du[i] / ORC_NORM_EPS;
            }
        }
        free(du);
    }

    /* sub-key gradients: sequential accumulation in (t, h, j) order */
    for (int64_t th = 0; th < TH; th++) {
        int h = (int)(th % H);
        for (int j = 0; j < k; j++) {
            double g = scale * dS_out[th * k + j];
            for (int c = 0; c < 2; c++) {
                int64_t a = c == 0 ? idx[th * k + j] / n : idx[th * k + j] % n;
                double *dk = dkap + ((int64_t)(h * 2 + c) * n + a) * dh;
                const double *u = uq + (th * 2 + c) * dh;
                for (int i = 0; i < dh; i++) dk[i] += g * u[i];
            }
        }
    }
    /* through the normalisation of each sub-key row */
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < (int64_t)H * 2 * n; r++) {
        double ss = 0.0;
        for (int i = 0; i < dh; i++) {
            double v = ld(K, k_dtype, r * dh + i);
            ss += v * v;
        }
        double nrm = sqrt(ss);
        const double *kr = kap + r * dh;
        const double *g = dkap + r * dh;
        double kd = 0.0;
        for (int i = 0; i < dh; i++) kd += kr[i] * g[i];
        double *o = dK_out + r * dh;
        if (nrm > ORC_NORM_EPS)
            for (int i = 0; i < dh; i++) o[i] = (g[i] - kr[i] * kd) / nrm;
        else
            for (int i = 0; i < dh; i++) o[i] = g[i] / ORC_NORM_EPS;
    }

    /* value-table gradient: sequential accumulation in (t, h, j) order */
    if (dv_out) {
        memset(dv_out, 0, sizeof(double) * (size_t)n_rows * dv);
        for (int64_t th = 0; th < TH; th++) {
            int64_t t = th / H;
            for (int j = 0; j < k; j++) {
                int64_t r = vrow[th * k + j];
                if (r < 0 || r >= n_rows) continue;
                double wj = w[th * k + j];
                double *o = dv_out + r * dv;
                for (int i = 0; i < dv; i++) o[i] += wj * ld(dy, dy_dtype, t * dv + i);
            }
        }
    }
    free(kap);
    free(uq);
    free(dkap);
    return err;
}

int orc_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Value-table gradient of selected rows only: for each requested row id
 * rows[u], out[u] = sum over (t,h,j) with idx[t,h,j] == rows[u] of
 * w[t,h,j] * dy[t], accumulated in (t, h, j) order.
 */
int orc_value_grad_rows(int64_t T, int H, int k, int dv, const int64_t *idx, const double *w,
                        const void *dy, int dy_dtype, const int64_t *rows, int64_t n_rows,
                        double *out) {
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < n_rows; u++) {
        double *o = out + u * dv;
        for (int i = 0; i < dv; i++) o[i] = 0.0;
        for (int64_t s = 0; s < T * H * k; s++) {
            if (idx[s] != rows[u]) continue;
            int64_t t = s / ((int64_t)H * k);
            for (int i = 0; i < dv; i++) o[i] += w[s] * ld(dy, dy_dtype, t * dv + i);
        }
    }
    return err;
}

/* ------------------------------------------------------------------ */
/* Memory+ backward and the query projection                           */
/* ------------------------------------------------------------------ */

/*
 * "Memory Layers at Scale" digest, "Memory+ 블록": out = (y ⊙ silu(x W1)) W2,
 * in row-vector form per token t (a = x W1, g = silu(a), z = y ⊙ g).  Given
 * the gradient dout of out:
 *   dz      = dout W2^T
 *   dy      = dz ⊙ g                      (into the lookup's backward)
 *   da      = dz ⊙ y ⊙ silu'(a),  silu'(a) = s(a) (1 + a (1 - s(a))),  s = sigmoid
 *   dx      = da W1^T
 *   dW1     = sum_t x_t^T da_t,   dW2 = sum_t z_t^T dout_t
 * y is given in double (the bag output); x, W1, W2, dout are decoded exactly.
 */
int orc_memplus_backward(int64_t T, int dm, int dv, const double *y, const void *x,
                         int x_dtype, const void *W1, int w1_dtype, const void *W2,
                         int w2_dtype, const void *dout, int dout_dtype, double *dy_out,
                         double *dx_out, double *dW1_out, double *dW2_out) {
    if (T < 0 || dm < 1 || dv < 1) return -2;
    double *z = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * dv);
    double *da = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * dv);
    if (!z || !da) {
        free(z);
        free(da);
        return -1;
    }
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; t++) {
        for (int v = 0; v < dv; v++) {
            double a = 0.0, dz = 0.0;
            for (int m = 0; m < dm; m++) {
                a += ld(x, x_dtype, t * dm + m) * ld(W1, w1_dtype, (int64_t)m * dv + v);
                dz += ld(dout, dout_dtype, t * dm + m) * ld(W2, w2_dtype, (int64_t)v * dm + m);
            }
            const double s = 1.0 / (1.0 + exp(-a));
            const double yv = y[t * dv + v];
            z[t * dv + v] = yv * a * s;
            dy_out[t * dv + v] = dz * a * s;
            da[t * dv + v] = dz * yv * s * (1.0 + a * (1.0 - s));
        }
        for (int m = 0; m < dm; m++) {
            double acc = 0.0;
            for (int v = 0; v < dv; v++)
                acc += da[t * dv + v] * ld(W1, w1_dtype, (int64_t)m * dv + v);
            dx_out[t * dm + m] = acc;
        }
    }
#pragma omp parallel for schedule(static)
    for (int m = 0; m < dm; m++)
        for (int v = 0; v < dv; v++) {
            double acc = 0.0;
            for (int64_t t = 0; t < T; t++) acc += ld(x, x_dtype, t * dm + m) * da[t * dv + v];
            dW1_out[(int64_t)m * dv + v] = acc;
        }
#pragma omp parallel for schedule(static)
    for (int v = 0; v < dv; v++)
        for (int m = 0; m < dm; m++) {
            double acc = 0.0;
            for (int64_t t = 0; t < T; t++)
                acc += z[t * dv + v] * ld(dout, dout_dtype, t * dm + m);
            dW2_out[(int64_t)v * dm + m] = acc;
        }
    free(z);
    free(da);
    return 0;
}

/* q = x Wq ([T, dm] x [dm, dq]): the query of every head and half from the
   layer input */
int orc_qproj(int64_t T, int dm, int dq, const void *x, int x_dtype, const void *Wq,
              int wq_dtype, double *q_out) {
    if (T < 0 || dm < 1 || dq < 1) return -2;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; t++)
        for (int j = 0; j < dq; j++) {
            double acc = 0.0;
            for (int m = 0; m < dm; m++)
                acc += ld(x, x_dtype, t * dm + m) * ld(Wq, wq_dtype, (int64_t)m * dq + j);
            q_out[t * dq + j] = acc;
        }
    return 0;
}

/* backward of q = x Wq: dWq = sum_t x_t^T dq_t, dx_t = dq_t Wq^T */
int orc_qproj_backward(int64_t T, int dm, int dq, const void *x, int x_dtype, const void *Wq,
                       int wq_dtype, const double *dqv, double *dWq_out, double *dx_out) {
    if (T < 0 || dm < 1 || dq < 1) return -2;
#pragma omp parallel for schedule(static)
    for (int m = 0; m < dm; m++)
        for (int j = 0; j < dq; j++) {
            double acc = 0.0;
            for (int64_t t = 0; t < T; t++) acc += ld(x, x_dtype, t * dm + m) * dqv[t * dq + j];
            dWq_out[(int64_t)m * dq + j] = acc;
        }
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; t++)
        for (int m = 0; m < dm; m++) {
            double acc = 0.0;
            for (int j = 0; j < dq; j++)
                acc += dqv[t * dq + j] * ld(Wq, wq_dtype, (int64_t)m * dq + j);
            dx_out[t * dm + m] = acc;
        }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Engram hashed n-gram lookup ["Conditional Memory via Scalable      */
/* Lookup" review, "희소 검색": multi-head hashing; "핵심 수식" 1 and 2] */
/* ------------------------------------------------------------------ */

/* phi_{n,k}(g): the page names independent hash functions per n-gram order
   and head but not the functions themselves.  This oracle's definition
   (shared with the CUDA path only through this statement, not code):
   h = seed; for each token id x of g, oldest first, taken as 32 unsigned
   bits: h ^= x; h *= 0x9E3779B97F4A7C15 (mod 2^64); h ^= h >> 32.
   The row inside the head's table is h mod M. */
static uint64_t engram_hash(const int32_t *seq, int64_t p, int n, uint64_t seed) {
    uint64_t h = seed;
    for (int i = n - 1; i >= 0; i--) {
        const int64_t q = p - i;
        const uint32_t x = q >= 0 ? (uint32_t)seq[q] : ORC_ENGRAM_PAD;
        h ^= (uint64_t)x;
        h *= 0x9E3779B97F4A7C15ull;
        h ^= h >> 32;
    }
    return h;
}

int orc_engram_rows(int64_t n_seq, int L, const int32_t *tokens, int n_orders,
                    const int *orders, int K, const uint64_t *seeds, const int64_t *M,
                    int64_t *rows_out) {
    if (n_seq < 0 || L < 1 || n_orders < 1 || K < 1) return -2;
    const int HK = n_orders * K;
    int64_t *offset = malloc(sizeof(int64_t) * HK);
    if (!offset) return -1;
    int64_t off = 0;
    for (int j = 0; j < HK; j++) {
        if (M[j] < 1 || orders[j / K] < 1) {
            free(offset);
            return -2;
        }
        offset[j] = off;  /* head j's table starts after the heads before it */
        off += M[j];
    }
#pragma omp parallel for schedule(static)
    for (int64_t s = 0; s < n_seq; s++)
        for (int p = 0; p < L; p++)
            for (int o = 0; o < n_orders; o++)
                for (int k = 0; k < K; k++) {
                    const int j = o * K + k;
                    const uint64_t h = engram_hash(tokens + s * L, p, orders[o], seeds[j]);
                    rows_out[(s * L + p) * HK + j] = offset[j] + (int64_t)(h % (uint64_t)M[j]);
                }
    free(offset);
    return 0;
}

/* e_t = sum over the HK heads of E[row]; the context gate
   alpha_t = sigmoid(<RMSNorm(h_t), RMSNorm(e_t)> / sqrt(d)) with the
   parameter-free RMSNorm x / sqrt(mean(x^2) + eps); v_t = alpha_t e_t. */
int orc_engram_gate(int64_t T, int HK, int d, const int64_t *rows, const void *E, int e_dtype,
                    int64_t n_rows, const void *h, int h_dtype, double eps, double *e_out,
                    double *alpha_out, double *v_out) {
    if (T < 0 || HK < 1 || d < 1) return -2;
    int err = 0;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; t++) {
        double *e = e_out + t * d;
        for (int i = 0; i < d; i++) e[i] = 0.0;
        for (int j = 0; j < HK; j++) {
            const int64_t r = rows[t * HK + j];
            if (r < 0 || r >= n_rows) {
                err = -3;
                continue;
            }
            for (int i = 0; i < d; i++) e[i] += ld(E, e_dtype, r * d + i);
        }
        double hh = 0.0, ee = 0.0, he = 0.0;
        for (int i = 0; i < d; i++) {
            const double hv = ld(h, h_dtype, t * d + i);
            hh += hv * hv;
            ee += e[i] * e[i];
            he += hv * e[i];
        }
        const double rh = sqrt(hh / d + eps), re = sqrt(ee / d + eps);
        const double logit = he / (rh * re) / sqrt((double)d);
        const double a = 1.0 / (1.0 + exp(-logit));
        alpha_out[t] = a;
        for (int i = 0; i < d; i++) v_out[t * d + i] = a * e[i];
    }
    return err;
}
