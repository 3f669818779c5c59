/*
 * pkm_oracle.h -- the CPU oracle's own declarations (test infrastructure
 * only; not part of the CUDA library, which neither includes nor links it).
 *
 * Conventions: tensors are row-major and contiguous.  Inputs tagged with a
 * dtype are decoded exactly to double; every result is double.  Shapes:
 *   q  [T, H, 2, dh]     query, the two halves of each head's query
 *   K  [H, 2, n, dh]     sub-keys: per head and half, n rows of dh
 *   idx/score/w [T, H, k] selected row ids (a*n + b), full scores, weights
 * Return value 0 on success, -1 out of host memory, -2 bad size,
 * -3 a row index out of range (the offending term is skipped).
 */
#ifndef PKM_ORACLE_H
#define PKM_ORACLE_H
#include <stdint.h>

#define ORC_F64 0
#define ORC_F32 1
#define ORC_BF16 2
#define ORC_NORM_EPS 1e-12
#define ORC_ENGRAM_PAD 0xFFFFFFFFu /* token id read before a sequence's start */

#ifdef __cplusplus
extern "C" {
#endif

/* s[t,h,c,a] = sqrt(dh) <q_c/|q_c|, K_c[a]/|K_c[a]|>, out [T,H,2,n] */
int orc_half_scores(int64_t T, int H, int dh, int n, const void *q, int q_dtype,
                    const void *K, int k_dtype, double *s_out);

/* positions of the k largest of s[0..n) (ties: smaller position first) */
int orc_topk(const double *s, int n, int k, int *pos_out);

/* product-key selection: per-half top-k, k*k combine, top-k, softmax.
   *n_half_dots receives the number of half-key dot products evaluated. */
int orc_pkm_select(int64_t T, int H, int dh, int n, int k, const void *q, int q_dtype,
                   const void *K, int k_dtype, int64_t *idx_out, double *score_out,
                   double *w_out, int64_t *n_half_dots);

/* the definition: top-k over all n*n full keys */
int orc_bruteforce_select(int64_t T, int H, int dh, int n, int k, const void *q,
                          int q_dtype, const void *K, int k_dtype, int64_t *idx_out,
                          double *score_out);

/* w = softmax(S) row by row, rows of k */
int orc_softmax(const double *S, int64_t rows, int k, double *w_out);

/* y[t] = sum_j w[t,j] table[idx[t,j]]; table [n_rows, d] */
int orc_bag(int64_t n_bags, int B, int d, const int64_t *idx, const double *w,
            const void *table, int t_dtype, int64_t n_rows, double *y_out);

/* out = (y ⊙ silu(x W1)) W2; x [T,dm], W1 [dm,dv], W2 [dv,dm], y [T,dv] */
int orc_memplus(int64_t T, int dm, int dv, const double *y, const void *x, int x_dtype,
                const void *W1, int w1_dtype, const void *W2, int w2_dtype,
                double *out);

/* backward of the lookup with the selection held fixed; see the .c file */
int orc_pkm_backward(int64_t T, int H, int dh, int n, int k, int dv,
                     const void *q, int q_dtype, const void *K, int k_dtype,
                     const void *table, int t_dtype, int64_t n_rows,
                     const int64_t *idx, const int64_t *vrow, const double *w,
                     const void *dy, int dy_dtype, double *dw_out, double *dS_out,
                     double *dq_out, double *dK_out, double *dv_out);

/* dV rows for the requested row ids only: out [n_rows, dv] */
/* Memory+ backward: given y [T,dv] (double), x [T,dm], W1 [dm,dv],
   W2 [dv,dm] and dout [T,dm]: dy [T,dv], dx [T,dm], dW1 [dm,dv], dW2 [dv,dm] */
int orc_memplus_backward(int64_t T, int dm, int dv, const double *y, const void *x,
                         int x_dtype, const void *W1, int w1_dtype, const void *W2,
                         int w2_dtype, const void *dout, int dout_dtype, double *dy_out,
                         double *dx_out, double *dW1_out, double *dW2_out);

/* query projection q = x Wq, x [T,dm], Wq [dm,dq], q [T,dq] */
int orc_qproj(int64_t T, int dm, int dq, const void *x, int x_dtype, const void *Wq,
              int wq_dtype, double *q_out);

/* its backward: dWq [dm,dq] = x^T dq, dx [T,dm] = dq Wq^T (dq double) */
int orc_qproj_backward(int64_t T, int dm, int dq, const void *x, int x_dtype, const void *Wq,
                       int wq_dtype, const double *dqv, double *dWq_out, double *dx_out);

int orc_value_grad_rows(int64_t T, int H, int k, int dv, const int64_t *idx, const double *w,
                        const void *dy, int dy_dtype, const int64_t *rows, int64_t n_rows,
                        double *out);

/* Engram ("Conditional Memory via Scalable Lookup" review): hashed n-gram
   rows.  tokens [n_seq, L] (ids >= 0); orders [n_orders]; seeds and M
   [n_orders * K] (head j = o*K + k); rows_out [n_seq*L, n_orders*K] are
   global rows of the stacked table (head j's rows after those of heads < j).
   Positions before a sequence's start read the pad id ORC_ENGRAM_PAD. */
int orc_engram_rows(int64_t n_seq, int L, const int32_t *tokens, int n_orders,
                    const int *orders, int K, const uint64_t *seeds, const int64_t *M,
                    int64_t *rows_out);

/* e = sum of the HK rows, alpha = sigmoid(<rms(h), rms(e)>/sqrt(d)), v = alpha e;
   E [n_rows, d], h [T, d]; e_out, v_out [T, d], alpha_out [T] */
int orc_engram_gate(int64_t T, int HK, int d, const int64_t *rows, const void *E, int e_dtype,
                    int64_t n_rows, const void *h, int h_dtype, double eps, double *e_out,
                    double *alpha_out, double *v_out);

int orc_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
