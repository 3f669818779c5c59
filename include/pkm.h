/*
 * pkm.h -- C ABI of libpkm.so, a B200 (sm_100a) implementation of the
 * product-key memory lookup that replaces a transformer FFN, and of its
 * training backward.
 *
 * The method (web pages cited by title and section):
 *  - "Memory Layers at Scale" digest, "Product-key 검색": every key is the
 *    concatenation of two sub-keys, so the top-k of N keys is found with
 *    2*sqrt(N) half-key comparisons instead of N.
 *  - "모델 안의 메모리", "작동 방식" (and figure D): the query is split into
 *    a front and a back half, each half is compared with its table of
 *    sqrt(N) half-keys, the best of each are combined, a few values are read
 *    and averaged with weights; a gate decides how much passes on.
 *  - "Memory Layers at Scale" digest, "Memory+ 블록": gated output
 *    (y ⊙ silu(x W1)) W2; qk-normalization for stability.
 *  - "Memory Layers at Scale" digest, "병렬 EmbeddingBag 구현": the layer is
 *    bound by memory bandwidth; its core is a weighted EmbeddingBag.
 *
 * Readings where the pages are silent (fixed by this library):
 *  - qk-normalization: each query half and each sub-key row is divided by
 *    max(||.||_2, 1e-12); half score s_c[a] = sqrt(d_half) * <q_c, K_c[a]>
 *    of the normalised vectors.
 *  - full score S(a, b) = s_1[a] + s_2[b]; value row id = a * n_sub + b.
 *  - weights: softmax over the k selected full scores.
 *  - heads: each head h has its own sub-key tables; all heads share one
 *    value table; the H bags of a token are summed into one output row.
 *  - order: larger score first.  Scores that are exactly equal in fp32 are
 *    ties: the bf16 tensor-core selections (d_half % 64 == 0, k <= 32) may
 *    keep either and list them in either order; the other paths put the
 *    smaller id first.
 *
 * Conventions for every entry point:
 *  - Device pointers are caller-owned, row-major, contiguous and 16-byte
 *    aligned.  Host pointers are named so.  The library never allocates or
 *    frees device memory; scratch comes from the caller's workspace.
 *  - Work is enqueued on `stream` (a cudaStream_t); nothing synchronises
 *    except pkm_get_device_error.
 *  - Arguments are validated on the host before any launch; an invalid call
 *    returns an error and launches nothing.
 *  - Anomalies found on the device (an out-of-range row id, a spin-wait that
 *    ran out, a sparse-output overflow) never trap: the offending work is
 *    skipped and a sticky per-device status word records the first one; read
 *    and clear it with pkm_get_device_error.
 *  - dtype applies to query, sub-keys, values, x, W1, W2, dy and out.
 *    Row ids are int32, weights and gradients fp32.
 */
#ifndef PKM_H
#define PKM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PKM_API __attribute__((visibility("default")))
#else
#define PKM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *pkm_stream_t; /* identical to cudaStream_t */

typedef enum {
    PKM_OK = 0,
    PKM_ERR_INVALID_ARG = 1, /* bad size, null or misaligned pointer */
    PKM_ERR_UNSUPPORTED = 2, /* valid but not implemented combination */
    PKM_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
    PKM_ERR_DEVICE = 4,      /* device status: out-of-range row id or overflow */
    PKM_ERR_TIMEOUT = 5,     /* device status: a bounded spin-wait ran out */
    PKM_ERR_WORKSPACE = 6    /* workspace missing or too small */
} pkm_status;

typedef enum { PKM_F32 = 0, PKM_BF16 = 1 } pkm_dtype;

/*
 * Forward of one memory layer.
 *
 *   query   [T, H, 2, d_half]      the two halves of each head's query
 *   subkeys [H, 2, n_sub, d_half]  per head, the half-key tables of both halves
 *   values  [n_sub*n_sub, d_v]     the value table (N = n_sub^2 rows)
 *   idx     [T, H, k]  out: selected row ids a*n_sub+b, best first
 *   weights [T, H, k]  out: softmax weights of the selected rows
 *   out     [T, d_v]   y[t] = sum_h sum_j weights[t,h,j] * values[idx[t,h,j]]
 *           or, with Memory+ (x, W1, W2 all non-NULL), [T, d_model]
 *           out = (y ⊙ silu(x W1)) W2 with x [T, d_model], W1 [d_model, d_v],
 *           W2 [d_v, d_model] (bf16 only).
 *
 * Limits: 1 <= k <= min(n_sub, 64); d_half, d_v, d_model multiples of 8;
 * n_sub*n_sub < 2^31; 0 <= T <= 2^36 (PKM_ERR_INVALID_ARG otherwise).
 * T = 0 is a valid empty call.
 */
typedef struct {
    int64_t T;
    int32_t H, d_half, n_sub, k, d_v;
    pkm_dtype dtype;
    const void *query;
    const void *subkeys;
    const void *values;
    const void *x; /* Memory+ gate input, or NULL */
    const void *W1;
    const void *W2;
    int32_t d_model;
    void *out;
    int32_t *idx;
    float *weights;
    void *workspace; /* device scratch of pkm_forward_workspace_size bytes */
    size_t workspace_bytes;
    /* Optional instrumentation: NULL, or PKM_FWD_N_EVENTS cudaEvent_t
       handles (host array) recorded at the phase boundaries:
       [0] start, [1] after the norms, [2] after scoring + per-half top-k,
       [3] after combine + softmax, [4] before the bag gather (after the
       Memory+ gate GEMM), [5] after the bag gather, [6] end (after the
       Memory+ output GEMM).  When the selection runs as one kernel (bf16,
       d_half % 64 == 0, 256 <= n_sub < 65536, n_sub % 4 == 0, k <= 32, and
       T > 64, or T <= 32 with n_sub <= 8192), [2] = [3] follow the whole
       selection and [1] follows the sub-key norms (T > 64) or equals [0]
       (T <= 32: the kernel computes them too).  Under stream capture the events are recorded as
       external event nodes of the graph, so every replay records them. */
    void **phase_events;
    /* Optional, Memory+ only: NULL, or [T, d_v] (dtype) receiving the bag
       output y before the gate, as pkm_memplus_backward needs it.  With it
       the gate product is applied in a separate pass (y rounded to the
       dtype first), otherwise fused into the gather. */
    void *y_out;
} pkm_fwd_args;

#define PKM_FWD_N_EVENTS 7

/*
 * pkm_forward_noalloc: the same forward for callers that cannot allocate
 * device memory (a C program linking only this library with no allocator,
 * a runtime whose memory budget is fixed at start-up, a serving loop that
 * must not call the synchronising cudaMalloc).  There is no counterpart on
 * the source pages: it is a service of this library.
 *
 * Arguments as for pkm_forward; `workspace` and `workspace_bytes` are
 * ignored.  The scratch is a fixed 32 MiB array inside the library on each
 * device (held by every device that loads the library until exit); calls
 * whose pkm_forward_workspace_size exceeds 32 MiB return PKM_ERR_WORKSPACE
 * and launch nothing.  The first call on a device looks up the array's
 * address on that device (make that first call before any stream capture).
 * All calls share the array: calls whose GPU work overlaps race.  Nothing is
 * allocated or freed.
 */
PKM_API pkm_status pkm_forward_noalloc(const pkm_fwd_args *args, pkm_stream_t stream);

/* Bytes of device workspace pkm_forward needs for these sizes (pointers
   are not read). */
PKM_API size_t pkm_forward_workspace_size(const pkm_fwd_args *args);

/* Enqueue the forward on `stream`. */
PKM_API pkm_status pkm_forward(const pkm_fwd_args *args, pkm_stream_t stream);

/*
 * The selection alone (norms, sub-key scores, per-half top-k, k x k combine,
 * softmax): writes idx and weights as pkm_forward does; values, out, x, W1,
 * W2, y_out and d_model are ignored (d_v is only validated).  The workspace
 * is that of pkm_forward for the same arguments.  It is the first step of a
 * lookup whose value table is sharded by rows across GPUs: every rank
 * selects for its own tokens with the replicated sub-keys, the selections
 * are exchanged and each rank gathers the rows it holds
 * (embbag_forward_range).
 */
PKM_API pkm_status pkm_select(const pkm_fwd_args *args, pkm_stream_t stream);

/*
 * Backward of the plain lookup (out = y), selection held fixed (top-k is
 * piecewise constant).  With w = softmax(S):
 *   dw_j      = <dy_t, values[idx_j]>
 *   dS_j      = w_j (dw_j - sum_l w_l dw_l)
 *   dvalues[r]= sum over (t,h,j) with idx = r of w_j dy_t
 *   dquery, dsubkeys: dS through S = s_1[a] + s_2[b] and the normalisation.
 *
 *   idx, weights  [T, H, k]  as written by pkm_forward
 *   dy            [T, d_v]   upstream gradient (dtype)
 *   dquery        [T, H, 2, d_half] fp32 out (overwritten)
 *   dsubkeys      [H, 2, n_sub, d_half] fp32 out (overwritten)
 *   value gradient, sparse: uniq_rows int32 [uniq_cap] (ascending row ids),
 *       grad_rows fp32 [uniq_cap, d_v], *n_uniq (device int64) = rows
 *       written; uniq_cap >= T*H*k always suffices.  Rows beyond the cap
 *       are dropped and the device status is set to PKM_ERR_DEVICE.
 *   and/or dense: dvalues_dense fp32 [n_sub^2, d_v] receives += per row.
 *   Either may be NULL (not both).  dscores [T,H,k] fp32 (optional) gets dS.
 * Every sum runs in a fixed order: results are bitwise reproducible.
 *
 * Streams: when dw comes from a per-slot re-gather of the value rows (more
 * slots than a quarter of the table rows), the value-gradient sort and
 * segmented sum run on a library-owned stream of the current device, forked
 * from `stream` by an event and joined back to it by another before the
 * call's last work item, so every output is ordered on `stream` as usual.
 * While `stream` is being captured into a CUDA graph all work stays on it.
 *
 * Limits beyond the forward's: d_half a multiple of 256 (bf16) or 128 (fp32)
 * and at most 2048 (one warp holds a query half in registers, 16 bytes per
 * lane per step); T*H*k*2 < 2^32.  Other sizes return PKM_ERR_UNSUPPORTED
 * and launch nothing.
 */
typedef struct {
    int64_t T;
    int32_t H, d_half, n_sub, k, d_v;
    pkm_dtype dtype;
    const void *query;
    const void *subkeys;
    const void *values;
    const int32_t *idx;
    const float *weights;
    const void *dy;
    float *dquery;
    float *dsubkeys;
    int32_t *uniq_rows;
    float *grad_rows;
    int64_t *n_uniq;
    int64_t uniq_cap;
    float *dvalues_dense;
    float *dscores;
    void *workspace;
    size_t workspace_bytes;
} pkm_bwd_args;

PKM_API size_t pkm_backward_workspace_size(const pkm_bwd_args *args);
PKM_API pkm_status pkm_backward(const pkm_bwd_args *args, pkm_stream_t stream);

/*
 * Partial bags over one shard of a table sharded by rows ("Memory Layers at
 * Scale" digest: memories of 64B and 128B parameters exceed one GPU): the
 * shard holds rows [row_lo, row_lo + n_local) of the full table as its own
 * [n_local, d] table.
 *   out[t] = sum over j with row_lo <= idx[t,j] < row_lo + n_local of
 *            w[t,j] * table[idx[t,j] - row_lo]
 *   idx int32 / w fp32 [n_bags, B] (full-table ids), out fp32 [n_bags, d].
 * Ids outside the shard contribute nothing and are not an error (another
 * shard holds them).  fp32 accumulation in j order, no rounding, so the
 * shards' partials sum (in shard order) to the full bag up to the order of
 * fp32 additions.
 */
PKM_API pkm_status embbag_forward_range(const void *table, int64_t row_lo, int64_t n_local,
                                        int32_t d, pkm_dtype dtype, const int32_t *idx,
                                        const float *w, int64_t n_bags, int32_t B, float *out,
                                        pkm_stream_t stream);

/*
 * Generic weighted bags ("병렬 EmbeddingBag 구현"):
 *   out[t] = (sum_j w[t,j] * table[idx[t,j]]) [⊙ gate[t]]
 *   table [n_rows, d] (dtype), idx int32 / w fp32 [n_bags, B],
 *   gate NULL or [n_bags, d] (dtype), out [n_bags, d] (dtype).
 * Accumulation is fp32 in j order, one rounding at the store.  A row id
 * outside [0, n_rows) is skipped and sets the device status.
 */
PKM_API pkm_status embbag_forward(const void *table, int64_t n_rows, int32_t d, pkm_dtype dtype,
                          const int32_t *idx, const float *w, int64_t n_bags, int32_t B,
                          const void *gate, void *out, pkm_stream_t stream);

/*
 * Backward of embbag_forward without gate:
 *   dw[t,j]  = <dy[t], table[idx[t,j]]>          (if table and dw non-NULL)
 *   grad[r]  = sum over (t,j) with idx = r of w[t,j] dy[t]
 * written sparse (uniq_rows/grad_rows/n_uniq as in pkm_bwd_args) and/or
 * added into dense_accum [n_rows, d].  Deterministic sorted reduction.
 */
PKM_API size_t embbag_backward_workspace_size(int64_t n_bags, int32_t B, int32_t d, int64_t n_rows);
PKM_API pkm_status embbag_backward(const void *dy, const int32_t *idx, const float *w,
                           int64_t n_bags, int32_t B, int32_t d, pkm_dtype dtype,
                           const void *table, int64_t n_rows, float *dw,
                           int32_t *uniq_rows, float *grad_rows, int64_t *n_uniq,
                           int64_t uniq_cap, float *dense_accum, void *workspace,
                           size_t workspace_bytes, pkm_stream_t stream);

/* Synchronise `stream`, then read and clear this device's sticky status
   word into *code (a pkm_status value; PKM_OK when nothing happened). */
PKM_API pkm_status pkm_get_device_error(pkm_stream_t stream, int32_t *code);

/* Static description of a status code. */
PKM_API const char *pkm_status_string(pkm_status status);

/* Library version: major*10000 + minor*100 + patch. */
PKM_API int32_t pkm_version(void);

/* Instrumentation: number of kernels this process has launched through the
   library so far (host-side counter, all devices). */
PKM_API uint64_t pkm_launch_count(void);

/*
 * Memory+ backward ("Memory Layers at Scale" digest, "Memory+ 블록": out =
 * (y ⊙ silu(x W1)) W2).  Row-vector form per token, a = x W1, g = silu(a):
 *   dz  = dout W2^T,          dy  = dz ⊙ g   (the lookup's upstream gradient)
 *   da  = dz ⊙ y ⊙ silu'(a),  dx  = da W1^T
 *   dW1 = x^T da,             dW2 = (y ⊙ g)^T dout
 * No counterpart in the sources beyond the forward they give; the formulas
 * are its derivatives.  All of x, W1, W2, y, dout are bf16.
 *
 *   x [T, d_model], W1 [d_model, d_v], W2 [d_v, d_model]  the forward's inputs
 *   y    [T, d_v]      the bag output (pkm_fwd_args.y_out of the forward)
 *   dout [T, d_model]  gradient of out
 *   dy   [T, d_v]      out (bf16): gradient of y, the dy of pkm_backward
 *   dx   [T, d_model]  out (fp32), overwritten
 *   dW1  [d_model, d_v], dW2 [d_v, d_model]  out (fp32)
 * Limits: d_model, d_v multiples of 8.  T = 0 is a valid empty call (the
 * weight gradients are then zero).
 */
typedef struct {
    int64_t T;
    int32_t d_model, d_v;
    const void *x;
    const void *W1;
    const void *W2;
    const void *y;
    const void *dout;
    void *dy;
    float *dx;
    float *dW1;
    float *dW2;
    void *workspace; /* device scratch of pkm_memplus_backward_workspace_size bytes */
    size_t workspace_bytes;
} pkm_memplus_bwd_args;

PKM_API size_t pkm_memplus_backward_workspace_size(const pkm_memplus_bwd_args *args);
PKM_API pkm_status pkm_memplus_backward(const pkm_memplus_bwd_args *args, pkm_stream_t stream);

/*
 * Query projection q = x Wq that feeds the lookup from the layer input
 * (the query of every head and half, d_q = H * 2 * d_half), and its
 * backward.  bf16 x [T, d_model], Wq [d_model, d_q].
 *   pkm_qproj_forward:  q [T, d_q] (bf16) out.
 *   pkm_qproj_backward: dq [T, d_q] (fp32, pkm_bwd_args.dquery) in;
 *                       dWq [d_model, d_q] (fp32) out; dx [T, d_model]
 *                       (fp32) += dq Wq^T (accumulates onto, e.g., the dx of
 *                       pkm_memplus_backward).
 * Limits: d_model, d_q multiples of 8.
 */
typedef struct {
    int64_t T;
    int32_t d_model, d_q;
    const void *x;
    const void *Wq;
    void *q;
    const float *dq;
    float *dWq;
    float *dx;
    void *workspace; /* device scratch of pkm_qproj_workspace_size bytes */
    size_t workspace_bytes;
} pkm_qproj_args;

PKM_API size_t pkm_qproj_workspace_size(const pkm_qproj_args *args);
PKM_API pkm_status pkm_qproj_forward(const pkm_qproj_args *args, pkm_stream_t stream);
PKM_API pkm_status pkm_qproj_backward(const pkm_qproj_args *args, pkm_stream_t stream);

/*
 * Optimiser step on the touched value rows only ("모델 안의 메모리", "잊지 않고
 * 배우기": a fact occupies a few memory slots, so only those are updated).
 * The rows and gradients are pkm_backward's sparse value gradient
 * (uniq_rows, grad_rows, n_uniq); each row is updated in place by one CTA:
 *   PKM_OPT_SGD   p -= lr * g
 *   PKM_OPT_ADAM  m = beta1 m + (1-beta1) g;  v = beta2 v + (1-beta2) g^2;
 *                 p -= lr * (m / c1) / (sqrt(v / c2) + eps),  c = 1 - beta^step;
 *                 the moments of untouched rows are left as they are.
 * bf16 tables are updated in fp32 and rounded once (nearest even).
 *   table [n_rows, d] (dtype), rows [cap] distinct ids, grads [cap, d] fp32,
 *   count device int64 (entries used: min(*count, cap); more sets
 *   PKM_ERR_DEVICE), m, v [n_rows, d] fp32 (Adam only).
 * Limits: d a multiple of 8; Adam: 0 <= beta < 1, eps >= 0, step >= 1.
 */
typedef enum { PKM_OPT_SGD = 0, PKM_OPT_ADAM = 1 } pkm_opt_kind;

typedef struct {
    pkm_opt_kind kind;
    float lr, beta1, beta2, eps;
    int64_t step;
    int64_t n_rows;
    int32_t d;
    pkm_dtype dtype;
    void *table;
    const int32_t *rows;
    const float *grads;
    const int64_t *count;
    int64_t cap;
    float *m;
    float *v;
} pkm_sparse_opt_args;

PKM_API pkm_status pkm_sparse_optimizer_step(const pkm_sparse_opt_args *args, pkm_stream_t stream);

/*
 * Engram lookup ("Conditional Memory via Scalable Lookup" review, "희소 검색"
 * and "핵심 수식" 1-2): hashed n-gram rows, their sum and the context gate.
 * For token t = s*L + p of sequence s and head j = o*K + k (n = orders[o]):
 *   g      = tokens[s, p-n+1 .. p], positions before 0 read the pad id
 *            0xFFFFFFFF; ids are taken as 32 unsigned bits
 *   hash   h = seeds[j]; for each id x of g, oldest first:
 *            h ^= x; h *= 0x9E3779B97F4A7C15 (mod 2^64); h ^= h >> 32
 *   row    = offset_j + h mod rows_per_head[j], offset_j the sum of
 *            rows_per_head of the heads before j (the heads' tables are
 *            stacked in one table)
 *   e_t    = sum over the heads of table[row]          (fp32, head order)
 *   alpha_t = sigmoid(<RMSNorm(h_t), RMSNorm(e_t)> / sqrt(d)),
 *            RMSNorm(x) = x / sqrt(mean(x^2) + 1e-6)  (no learned scale)
 *   v_t    = alpha_t e_t                                (one rounding)
 * The page names independent hash functions per order and head but not
 * the functions; the one above is this library's definition.
 *   tokens [n_seq, L] int32 (device), table [sum rows_per_head, d], h and v
 *   [T, d] (dtype, device); optional outputs (NULL to skip): alpha [T] fp32,
 *   rows [T, heads] int32, e [T, d] (dtype).  orders, seeds and
 *   rows_per_head are HOST arrays read during the call.
 * Limits: 1 <= n_orders <= 8, orders in 1..8, heads = n_orders*K <= 64,
 * rows_per_head >= 1 with their sum < 2^31, d a multiple of 8 with
 * d <= 8192 (bf16) or 4096 (fp32).  Nothing is allocated; no workspace.
 */
#define PKM_ENGRAM_MAX_ORDERS 8
#define PKM_ENGRAM_MAX_HEADS 64

typedef struct {
    int64_t n_seq;
    int32_t L;
    int32_t n_orders;
    int32_t K;
    const int32_t *orders;        /* host [n_orders] */
    const uint64_t *seeds;        /* host [n_orders * K] */
    const int64_t *rows_per_head; /* host [n_orders * K] */
    int32_t d;
    pkm_dtype dtype;
    const int32_t *tokens;
    const void *table;
    const void *h;
    void *v;
    float *alpha;
    int32_t *rows;
    void *e;
} pkm_engram_args;

PKM_API pkm_status pkm_engram_forward(const pkm_engram_args *args, pkm_stream_t stream);

/*
 * Failure-path check of the bounded waits (no counterpart on the pages; a
 * service for tests and operators): one CTA waits, with the wait every
 * pipelined kernel of the library uses, on an mbarrier phase that nothing
 * completes.  After `polls` polls (1 .. 2^20) the wait gives up, the device
 * status word records PKM_ERR_TIMEOUT (read it with pkm_get_device_error)
 * and the kernel returns, writing 1 to *done (device int32; 2 would mean the
 * phase completed, which cannot happen).  No GPU fault is involved and the
 * context stays usable.
 */
PKM_API pkm_status pkm_check_wait_timeout(int64_t polls, int32_t *done, pkm_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* PKM_H */
