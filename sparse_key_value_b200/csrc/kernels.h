// kernels.h -- internal launchers of libpkm.so (host side, C++).  Each
// launcher enqueues its kernel(s) on `stream` and returns the launch error.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pkm.h"

namespace pkm {

// Host-side count of kernels this library has launched (instrumentation).
void note_launch(int n = 1);

// Launch `kern` with programmatic stream serialization (it may start while
// the previous kernel of the stream still runs; it calls pdl_wait() before
// touching that kernel's results) when `pdl`, as an ordinary launch otherwise.
template <typename... KArgs, typename... Args>
cudaError_t launch_maybe_pdl(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block,
                             size_t smem, cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Device address of the current device's sticky status word.
int32_t* status_ptr();

// Upper bound of T in every entry point: keeps all size products in range.
constexpr int64_t kMaxTokens = int64_t(1) << 36;

// The forward's argument checks without the workspace (PKM_OK or the error).
pkm_status check_fwd_args(const pkm_fwd_args* a);

// pkm_forward with a library-chosen workspace, and the workspace size it needs.
pkm_status forward_into(const pkm_fwd_args* a, void* workspace, size_t workspace_bytes,
                        cudaStream_t st);
size_t forward_workspace_bytes(const pkm_fwd_args* a);

// r[i] = 1 / max(||x[i, :]||_2, 1e-12) for rows of d elements.
cudaError_t launch_row_rnorm(const void* x, pkm_dtype dt, int64_t rows, int d, float* r,
                             cudaStream_t stream);

// Per-half top-k lists of the sub-key scores, SIMT cores (any dtype, k <= 64).
//   hv/hi [T, H, 2, k]: s_c and the sub-key position a, best first.
cudaError_t launch_score_topk_simt(const void* q, const void* K, pkm_dtype dt, int64_t T,
                                   int H, int dh, int n, int k, const float* rq,
                                   const float* rk, float* hv, int32_t* hi,
                                   cudaStream_t stream);

// Same lists on the tensor cores (tcgen05, bf16, k <= 32).  `splits` > 1
// cuts each sub-key table into that many column ranges, written as
// separate lists hv/hi [splits][T, H, 2, k] that the combine step merges.
bool score_tc_supported(pkm_dtype dt, int dh, int n, int k);
int score_tc_splits(int64_t T, int H, int n);
cudaError_t launch_score_topk_tc(const void* q, const void* K, int64_t T, int H, int dh, int n,
                                 int k, int splits, const float* rq, const float* rk, float* hv,
                                 int32_t* hi, int32_t* status, cudaStream_t stream);

// The whole selection in one kernel for batches of at most 32 tokens
// (k_select_small.cu): sub-key and query norms, scores on the tensor cores,
// per-chunk and per-half top-k, k x k combine, top-k and softmax ->
// idx [T,H,k], w [T,H,k].  bf16, d_half % 64 == 0, 256 <= n, n % 4 == 0,
// at most 32 chunks of 256 columns, k <= 32.  `workspace` holds
// select_small_workspace(T, H, n) bytes (lists and counters).
bool select_small_supported(pkm_dtype dt, int64_t T, int dh, int n, int k);
size_t select_small_workspace(int64_t T, int H, int n);
cudaError_t launch_select_small(const void* q, const void* K, int64_t T, int H, int dh, int n,
                                int k, int32_t* idx, float* w, void* workspace, int32_t* status,
                                cudaStream_t stream);

// The whole selection in one kernel (k_select_tc.cu): query norms, scores
// on the tensor cores, per-half top-k, k x k combine, top-k and softmax ->
// idx [T,H,k], w [T,H,k].  bf16, d_half % 64 == 0, 256 <= n < 65536,
// n % 4 == 0, k <= 32; rk [2H*n + 256] (padded) from launch_row_rnorm;
// `workspace` (select_tc_workspace bytes, 256-aligned) holds the per-half
// lists the two CTAs of a (token tile, head) exchange and their counters.
bool select_tc_supported(pkm_dtype dt, int dh, int n, int k);
size_t select_tc_workspace(int64_t T, int H);
cudaError_t launch_select_tc(const void* q, const void* K, int64_t T, int H, int dh, int n,
                             int k, const float* rk, int32_t* idx, float* w, void* workspace,
                             int32_t* status, cudaStream_t stream);

// Merge the split lists, combine the two halves' k x k candidates, keep the
// top k, softmax -> idx [T,H,k] (a*n+b), w [T,H,k].
cudaError_t launch_combine(const float* hv, const int32_t* hi, int splits, int64_t T, int H,
                           int n, int k, int32_t* idx, float* w, cudaStream_t stream);

// out[t] = sum_j w[t,j] * table[idx[t,j]] (⊙ gate[t]); a persistent grid of
// at most ctas_per_sm CTAs per SM (fewer leave room for concurrent kernels).
cudaError_t launch_embbag_fwd(const void* table, int64_t n_rows, int d, pkm_dtype dt,
                              const int32_t* idx, const float* w, int64_t n_bags, int B,
                              const void* gate, void* out, int32_t* status, cudaStream_t stream,
                              int ctas_per_sm = 4);

// The same gather for small batches (see k_embbag_split.cu): fp32 partial
// sums of row groups in `part` (embbag_split_workspace bytes), then an
// ordered reduction.
// Partial bags of one shard of a row-sharded table: fp32 out [n_bags, d];
// only ids in [row_lo, row_lo + n_local) contribute (read at id - row_lo).
cudaError_t launch_embbag_range(const void* table, int64_t row_lo, int64_t n_local, int d,
                                pkm_dtype dt, const int32_t* idx, const float* w, int64_t n_bags,
                                int B, float* out, cudaStream_t stream);

// pdl: both kernels by programmatic dependent launch (each waits for the
// previous kernel's results before reading idx / w / the partial sums).
constexpr int64_t kSplitGatherMaxBags = 64;
size_t embbag_split_workspace(int64_t n_bags, int B, int d);
cudaError_t launch_embbag_fwd_split(const void* table, int64_t n_rows, int d, pkm_dtype dt,
                                    const int32_t* idx, const float* w, int64_t n_bags, int B,
                                    const void* gate, void* out, float* part, int32_t* status,
                                    cudaStream_t stream, bool pdl = false);

// Memory+ helpers (bf16).
// z = y ⊙ g elementwise (bf16, one rounding)
cudaError_t launch_gate_mul_bf16(const void* y, const void* g, int64_t n, void* z,
                                 cudaStream_t stream);
// dst[c][r] = src[r][c]; dst rows are ld >= rows long, zero past rows (ld <= 0: ld = rows).
cudaError_t launch_transpose_bf16(const void* src, int rows, int cols, void* dst,
                                  cudaStream_t stream, int ld = 0);
// C[M,N] = epi(A[M,K] * B[N,K]^T) in bf16; epi: 0 none, 1 silu.  A is
// [M][K]; B is [N][K], or [K][N] with b_mn (a weight [d_in, d_out] used as x W).
// pdl_mode: 0 ordinary launch; programmatic dependent launch with 1 -- A
// comes from the previous kernel, 2 -- A and B do not (the kernel overlaps
// the previous one and waits for it only before finishing).
// The same GEMMs on CTA pairs (tcgen05 cta_group::2, 256 x 256 tiles);
// cudaErrorNotSupported (nothing launched) when no pair can be resident.
bool gemm_tc2_useful(int64_t M);
cudaError_t launch_gemm_tc2(const void* A, const void* B, int64_t M, int N, int K, int epi,
                            int out_mode, void* C, int32_t* status, cudaStream_t stream,
                            int splits, int64_t c_split, bool a_mn, bool b_mn, int pdl_mode = 0);
bool gemm_tc_supported(int64_t M, int N, int K);
cudaError_t launch_gemm_bf16(const void* A, const void* B, int64_t M, int N, int K, int epi,
                             void* C, int32_t* status, cudaStream_t stream, bool b_mn = false,
                             int pdl_mode = 0);
// C[M,N] (fp32) = A B^T, or C += it when accumulate; A [M][K] or, with a_mn,
// [K][M]; B [N][K] or, with b_mn, [K][N].
cudaError_t launch_gemm_f32(const void* A, const void* B, int64_t M, int N, int K,
                            bool accumulate, float* C, int32_t* status, cudaStream_t stream,
                            bool a_mn = false, bool b_mn = false);
// The same (C overwritten) split over K into slices when the output has few
// tiles (weight gradients contracting over tokens): partial products in
// `part` (gemm_splitk_workspace bytes), summed in slice order.
size_t gemm_splitk_workspace(int64_t M, int N, int K);
cudaError_t launch_gemm_f32_splitk(const void* A, const void* B, int64_t M, int N, int K,
                                   float* C, float* part, int32_t* status, cudaStream_t stream,
                                   bool a_mn = false, bool b_mn = false);

// In-place SGD / touched-rows Adam on the rows of a sparse value gradient
// (see k_sparse_opt.cu); m, v are [n_rows, d] fp32 Adam moments.
cudaError_t launch_sparse_opt(void* table, pkm_dtype dt, int64_t n_rows, int d,
                              const int32_t* rows, const float* grads, const int64_t* count,
                              int64_t cap, bool adam, float* m, float* v, float lr, float b1,
                              float b2, float eps, int64_t step, int32_t* status,
                              cudaStream_t stream);

// ---------------------------------------------------------------- backward
// dw[t,j] = <dy[t], table[idx[t,j]]>; with H>0 also dS = w (dw - sum w dw)
// per (t, h) group of k.
cudaError_t launch_bag_dw(const void* dy, const void* table, int64_t n_rows, int d,
                          pkm_dtype dt, const int32_t* idx, const float* w, int64_t n_bags,
                          int B, int group, float* dw, float* dS, int32_t* status,
                          cudaStream_t stream);

cudaError_t launch_iota(uint32_t* v, int64_t n, cudaStream_t stream);
cudaError_t launch_sanitize_keys(const int32_t* idx, int64_t n, int64_t limit, uint32_t* keys,
                                 int32_t* status, cudaStream_t stream);

// dq of one (token, head) per warp (the query norms computed in the same
// pass): d_half must be a multiple of 32 x (elements per 16 bytes), at most
// 2048.  With `keys` (2 T H k entries) it
// also writes the sub-key gradient's entries (distinct positions per token,
// head and half; the other slots get `mark`) and their coefficients.
bool backward_dh_supported(pkm_dtype dt, int dh);
cudaError_t launch_dq(const void* q, const void* K, pkm_dtype dt, const float* rk,
                      const int32_t* idx, const float* dS, int64_t T, int H, int dh, int n,
                      int k, float* dq, uint32_t mark, uint32_t* keys, float* coef,
                      cudaStream_t stream);
cudaError_t launch_dk_jacobian(const void* K, pkm_dtype dt, const float* rk, int64_t rows, int dh,
                               float* g, cudaStream_t stream);

// Deterministic segmented sums over sorted (key, entry) pairs.  With `table`
// and `dw` (bf16, d a multiple of 256 up to 2048): also dw[entry] =
// <src[entry / div], table[key]>, each segment's table row read once;
// entries with an invalid key get 0.  segsum_has_dw says whether a shape
// takes that path.
size_t segsum_workspace(int64_t n, int d);
bool segsum_has_dw(pkm_dtype dt, int d);
int segsum_dw_slices(int d);  // dw comes as [slices][entries] partial sums
cudaError_t launch_segsum(const uint32_t* skey, const uint32_t* sval, int64_t n, uint32_t mark,
                          const float* coef, const void* src, pkm_dtype dt, int64_t div, int d,
                          int32_t* uniq_rows, float* grad_rows, int64_t cap, int64_t* n_uniq,
                          float* dense_add, float* dense_set, void* workspace, int32_t* status,
                          cudaStream_t stream, const void* table = nullptr, float* dw = nullptr);
// dS = w (dw - sum over the group of w dw), groups of k consecutive entries;
// dw = the sum of `slices` partials [slices][groups * k], in slice order
cudaError_t launch_softmax_bwd(const float* w, const float* dw, int slices, int64_t groups, int k,
                               float* dS, cudaStream_t stream);
cudaError_t launch_scan_exclusive(uint32_t* data, int64_t len, uint32_t* total, int64_t* total64,
                                  cudaStream_t stream);

// Stable LSD radix sort of (key, value) pairs, key < 2^key_bits.
size_t radix_sort_workspace(int64_t n);
cudaError_t launch_radix_sort(const uint32_t* keys_in, const uint32_t* vals_in, int64_t n,
                              int key_bits, uint32_t* keys_out, uint32_t* vals_out,
                              void* workspace, cudaStream_t stream);

}  // namespace pkm
