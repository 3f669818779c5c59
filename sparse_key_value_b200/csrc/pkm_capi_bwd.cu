// pkm_capi_bwd.cu -- C ABI of the backward entry points: validation,
// workspace carving and the launch sequence (see include/pkm.h).
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace pkm {
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t round_up(size_t x) { return (x + 255) / 256 * 256; }

int bits_for(uint64_t max_value) {  // bits needed to hold values 0..max_value
  int b = 1;
  while (b < 32 && (max_value >> b) != 0) ++b;
  return b;
}

struct BwdLayout {
  size_t rk, dS, dwp, iota, skeys, svals, ekeys, ecoef, radix, seg;
  // the value-gradient branch's own sort and segment buffers when it runs
  // beside the rest of the backward (see backward_impl)
  size_t vkeys, vskeys, vsvals, vradix, vseg, total;
};

// dw = <dy, V[idx]> from the value-gradient walk (each distinct value row
// read once) instead of a per-slot re-gather of the value rows: for batches
// with few slots per table row -- rows then rarely repeat; with many slots per
// row (R > N/4) the repeated rows make the re-gather cheap in L2 and the plain
// walk faster (measured: Memory+ shapes 3.78 ms against 4.28 ms, PKM training
// shapes 2.31 ms against 1.73 ms)
bool fused_value_dw(pkm_dtype dt, int d_v, size_t R, size_t N) {
  return segsum_has_dw(dt, d_v) && 4 * R <= N;
}

BwdLayout bwd_layout(const pkm_bwd_args* a) {
  BwdLayout L{};
  const size_t T = (size_t)(a->T > 0 ? a->T : 0), H = (size_t)a->H, n = (size_t)a->n_sub,
               k = (size_t)a->k;
  const size_t R = T * H * k, R2 = 2 * R;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += round_up(bytes);
    return o;
  };
  L.rk = take(H * 2 * n * 4);
  L.dS = take(R * 4);
  // partial dot products dw [slices][R] of the value-gradient walk
  const bool fused = fused_value_dw(a->dtype, a->d_v, R, n * n);
  L.dwp = fused ? take((size_t)segsum_dw_slices(a->d_v) * R * 4) : 0;
  L.iota = take(R2 * 4);
  L.skeys = take(R2 * 4);
  L.svals = take(R2 * 4);
  L.ekeys = take(R2 * 4);
  L.ecoef = take(R2 * 4);
  L.radix = take(radix_sort_workspace((int64_t)R2));
  const size_t s1 = segsum_workspace((int64_t)R, a->d_v);
  const size_t s2 = segsum_workspace((int64_t)R2, a->d_half);
  if (fused) {  // one branch: the buffers are shared in turn
    L.seg = take(s1 > s2 ? s1 : s2);
  } else {
    L.seg = take(s2);
    L.vkeys = take(R * 4);
    L.vskeys = take(R * 4);
    L.vsvals = take(R * 4);
    L.vradix = take(radix_sort_workspace((int64_t)R));
    L.vseg = take(s1);
  }
  L.total = off;
  return L;
}

pkm_status validate_bwd(const pkm_bwd_args* a) {
  if (!a) return PKM_ERR_INVALID_ARG;
  if (a->T < 0 || a->T > kMaxTokens || a->H < 1 || a->n_sub < 1 || a->k < 1 || a->k > 64 ||
      a->k > a->n_sub)
    return PKM_ERR_INVALID_ARG;
  if (a->d_half < 8 || a->d_half % 8 || a->d_v < 8 || a->d_v % 8) return PKM_ERR_INVALID_ARG;
  if ((int64_t)a->n_sub * a->n_sub >= (int64_t(1) << 31)) return PKM_ERR_INVALID_ARG;
  if (a->dtype != PKM_F32 && a->dtype != PKM_BF16) return PKM_ERR_INVALID_ARG;
  if ((int64_t)a->H * a->k > 4096) return PKM_ERR_INVALID_ARG;
  if (!backward_dh_supported(a->dtype, a->d_half)) return PKM_ERR_UNSUPPORTED;
  if (a->T * a->H * a->k * 2 >= (int64_t(1) << 32)) return PKM_ERR_UNSUPPORTED;
  if (a->T == 0) return PKM_OK;
  const void* need[] = {a->query, a->subkeys, a->values, a->idx, a->weights, a->dy,
                        a->dquery, a->dsubkeys};
  for (const void* p : need)
    if (!p || !aligned16(p)) return PKM_ERR_INVALID_ARG;
  const bool sparse = a->grad_rows != nullptr;
  if (!sparse && !a->dvalues_dense) return PKM_ERR_INVALID_ARG;
  if (sparse && (!a->uniq_rows || !a->n_uniq || a->uniq_cap < 0 || !aligned16(a->grad_rows)))
    return PKM_ERR_INVALID_ARG;
  if (a->dvalues_dense && !aligned16(a->dvalues_dense)) return PKM_ERR_INVALID_ARG;
  if (!a->workspace || !aligned16(a->workspace) || a->workspace_bytes < bwd_layout(a).total)
    return PKM_ERR_WORKSPACE;
  return PKM_OK;
}

#define PKM_TRY(expr)                           \
  do {                                          \
    cudaError_t e_ = (expr);                    \
    if (e_ != cudaSuccess) return PKM_ERR_CUDA; \
  } while (0)

// The library's second stream on the current device (created once), where
// the backward runs its value-gradient branch beside the rest; null -- the
// branch then runs in line -- while `st` is being captured into a graph or
// if the stream cannot be created.
cudaStream_t side_stream(cudaStream_t st) {
  static cudaStream_t streams[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone)
    return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!streams[dev]) {
    cudaStream_t s = nullptr;
    if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    streams[dev] = s;
  }
  return streams[dev];
}

pkm_status backward_impl(const pkm_bwd_args* a, cudaStream_t st) {
  int32_t* status = status_ptr();
  if (!status) return PKM_ERR_CUDA;
  const BwdLayout L = bwd_layout(a);
  char* ws = static_cast<char*>(a->workspace);
  float* rk = reinterpret_cast<float*>(ws + L.rk);
  float* dS = a->dscores ? a->dscores : reinterpret_cast<float*>(ws + L.dS);
  float* dwp = reinterpret_cast<float*>(ws + L.dwp);
  uint32_t* iota = reinterpret_cast<uint32_t*>(ws + L.iota);
  uint32_t* skeys = reinterpret_cast<uint32_t*>(ws + L.skeys);
  uint32_t* svals = reinterpret_cast<uint32_t*>(ws + L.svals);
  uint32_t* ekeys = reinterpret_cast<uint32_t*>(ws + L.ekeys);
  float* ecoef = reinterpret_cast<float*>(ws + L.ecoef);
  void* radix = ws + L.radix;
  void* seg = ws + L.seg;
  const int64_t T = a->T;
  const int H = a->H, dh = a->d_half, n = a->n_sub, k = a->k, dv = a->d_v;
  const int64_t N = (int64_t)n * n, R = T * H * k;

  PKM_TRY(launch_iota(iota, 2 * R, st));
  // value gradient: sort the (row, slot) pairs, then segmented sums of w * dy;
  // dw and the softmax backward dS from the same walk where fused_value_dw
  // says so.  Otherwise dS comes from a per-slot re-gather of the value rows,
  // and the value-gradient branch (sort + walk, its own buffers) needs
  // nothing the rest of the backward computes: it runs on the library's
  // second stream beside the re-gather and the query and sub-key gradients,
  // and the caller's stream waits for it at the end.
  const bool fused_dw = fused_value_dw(a->dtype, dv, (size_t)R, (size_t)N);
  // the caller's stream waits for the side branch on every way out
  struct SideJoin {
    cudaStream_t st = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    bool pending = false;  // join recorded on the side stream, not yet waited for
    cudaError_t finish() {
      const cudaError_t e = pending ? cudaStreamWaitEvent(st, join, 0) : cudaSuccess;
      pending = false;
      return e;
    }
    ~SideJoin() {
      finish();
      if (fork) cudaEventDestroy(fork);
      if (join) cudaEventDestroy(join);
    }
  } sj;
  sj.st = st;
  cudaStream_t vst = st;
  if (!fused_dw) {
    cudaStream_t side = side_stream(st);
    if (side && cudaEventCreateWithFlags(&sj.fork, cudaEventDisableTiming) == cudaSuccess &&
        cudaEventCreateWithFlags(&sj.join, cudaEventDisableTiming) == cudaSuccess &&
        cudaEventRecord(sj.fork, st) == cudaSuccess &&
        cudaStreamWaitEvent(side, sj.fork, 0) == cudaSuccess)
      vst = side;
  }
  uint32_t* vkeys = fused_dw ? ekeys : reinterpret_cast<uint32_t*>(ws + L.vkeys);
  uint32_t* vskeys = fused_dw ? skeys : reinterpret_cast<uint32_t*>(ws + L.vskeys);
  uint32_t* vsvals = fused_dw ? svals : reinterpret_cast<uint32_t*>(ws + L.vsvals);
  void* vradix = fused_dw ? radix : ws + L.vradix;
  void* vseg = fused_dw ? seg : ws + L.vseg;
  cudaError_t ve = launch_sanitize_keys(a->idx, R, N, vkeys, status, vst);
  if (ve == cudaSuccess)
    ve = launch_radix_sort(vkeys, iota, R, bits_for((uint64_t)N), vskeys, vsvals, vradix, vst);
  if (ve == cudaSuccess)
    ve = launch_segsum(vskeys, vsvals, R, (uint32_t)N, a->weights, a->dy, a->dtype,
                       (int64_t)H * k, dv, a->uniq_rows, a->grad_rows,
                       a->grad_rows ? a->uniq_cap : 0, a->n_uniq, a->dvalues_dense, nullptr, vseg,
                       status, vst, fused_dw ? a->values : nullptr, fused_dw ? dwp : nullptr);
  if (vst != st) {
    if (cudaEventRecord(sj.join, vst) == cudaSuccess) {
      sj.pending = true;
    } else {  // no event to wait on: let the side branch finish before returning
      cudaStreamSynchronize(vst);
      return PKM_ERR_CUDA;
    }
  }
  if (ve != cudaSuccess) return PKM_ERR_CUDA;
  if (fused_dw)
    PKM_TRY(launch_softmax_bwd(a->weights, dwp, segsum_dw_slices(dv), T * H, k, dS, st));
  else
    PKM_TRY(launch_bag_dw(a->dy, a->values, N, dv, a->dtype, a->idx, a->weights, T, H * k, k,
                          nullptr, dS, status, st));
  // the sub-keys' normalisation factors (recomputed; the query's come with dq)
  PKM_TRY(launch_row_rnorm(a->subkeys, a->dtype, (int64_t)H * 2 * n, dh, rk, st));
  // query gradient, and the sub-key gradient's entries per distinct (head,
  // half, sub-key) and token in the same pass; then the entries sorted,
  // summed into the dense output, and the normalisation Jacobian
  const uint32_t mark = (uint32_t)(2 * H * n);
  PKM_TRY(launch_dq(a->query, a->subkeys, a->dtype, rk, a->idx, dS, T, H, dh, n, k, a->dquery,
                    mark, ekeys, ecoef, st));
  PKM_TRY(launch_radix_sort(ekeys, iota, 2 * R, bits_for(mark), skeys, svals, radix, st));
  PKM_TRY(cudaMemsetAsync(a->dsubkeys, 0, sizeof(float) * (size_t)H * 2 * n * dh, st));
  PKM_TRY(launch_segsum(skeys, svals, 2 * R, mark, ecoef, a->query, a->dtype, k, dh, nullptr,
                        nullptr, 0, nullptr, nullptr, a->dsubkeys, seg, status, st));
  PKM_TRY(launch_dk_jacobian(a->subkeys, a->dtype, rk, (int64_t)H * 2 * n, dh, a->dsubkeys, st));
  PKM_TRY(sj.finish());
  return PKM_OK;
}

size_t embbag_bwd_bytes(int64_t n_bags, int32_t B, int32_t d, int64_t n_rows, size_t* parts) {
  const size_t R = (size_t)(n_bags > 0 ? n_bags : 0) * (size_t)(B > 0 ? B : 0);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += round_up(bytes);
    return o;
  };
  parts[0] = take(R * 4);  // iota
  parts[1] = take(R * 4);  // sorted keys
  parts[2] = take(R * 4);  // sorted values
  parts[3] = take(radix_sort_workspace((int64_t)R));
  parts[4] = take(segsum_workspace((int64_t)R, d > 0 ? d : 8));
  parts[5] = take(R * 4);  // range-checked keys
  (void)n_rows;
  return off;
}

}  // namespace
}  // namespace pkm

using namespace pkm;

extern "C" {

size_t pkm_backward_workspace_size(const pkm_bwd_args* args) {
  if (!args) return 0;
  return bwd_layout(args).total;
}

pkm_status pkm_backward(const pkm_bwd_args* args, pkm_stream_t stream) {
  pkm_status s = validate_bwd(args);
  if (s != PKM_OK || args->T == 0) {
    if (s == PKM_OK && args->n_uniq)
      return cudaMemsetAsync(args->n_uniq, 0, sizeof(int64_t),
                             reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
                 ? PKM_OK
                 : PKM_ERR_CUDA;
    return s;
  }
  return backward_impl(args, reinterpret_cast<cudaStream_t>(stream));
}

size_t embbag_backward_workspace_size(int64_t n_bags, int32_t B, int32_t d, int64_t n_rows) {
  size_t parts[6];
  return embbag_bwd_bytes(n_bags, B, d, n_rows, parts);
}

pkm_status embbag_backward(const void* dy, const int32_t* idx, const float* w, int64_t n_bags,
                           int32_t B, int32_t d, pkm_dtype dtype, const void* table,
                           int64_t n_rows, float* dw, int32_t* uniq_rows, float* grad_rows,
                           int64_t* n_uniq, int64_t uniq_cap, float* dense_accum,
                           void* workspace, size_t workspace_bytes, pkm_stream_t stream) {
  if (n_bags < 0 || n_rows < 1 || n_rows > 0x7fffffff || d < 8 || d % 8 || B < 1 || B > 4096)
    return PKM_ERR_INVALID_ARG;
  if (dtype != PKM_F32 && dtype != PKM_BF16) return PKM_ERR_INVALID_ARG;
  if (n_bags * (int64_t)B >= (int64_t(1) << 32)) return PKM_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (n_bags == 0)
    return n_uniq && cudaMemsetAsync(n_uniq, 0, sizeof(int64_t), st) != cudaSuccess ? PKM_ERR_CUDA
                                                                                      : PKM_OK;
  if (!dy || !idx || !w || !aligned16(dy)) return PKM_ERR_INVALID_ARG;
  if (dw && (!table || !aligned16(table))) return PKM_ERR_INVALID_ARG;
  const bool sparse = grad_rows != nullptr;
  if (sparse && (!uniq_rows || !n_uniq || uniq_cap < 0 || !aligned16(grad_rows)))
    return PKM_ERR_INVALID_ARG;
  if (dense_accum && !aligned16(dense_accum)) return PKM_ERR_INVALID_ARG;
  size_t parts[6];
  const size_t need = embbag_bwd_bytes(n_bags, B, d, n_rows, parts);
  if ((sparse || dense_accum) && (!workspace || !aligned16(workspace) || workspace_bytes < need))
    return PKM_ERR_WORKSPACE;
  int32_t* status = status_ptr();
  if (!status) return PKM_ERR_CUDA;
  if (dw && launch_bag_dw(dy, table, n_rows, d, dtype, idx, w, n_bags, B, 0, dw, nullptr, status,
                          st) != cudaSuccess)
    return PKM_ERR_CUDA;
  if (!sparse && !dense_accum) return PKM_OK;
  char* ws = static_cast<char*>(workspace);
  uint32_t* iota = reinterpret_cast<uint32_t*>(ws + parts[0]);
  uint32_t* skeys = reinterpret_cast<uint32_t*>(ws + parts[1]);
  uint32_t* svals = reinterpret_cast<uint32_t*>(ws + parts[2]);
  uint32_t* ckeys = reinterpret_cast<uint32_t*>(ws + parts[5]);
  const int64_t R = n_bags * B;
  // out-of-range row ids become the key n_rows: sorted last, never summed
  if (launch_iota(iota, R, st) != cudaSuccess) return PKM_ERR_CUDA;
  if (launch_sanitize_keys(idx, R, n_rows, ckeys, status, st) != cudaSuccess) return PKM_ERR_CUDA;
  if (launch_radix_sort(ckeys, iota, R, bits_for((uint64_t)n_rows), skeys, svals, ws + parts[3],
                        st) != cudaSuccess)
    return PKM_ERR_CUDA;
  if (launch_segsum(skeys, svals, R, (uint32_t)n_rows, w, dy, dtype, B, d, uniq_rows, grad_rows,
                    sparse ? uniq_cap : 0, n_uniq, dense_accum, nullptr, ws + parts[4], status,
                    st) != cudaSuccess)
    return PKM_ERR_CUDA;
  return PKM_OK;
}

}  // extern "C"
