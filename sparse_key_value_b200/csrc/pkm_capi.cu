// pkm_capi.cu -- the C ABI of libpkm.so: argument validation, workspace
// carving and the launch sequence of each entry point (see include/pkm.h).
#include <atomic>
#include <mutex>
#include <stdio.h>

#include "common.cuh"
#include "kernels.h"

namespace pkm {

__device__ int32_t g_status = 0;  // sticky per-device status word

static std::atomic<unsigned long long> g_launches{0};
void note_launch(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

static std::mutex g_status_mu;
static int32_t* g_status_ptr[64] = {nullptr};

// Device address of this device's status word (looked up once per device).
int32_t* status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_status_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int32_t*>(p);
  }
  return g_status_ptr[dev];
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ------------------------------------------------------------ forward ----

struct FwdLayout {
  size_t rq, rk, hv, hi, sel, g, z, part, total;
  int splits;
  bool tc;
  bool fused;  // the one-kernel selection (k_select_tc.cu)
  bool small;  // decode-sized batches: the one-kernel selection of k_select_small.cu
};

static bool has_memplus(const pkm_fwd_args* a) { return a->x || a->W1 || a->W2; }

static FwdLayout fwd_layout(const pkm_fwd_args* a) {
  FwdLayout L{};
  const size_t T = (size_t)(a->T > 0 ? a->T : 0);
  const size_t H = (size_t)a->H, n = (size_t)a->n_sub, k = (size_t)a->k;
  // batches beyond the decode sizes run the one-kernel selection; small ones
  // split the sub-key columns over CTAs (score_topk_tc) and combine apart
  L.fused = select_tc_supported(a->dtype, a->d_half, a->n_sub, a->k) &&
            a->T > kSplitGatherMaxBags;
  L.small = !L.fused && select_small_supported(a->dtype, a->T, a->d_half, a->n_sub, a->k);
  L.tc = !L.fused && !L.small && score_tc_supported(a->dtype, a->d_half, a->n_sub, a->k);
  L.splits = L.tc ? score_tc_splits(a->T, a->H, a->n_sub) : 1;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = round_up(off + bytes, 256);
    return o;
  };
  // padded by one chunk of columns: the scoring epilogues read 8 at a time
  if (!L.small) L.rk = take((H * 2 * n + 256) * sizeof(float));
  if (L.fused) {
    L.sel = take(select_tc_workspace((int64_t)T, (int)H));
  } else if (L.small) {
    L.sel = take(select_small_workspace((int64_t)T, (int)H, (int)n));
  } else {
    L.rq = take(T * H * 2 * sizeof(float));
    L.hv = take((size_t)L.splits * T * H * 2 * k * sizeof(float));
    L.hi = take((size_t)L.splits * T * H * 2 * k * sizeof(int32_t));
  }
  if (has_memplus(a)) {
    const size_t dv = (size_t)a->d_v;
    L.g = take(T * dv * 2);
    L.z = take(T * dv * 2);
  }
  // small batches gather through row-group partial sums
  if ((int64_t)T <= kSplitGatherMaxBags)
    L.part = take(embbag_split_workspace((int64_t)T, (int)(H * k), a->d_v));
  L.total = off;
  return L;
}

// Arguments of a forward, without the workspace (sizes, dtype, pointers).
// T is bounded so that no workspace size computed from the arguments wraps.
pkm_status check_fwd_args(const pkm_fwd_args* a) {
  if (!a) return PKM_ERR_INVALID_ARG;
  if (a->T < 0 || a->T > kMaxTokens || a->H < 1 || a->n_sub < 1 || a->k < 1 || a->k > 64 ||
      a->k > a->n_sub)
    return PKM_ERR_INVALID_ARG;
  if (a->d_half < 8 || a->d_half % 8 || a->d_v < 8 || a->d_v % 8) return PKM_ERR_INVALID_ARG;
  if ((int64_t)a->n_sub * a->n_sub >= (int64_t(1) << 31)) return PKM_ERR_INVALID_ARG;
  if (a->dtype != PKM_F32 && a->dtype != PKM_BF16) return PKM_ERR_INVALID_ARG;
  if (a->H * a->k > 4096) return PKM_ERR_INVALID_ARG;
  if (a->d_half > 2048) return PKM_ERR_UNSUPPORTED;
  if (a->T == 0) return PKM_OK;
  const void* need[] = {a->query, a->subkeys, a->values, a->out, a->idx, a->weights};
  for (const void* p : need)
    if (!p || !aligned16(p)) return PKM_ERR_INVALID_ARG;
  if (a->y_out && (!has_memplus(a) || !aligned16(a->y_out))) return PKM_ERR_INVALID_ARG;
  if (has_memplus(a)) {
    if (!a->x || !a->W1 || !a->W2) return PKM_ERR_INVALID_ARG;
    if (!aligned16(a->x) || !aligned16(a->W1) || !aligned16(a->W2)) return PKM_ERR_INVALID_ARG;
    if (a->d_model < 8 || a->d_model % 8) return PKM_ERR_INVALID_ARG;
    if (a->dtype != PKM_BF16) return PKM_ERR_UNSUPPORTED;
  }
  return PKM_OK;
}

static pkm_status validate_fwd(const pkm_fwd_args* a) {
  const pkm_status s = check_fwd_args(a);
  if (s != PKM_OK || a->T == 0) return s;
  const FwdLayout L = fwd_layout(a);
  if (!a->workspace || !aligned16(a->workspace) || a->workspace_bytes < L.total)
    return PKM_ERR_WORKSPACE;
  return PKM_OK;
}

#define PKM_TRY(expr)                          \
  do {                                         \
    cudaError_t e_ = (expr);                   \
    if (e_ != cudaSuccess) return PKM_ERR_CUDA; \
  } while (0)

// Phase event i on the stream; under stream capture it becomes an event
// record node of the graph, so replays time their phases too.
static void mark(const pkm_fwd_args* a, int i, cudaStream_t st) {
  if (a->phase_events && a->phase_events[i]) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) cs = cudaStreamCaptureStatusNone;
    cudaEventRecordWithFlags(static_cast<cudaEvent_t>(a->phase_events[i]), st,
                             cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal
                                                                 : cudaEventRecordDefault);
  }
}

static pkm_status forward_impl(const pkm_fwd_args* a, cudaStream_t st,
                               bool select_only = false) {
  int32_t* status = status_ptr();
  if (!status) return PKM_ERR_CUDA;
  const FwdLayout L = fwd_layout(a);
  char* ws = static_cast<char*>(a->workspace);
  float* rq = reinterpret_cast<float*>(ws + L.rq);
  float* rk = reinterpret_cast<float*>(ws + L.rk);
  float* hv = reinterpret_cast<float*>(ws + L.hv);
  int32_t* hi = reinterpret_cast<int32_t*>(ws + L.hi);
  const int64_t T = a->T;
  const int H = a->H, dh = a->d_half, n = a->n_sub, k = a->k;
  const int64_t N = (int64_t)n * n;
  const bool mp = has_memplus(a);
  const int dm = a->d_model, dv = a->d_v;
  char* g = mp ? ws + L.g : nullptr;
  char* z = mp ? ws + L.z : nullptr;

  // a1: qk-normalisation factors (inside the one-kernel selections: the
  // query's in both, the sub-keys' too in the small-batch one)
  mark(a, 0, st);
  if (!L.fused && !L.small) PKM_TRY(launch_row_rnorm(a->query, a->dtype, T * H * 2, dh, rq, st));
  if (!L.small)
    PKM_TRY(launch_row_rnorm(a->subkeys, a->dtype, (int64_t)H * 2 * n, dh, rk, st));
  mark(a, 1, st);

  if (L.fused) {
    // a1 (query) + a2 .. a5 in one kernel
    PKM_TRY(launch_select_tc(a->query, a->subkeys, T, H, dh, n, k, rk, a->idx, a->weights,
                             ws + L.sel, status, st));
    mark(a, 2, st);
  } else if (L.small) {
    // a1 .. a5 in one kernel
    PKM_TRY(launch_select_small(a->query, a->subkeys, T, H, dh, n, k, a->idx, a->weights,
                                ws + L.sel, status, st));
    mark(a, 2, st);
  } else {
    // a2 + a3: sub-key scores and per-half top-k
    if (L.tc)
      PKM_TRY(launch_score_topk_tc(a->query, a->subkeys, T, H, dh, n, k, L.splits, rq, rk, hv,
                                   hi, status, st));
    else
      PKM_TRY(launch_score_topk_simt(a->query, a->subkeys, a->dtype, T, H, dh, n, k, rq, rk,
                                     hv, hi, st));
    mark(a, 2, st);
    // a4 + a5: k x k combine, top-k, softmax
    PKM_TRY(launch_combine(hv, hi, L.splits, T, H, n, k, a->idx, a->weights, st));
  }
  mark(a, 3, st);
  if (select_only) return PKM_OK;
  // Programmatic dependent launch: the gate GEMM runs beside the selection
  // (it reads neither idx nor w) on the SMs the selection's last wave leaves
  // free.  Few-token batches chain the later kernels the same way (each
  // waits in-kernel for its predecessor's results instead of at the launch);
  // for large batches an early-launched gather measured slower (its waiting
  // CTAs crowd the SMs as the selection drains), so those launch as usual.
  const bool few = T <= kSplitGatherMaxBags;
  // (a7) gate GEMM, a6 bag gather over the H*k selected rows of each token
  if (mp)  // g = silu(x W1), W1 [d_model][d_v] read as it is held
    PKM_TRY(launch_gemm_bf16(a->x, a->W1, T, dv, dm, /*silu*/ 1, g, status, st, /*b_mn*/ true,
                             /*pdl: overlap*/ 2));
  mark(a, 4, st);
  // with y_out the bag output is kept and the gate applied in a second pass
  const void* gate = a->y_out ? nullptr : g;
  void* bag_out = a->y_out ? a->y_out : (mp ? z : a->out);
  if (few)
    PKM_TRY(launch_embbag_fwd_split(a->values, N, dv, a->dtype, a->idx, a->weights, T, H * k,
                                    gate, bag_out, reinterpret_cast<float*>(ws + L.part),
                                    status, st, /*pdl*/ true));
  else
    PKM_TRY(launch_embbag_fwd(a->values, N, dv, a->dtype, a->idx, a->weights, T, H * k, gate,
                              bag_out, status, st));
  if (a->y_out) PKM_TRY(launch_gate_mul_bf16(a->y_out, g, T * dv, z, st));
  mark(a, 5, st);
  if (mp)  // out = z W2, W2 [d_v][d_model] read as it is held
    PKM_TRY(launch_gemm_bf16(z, a->W2, T, dm, dv, /*none*/ 0, a->out, status, st, true,
                             few && !a->y_out ? /*pdl: z from the gather*/ 1 : 0));
  mark(a, 6, st);
  return PKM_OK;
}

// Arguments of a selection-only call: the forward's, without the value table,
// the output and Memory+ (those fields are ignored).
static pkm_fwd_args select_args(const pkm_fwd_args* a) {
  pkm_fwd_args b = *a;
  b.x = b.W1 = b.W2 = nullptr;
  b.y_out = nullptr;
  b.d_model = 0;
  return b;
}

static pkm_status validate_select(const pkm_fwd_args* b) {
  if (b->T < 0 || b->T > kMaxTokens || b->H < 1 || b->n_sub < 1 || b->k < 1 || b->k > 64 ||
      b->k > b->n_sub)
    return PKM_ERR_INVALID_ARG;
  if (b->d_half < 8 || b->d_half % 8 || b->d_v < 8 || b->d_v % 8) return PKM_ERR_INVALID_ARG;
  if ((int64_t)b->n_sub * b->n_sub >= (int64_t(1) << 31)) return PKM_ERR_INVALID_ARG;
  if (b->dtype != PKM_F32 && b->dtype != PKM_BF16) return PKM_ERR_INVALID_ARG;
  if (b->H * b->k > 4096) return PKM_ERR_INVALID_ARG;
  if (b->d_half > 2048) return PKM_ERR_UNSUPPORTED;
  if (b->T == 0) return PKM_OK;
  const void* need[] = {b->query, b->subkeys, b->idx, b->weights};
  for (const void* p : need)
    if (!p || !aligned16(p)) return PKM_ERR_INVALID_ARG;
  if (!b->workspace || !aligned16(b->workspace) || b->workspace_bytes < fwd_layout(b).total)
    return PKM_ERR_WORKSPACE;
  return PKM_OK;
}

// The forward with a workspace chosen inside the library (the allocation-free
// entry point in pkm_noalloc.cu passes its static scratch array here).
pkm_status forward_into(const pkm_fwd_args* a, void* workspace, size_t workspace_bytes,
                        cudaStream_t st) {
  if (!a) return PKM_ERR_INVALID_ARG;
  pkm_fwd_args b = *a;
  b.workspace = workspace;
  b.workspace_bytes = workspace_bytes;
  pkm_status s = validate_fwd(&b);
  if (s != PKM_OK || b.T == 0) return s;
  return forward_impl(&b, st);
}

size_t forward_workspace_bytes(const pkm_fwd_args* a) { return a ? fwd_layout(a).total : 0; }

}  // namespace pkm

using namespace pkm;

extern "C" {

size_t pkm_forward_workspace_size(const pkm_fwd_args* args) {
  if (!args) return 0;
  return fwd_layout(args).total;
}

pkm_status pkm_select(const pkm_fwd_args* args, pkm_stream_t stream) {
  if (!args) return PKM_ERR_INVALID_ARG;
  const pkm_fwd_args b = select_args(args);
  pkm_status s = validate_select(&b);
  if (s != PKM_OK || b.T == 0) return s;
  return forward_impl(&b, reinterpret_cast<cudaStream_t>(stream), /*select_only*/ true);
}

pkm_status pkm_forward(const pkm_fwd_args* args, pkm_stream_t stream) {
  pkm_status s = validate_fwd(args);
  if (s != PKM_OK || args->T == 0) return s;
  return forward_impl(args, reinterpret_cast<cudaStream_t>(stream));
}

pkm_status embbag_forward(const void* table, int64_t n_rows, int32_t d, pkm_dtype dtype,
                          const int32_t* idx, const float* w, int64_t n_bags, int32_t B,
                          const void* gate, void* out, pkm_stream_t stream) {
  if (n_bags < 0 || n_rows < 1 || d < 8 || d % 8 || B < 1 || B > 4096)
    return PKM_ERR_INVALID_ARG;
  if (dtype != PKM_F32 && dtype != PKM_BF16) return PKM_ERR_INVALID_ARG;
  if (n_bags == 0) return PKM_OK;
  if (!table || !idx || !w || !out || !aligned16(table) || !aligned16(out) ||
      (gate && !aligned16(gate)))
    return PKM_ERR_INVALID_ARG;
  int32_t* status = status_ptr();
  if (!status) return PKM_ERR_CUDA;
  cudaError_t e = launch_embbag_fwd(table, n_rows, d, dtype, idx, w, n_bags, B, gate, out,
                                    status, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PKM_OK : PKM_ERR_CUDA;
}

pkm_status embbag_forward_range(const void* table, int64_t row_lo, int64_t n_local, int32_t d,
                                pkm_dtype dtype, const int32_t* idx, const float* w,
                                int64_t n_bags, int32_t B, float* out, pkm_stream_t stream) {
  if (n_bags < 0 || row_lo < 0 || n_local < 1 || d < 8 || d % 8 || B < 1 || B > 4096)
    return PKM_ERR_INVALID_ARG;
  if (dtype != PKM_F32 && dtype != PKM_BF16) return PKM_ERR_INVALID_ARG;
  if (n_bags == 0) return PKM_OK;
  if (!table || !idx || !w || !out || !aligned16(table) || !aligned16(out))
    return PKM_ERR_INVALID_ARG;
  return launch_embbag_range(table, row_lo, n_local, d, dtype, idx, w, n_bags, B, out,
                             reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? PKM_OK
             : PKM_ERR_CUDA;
}

pkm_status pkm_get_device_error(pkm_stream_t stream, int32_t* code) {
  if (!code) return PKM_ERR_INVALID_ARG;
  int32_t* status = status_ptr();
  if (!status) return PKM_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, status, sizeof v, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return PKM_ERR_CUDA;
  if (cudaMemsetAsync(status, 0, sizeof v, st) != cudaSuccess) return PKM_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return PKM_ERR_CUDA;
  *code = v;
  return PKM_OK;
}

const char* pkm_status_string(pkm_status s) {
  switch (s) {
    case PKM_OK: return "ok";
    case PKM_ERR_INVALID_ARG: return "invalid argument";
    case PKM_ERR_UNSUPPORTED: return "unsupported combination";
    case PKM_ERR_CUDA: return "CUDA call failed";
    case PKM_ERR_DEVICE: return "device anomaly: row id out of range or output overflow";
    case PKM_ERR_TIMEOUT: return "device spin-wait ran out";
    case PKM_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

int32_t pkm_version(void) { return 100; }

uint64_t pkm_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
