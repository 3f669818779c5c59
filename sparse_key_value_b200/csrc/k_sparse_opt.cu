// k_sparse_opt.cu -- optimiser step on the touched value rows only.
//
// "모델 안의 메모리", "잊지 않고 배우기": a fact occupies a few memory slots, so
// only those slots need updating.  The backward's sparse value gradient
// (distinct row ids + one fp32 row each, in sorted order) drives an in-place
// update of exactly those table rows:
//   SGD   p -= lr * g
//   Adam  m = b1 m + (1 - b1) g,  v = b2 v + (1 - b2) g^2,
//         p -= lr * (m / c1) / (sqrt(v / c2) + eps),  c = 1 - b^step,
// moments of untouched rows are left as they are.  Every row is handled by
// one CTA (rows are distinct), so the result is deterministic.  bf16 tables
// are updated in fp32 and rounded once (nearest even).  The C entry point
// pkm_sparse_optimizer_step (include/pkm.h) validates and launches.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace pkm {

namespace {

__device__ __forceinline__ void load4(const float* p, float (&x)[4]) {
  const float4 v = *reinterpret_cast<const float4*>(p);
  x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
}
__device__ __forceinline__ void store4(float* p, const float (&x)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
}
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&x)[4]) {
  const uint2 v = *reinterpret_cast<const uint2*>(p);
  x[0] = bf16_lo(v.x); x[1] = bf16_hi(v.x); x[2] = bf16_lo(v.y); x[3] = bf16_hi(v.y);
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, const float (&x)[4]) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]));
}

template <typename T, bool ADAM>
__global__ void __launch_bounds__(256) sparse_opt_kernel(
    T* __restrict__ table, int64_t n_rows, int d, const int32_t* __restrict__ rows,
    const float* __restrict__ grads, const int64_t* __restrict__ count, int64_t cap,
    float* __restrict__ m, float* __restrict__ v, float lr, float b1, float b2, float eps,
    float c1, float c2, int32_t* status) {
  int64_t n = *count;
  if (n > cap) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, PKM_ERR_DEVICE);
    n = cap;
  }
  for (int64_t i = blockIdx.x; i < n; i += gridDim.x) {
    const int32_t r = rows[i];
    if (r < 0 || r >= n_rows) {
      if (threadIdx.x == 0) set_status(status, PKM_ERR_DEVICE);
      continue;
    }
    for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4) {
      const int64_t o = (int64_t)r * d + c;
      float p[4], g[4];
      load4(table + o, p);
      load4(grads + i * d + c, g);
      if (ADAM) {
        float mm[4], vv[4];
        load4(m + o, mm);
        load4(v + o, vv);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          mm[e] = b1 * mm[e] + (1.0f - b1) * g[e];
          vv[e] = b2 * vv[e] + (1.0f - b2) * g[e] * g[e];
          p[e] -= lr * (mm[e] / c1) / (sqrtf(vv[e] / c2) + eps);
        }
        store4(m + o, mm);
        store4(v + o, vv);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) p[e] -= lr * g[e];
      }
      store4(table + o, p);
    }
  }
}

}  // namespace

cudaError_t launch_sparse_opt(void* table, pkm_dtype dt, int64_t n_rows, int d,
                              const int32_t* rows, const float* grads, const int64_t* count,
                              int64_t cap, bool adam, float* m, float* v, float lr, float b1,
                              float b2, float eps, int64_t step, int32_t* status,
                              cudaStream_t stream) {
  if (cap <= 0) return cudaSuccess;
  const float c1 = adam ? (float)(1.0 - pow((double)b1, (double)step)) : 1.f;
  const float c2 = adam ? (float)(1.0 - pow((double)b2, (double)step)) : 1.f;
  const int threads = min(256, ((d / 4) + 31) / 32 * 32);
  const int64_t blocks = cap < 148 * 16 ? cap : 148 * 16;
#define PKM_OPT(T_, A_)                                                                    \
  sparse_opt_kernel<T_, A_><<<(unsigned)blocks, threads, 0, stream>>>(                     \
      static_cast<T_*>(table), n_rows, d, rows, grads, count, cap, m, v, lr, b1, b2, eps, c1, \
      c2, status)
  if (dt == PKM_BF16) {
    if (adam) PKM_OPT(__nv_bfloat16, true);
    else PKM_OPT(__nv_bfloat16, false);
  } else {
    if (adam) PKM_OPT(float, true);
    else PKM_OPT(float, false);
  }
#undef PKM_OPT
  note_launch();
  return cudaGetLastError();
}

}  // namespace pkm

using namespace pkm;

static bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

extern "C" {

PKM_API pkm_status pkm_sparse_optimizer_step(const pkm_sparse_opt_args* a, pkm_stream_t stream) {
  if (!a || a->n_rows < 1 || a->d < 8 || a->d % 8 || a->cap < 0) return PKM_ERR_INVALID_ARG;
  if (a->dtype != PKM_F32 && a->dtype != PKM_BF16) return PKM_ERR_INVALID_ARG;
  if (!(fabsf(a->lr) < INFINITY)) return PKM_ERR_INVALID_ARG;
  const bool adam = a->kind == PKM_OPT_ADAM;
  if (!adam && a->kind != PKM_OPT_SGD) return PKM_ERR_INVALID_ARG;
  if (adam && (!(a->beta1 >= 0.f && a->beta1 < 1.f) || !(a->beta2 >= 0.f && a->beta2 < 1.f) ||
               !(a->eps >= 0.f) || a->step < 1 || !a->m || !a->v || !al16(a->m) || !al16(a->v)))
    return PKM_ERR_INVALID_ARG;
  const void* need[] = {a->table, a->rows, a->grads, a->count};
  for (const void* p : need)
    if (!p || !al16(p)) return PKM_ERR_INVALID_ARG;
  int32_t* status = status_ptr();
  if (!status) return PKM_ERR_CUDA;
  return launch_sparse_opt(a->table, a->dtype, a->n_rows, a->d, a->rows, a->grads, a->count,
                           a->cap, adam, a->m, a->v, a->lr, a->beta1, a->beta2, a->eps, a->step,
                           status, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? PKM_OK
             : PKM_ERR_CUDA;
}

}  // extern "C"
