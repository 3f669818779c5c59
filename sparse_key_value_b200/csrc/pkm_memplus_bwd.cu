// pkm_memplus_bwd.cu -- Memory+ backward and the query projection (C ABI,
// see include/pkm.h).
//
// "Memory Layers at Scale" digest, "Memory+ 블록": out = (y ⊙ silu(x W1)) W2.
// Per token, a = x W1, g = silu(a), z = y ⊙ g:
//   dz = dout W2^T, dy = dz ⊙ g, da = dz ⊙ y ⊙ silu'(a), dx = da W1^T,
//   dW1 = x^T da, dW2 = z^T dout.
// The products run on the tcgen05 GEMM (fp32 accumulation), every operand
// read in the layout it is held: W1 [d_model][d_v] as the MN-major B of x W1,
// and the token rows x, da, z, dout as MN-major operands of the weight
// gradients, which contract over the tokens (split over K when the output
// has few tiles, the slices summed in order).
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace pkm {

namespace {

size_t rup(size_t x) { return (x + 255) / 256 * 256; }
bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define PKM_TRY(expr)                           \
  do {                                          \
    cudaError_t e_ = (expr);                    \
    if (e_ != cudaSuccess) return PKM_ERR_CUDA; \
  } while (0)

// dy = dz * g, da = dz * y * silu'(a), z = y * g with g = silu(a); bf16 out
__global__ void memplus_bwd_elem_kernel(const float* __restrict__ a, const float* __restrict__ dz,
                                        const __nv_bfloat16* __restrict__ y, int64_t n,
                                        __nv_bfloat16* __restrict__ dy,
                                        __nv_bfloat16* __restrict__ da,
                                        __nv_bfloat16* __restrict__ z) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float av = a[i], dzv = dz[i], yv = __bfloat162float(y[i]);
    const float s = 1.0f / (1.0f + expf(-av));
    const float g = av * s;
    dy[i] = __float2bfloat16_rn(dzv * g);
    da[i] = __float2bfloat16_rn(dzv * yv * s * (1.0f + av * (1.0f - s)));
    z[i] = __float2bfloat16_rn(yv * g);
  }
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ x, int64_t n,
                                   __nv_bfloat16* __restrict__ y) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    y[i] = __float2bfloat16_rn(x[i]);
}

unsigned elem_grid(int64_t n) {
  const int64_t b = (n + 255) / 256;
  return (unsigned)(b < 148 * 16 ? (b > 0 ? b : 1) : 148 * 16);
}

struct MpLayout {
  size_t a, dz, da, z, part, total;
};

MpLayout mp_layout(const pkm_memplus_bwd_args* g) {
  MpLayout L{};
  const size_t T = (size_t)(g->T > 0 ? g->T : 0), dm = (size_t)g->d_model, dv = (size_t)g->d_v;
  size_t off = 0;
  auto take = [&](size_t b) {
    const size_t o = off;
    off += rup(b);
    return o;
  };
  L.a = take(T * dv * 4);
  L.dz = take(T * dv * 4);
  L.da = take(T * dv * 2);
  L.z = take(T * dv * 2);
  const size_t p1 = gemm_splitk_workspace((int64_t)dm, (int)dv, (int)T);
  const size_t p2 = gemm_splitk_workspace((int64_t)dv, (int)dm, (int)T);
  L.part = take(p1 > p2 ? p1 : p2);
  L.total = off;
  return L;
}

pkm_status mp_validate(const pkm_memplus_bwd_args* g) {
  if (!g || g->T < 0 || g->d_model < 8 || g->d_model % 8 || g->d_v < 8 || g->d_v % 8)
    return PKM_ERR_INVALID_ARG;
  if (g->T > (int64_t(1) << 31) - 64) return PKM_ERR_UNSUPPORTED;
  const void* need[] = {g->W1, g->W2, g->dW1, g->dW2};
  for (const void* p : need)
    if (!p || !al16(p)) return PKM_ERR_INVALID_ARG;
  if (g->T > 0) {
    const void* need_t[] = {g->x, g->y, g->dout, g->dy, g->dx};
    for (const void* p : need_t)
      if (!p || !al16(p)) return PKM_ERR_INVALID_ARG;
  }
  if (!g->workspace || !al16(g->workspace) || g->workspace_bytes < mp_layout(g).total)
    return PKM_ERR_WORKSPACE;
  return PKM_OK;
}

struct QpLayout {
  size_t dqb, part, total;
};

QpLayout qp_layout(const pkm_qproj_args* g) {
  QpLayout L{};
  const size_t T = (size_t)(g->T > 0 ? g->T : 0), dm = (size_t)g->d_model, dq = (size_t)g->d_q;
  size_t off = 0;
  auto take = [&](size_t b) {
    const size_t o = off;
    off += rup(b);
    return o;
  };
  L.dqb = take(T * dq * 2);
  L.part = take(gemm_splitk_workspace((int64_t)dm, (int)dq, (int)T));
  L.total = off;
  return L;
}

pkm_status qp_validate(const pkm_qproj_args* g, bool backward) {
  if (!g || g->T < 0 || g->d_model < 8 || g->d_model % 8 || g->d_q < 8 || g->d_q % 8)
    return PKM_ERR_INVALID_ARG;
  if (g->T > (int64_t(1) << 31) - 64) return PKM_ERR_UNSUPPORTED;
  if (!g->Wq || !al16(g->Wq)) return PKM_ERR_INVALID_ARG;
  if (backward && (!g->dWq || !al16(g->dWq))) return PKM_ERR_INVALID_ARG;
  if (g->T > 0) {
    if (!g->x || !al16(g->x)) return PKM_ERR_INVALID_ARG;
    if (!backward && (!g->q || !al16(g->q))) return PKM_ERR_INVALID_ARG;
    if (backward && (!g->dq || !al16(g->dq) || !g->dx || !al16(g->dx)))
      return PKM_ERR_INVALID_ARG;
  }
  if (!g->workspace || !al16(g->workspace) || g->workspace_bytes < qp_layout(g).total)
    return PKM_ERR_WORKSPACE;
  return PKM_OK;
}

__global__ void gate_mul_kernel(const __nv_bfloat16* __restrict__ y,
                                const __nv_bfloat16* __restrict__ g, int64_t n,
                                __nv_bfloat16* __restrict__ z) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    z[i] = __float2bfloat16_rn(__bfloat162float(y[i]) * __bfloat162float(g[i]));
}

}  // namespace

cudaError_t launch_gate_mul_bf16(const void* y, const void* g, int64_t n, void* z,
                                 cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  gate_mul_kernel<<<elem_grid(n), 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(y),
                                                    static_cast<const __nv_bfloat16*>(g), n,
                                                    static_cast<__nv_bfloat16*>(z));
  note_launch();
  return cudaGetLastError();
}

pkm_status memplus_backward_impl(const pkm_memplus_bwd_args* g, cudaStream_t st) {
  int32_t* status = status_ptr();
  if (!status) return PKM_ERR_CUDA;
  const int64_t T = g->T;
  const int dm = g->d_model, dv = g->d_v;
  if (T == 0) {
    PKM_TRY(cudaMemsetAsync(g->dW1, 0, sizeof(float) * (size_t)dm * dv, st));
    PKM_TRY(cudaMemsetAsync(g->dW2, 0, sizeof(float) * (size_t)dv * dm, st));
    return PKM_OK;
  }
  const MpLayout L = mp_layout(g);
  char* ws = static_cast<char*>(g->workspace);
  auto* a = reinterpret_cast<float*>(ws + L.a);
  auto* dz = reinterpret_cast<float*>(ws + L.dz);
  auto* da = reinterpret_cast<__nv_bfloat16*>(ws + L.da);
  auto* z = reinterpret_cast<__nv_bfloat16*>(ws + L.z);
  // a = x W1 (W1 [d_model][d_v] read as held), dz = dout W2^T (W2 is [d_v, d_model])
  PKM_TRY(launch_gemm_f32(g->x, g->W1, T, dv, dm, false, a, status, st, false, /*b_mn*/ true));
  PKM_TRY(launch_gemm_f32(g->dout, g->W2, T, dv, dm, false, dz, status, st));
  const int64_t n = T * dv;
  memplus_bwd_elem_kernel<<<elem_grid(n), 256, 0, st>>>(
      a, dz, static_cast<const __nv_bfloat16*>(g->y), n, static_cast<__nv_bfloat16*>(g->dy), da,
      z);
  note_launch();
  PKM_TRY(cudaGetLastError());
  // dx = da W1^T (W1 is [d_model, d_v])
  PKM_TRY(launch_gemm_f32(da, g->W1, T, dm, dv, false, g->dx, status, st));
  // dW1 = x^T da, dW2 = z^T dout: contract over the tokens, every operand read
  // as held ([T][d] rows: MN-major for these products)
  float* part = reinterpret_cast<float*>(ws + L.part);
  PKM_TRY(launch_gemm_f32_splitk(g->x, da, dm, dv, (int)T, g->dW1, part, status, st, true,
                                 true));
  PKM_TRY(launch_gemm_f32_splitk(z, g->dout, dv, dm, (int)T, g->dW2, part, status, st, true,
                                 true));
  return PKM_OK;
}

}  // namespace pkm

using namespace pkm;

extern "C" {

PKM_API size_t pkm_memplus_backward_workspace_size(const pkm_memplus_bwd_args* args) {
  return args ? mp_layout(args).total : 0;
}

PKM_API pkm_status pkm_memplus_backward(const pkm_memplus_bwd_args* args, pkm_stream_t stream) {
  const pkm_status s = mp_validate(args);
  if (s != PKM_OK) return s;
  return memplus_backward_impl(args, reinterpret_cast<cudaStream_t>(stream));
}

PKM_API size_t pkm_qproj_workspace_size(const pkm_qproj_args* args) {
  return args ? qp_layout(args).total : 0;
}

PKM_API pkm_status pkm_qproj_forward(const pkm_qproj_args* g, pkm_stream_t stream) {
  const pkm_status s = qp_validate(g, false);
  if (s != PKM_OK || g->T == 0) return s;
  int32_t* status = status_ptr();
  if (!status) return PKM_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const QpLayout L = qp_layout(g);
  char* ws = static_cast<char*>(g->workspace);
  // q = x Wq, Wq [d_model][d_q] read as held
  (void)L;
  (void)ws;
  PKM_TRY(launch_gemm_bf16(g->x, g->Wq, g->T, g->d_q, g->d_model, 0, g->q, status, st, true));
  return PKM_OK;
}

PKM_API pkm_status pkm_qproj_backward(const pkm_qproj_args* g, pkm_stream_t stream) {
  const pkm_status s = qp_validate(g, true);
  if (s != PKM_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (g->T == 0)
    return cudaMemsetAsync(g->dWq, 0, sizeof(float) * (size_t)g->d_model * g->d_q, st) ==
                   cudaSuccess
               ? PKM_OK
               : PKM_ERR_CUDA;
  int32_t* status = status_ptr();
  if (!status) return PKM_ERR_CUDA;
  const QpLayout L = qp_layout(g);
  char* ws = static_cast<char*>(g->workspace);
  const int64_t T = g->T;
  const int dm = g->d_model, dq = g->d_q;
  auto* dqb = reinterpret_cast<__nv_bfloat16*>(ws + L.dqb);
  f32_to_bf16_kernel<<<elem_grid(T * dq), 256, 0, st>>>(g->dq, T * dq, dqb);
  note_launch();
  PKM_TRY(cudaGetLastError());
  // dx += dq Wq^T (Wq is [d_model, d_q]); dWq = x^T dq over the tokens
  PKM_TRY(launch_gemm_f32(dqb, g->Wq, T, dm, dq, true, g->dx, status, st));
  PKM_TRY(launch_gemm_f32_splitk(g->x, dqb, dm, dq, (int)T, g->dWq,
                                 reinterpret_cast<float*>(ws + L.part), status, st, true, true));
  return PKM_OK;
}

}  // extern "C"
