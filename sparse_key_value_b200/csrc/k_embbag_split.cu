// k_embbag_split.cu -- the weighted bag gather for small batches.
//
// Same result as embbag_fwd_kernel ("Memory Layers at Scale" digest, "병렬
// EmbeddingBag 구현": out[t] = sum_j w[t,j] * table[idx[t,j]], optionally
// times the gate row), for batches too small to occupy the GPU (decode
// steps): each bag's rows are cut into groups of kGroupRows and every
// (bag, group) is one CTA, so all of a bag's row loads are in flight at once.
// The groups' fp32 partial sums go to a workspace; a second kernel adds them
// in group order (deterministic), applies the gate and rounds once.
#include "common.cuh"
#include "kernels.h"

namespace pkm {

namespace {
constexpr int kGroupRows = 16;  // rows per partial sum (one batch of loads)
}

// grid (n_bags, groups); one thread per 16-byte column chunk
template <pkm_dtype DT>
__global__ void __launch_bounds__(256) embbag_part_kernel(
    const typename Elem<DT>::T* __restrict__ table, int64_t n_rows, int d,
    const int32_t* __restrict__ idx, const float* __restrict__ w, int B,
    float* __restrict__ part, int32_t* status) {
  constexpr int V = Elem<DT>::kVec;
  const int64_t bag = blockIdx.x;
  const int g = blockIdx.y, groups = gridDim.y;
  const int j0 = g * kGroupRows;
  const int nr = min(kGroupRows, B - j0);
  __shared__ int32_t s_idx[kGroupRows];
  __shared__ float s_w[kGroupRows];
  pdl_launch_dependents();
  pdl_wait();  // idx and w come from the selection
  if (threadIdx.x < nr) {
    int32_t r = idx[bag * B + j0 + threadIdx.x];
    if (r < 0 || r >= n_rows) {
      set_status(status, PKM_ERR_DEVICE);
      r = -1;
    }
    s_idx[threadIdx.x] = r;
    s_w[threadIdx.x] = w[bag * B + j0 + threadIdx.x];
  }
  __syncthreads();
  const int chunks = d / V;
  for (int ch = threadIdx.x; ch < chunks; ch += blockDim.x) {
    const typename Elem<DT>::T* col = table + (int64_t)ch * V;
    uint4 v[kGroupRows];
#pragma unroll
    for (int u = 0; u < kGroupRows; ++u) {
      const int32_t r = u < nr ? s_idx[u] : -1;
      v[u] = r >= 0 ? ldg_nc_16(col + (int64_t)r * d) : make_uint4(0, 0, 0, 0);
    }
    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
#pragma unroll
    for (int u = 0; u < kGroupRows; ++u) {
      if (u < nr && s_idx[u] >= 0) {
        float f[V];
        unpack16<DT>(v[u], f);
        const float wv = s_w[u];
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = fmaf(wv, f[e], acc[e]);
      }
    }
    float* dst = part + ((int64_t)bag * groups + g) * d + (int64_t)ch * V;
#pragma unroll
    for (int e = 0; e < V; e += 4)
      *reinterpret_cast<float4*>(dst + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
  }
}

// grid n_bags: out[bag] = round((sum over groups in order) * gate)
template <pkm_dtype DT, bool GATE>
__global__ void __launch_bounds__(256) embbag_reduce_kernel(
    const float* __restrict__ part, int groups, int d,
    const typename Elem<DT>::T* __restrict__ gate, typename Elem<DT>::T* __restrict__ out) {
  constexpr int V = Elem<DT>::kVec;
  const int64_t bag = blockIdx.x;
  const int chunks = d / V;
  pdl_launch_dependents();
  pdl_wait();  // the partial sums come from the previous kernel
  for (int ch = threadIdx.x; ch < chunks; ch += blockDim.x) {
    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
    for (int g = 0; g < groups; ++g) {
      const float* src = part + ((int64_t)bag * groups + g) * d + (int64_t)ch * V;
#pragma unroll
      for (int e = 0; e < V; e += 4) {
        const float4 p = *reinterpret_cast<const float4*>(src + e);
        acc[e] += p.x;
        acc[e + 1] += p.y;
        acc[e + 2] += p.z;
        acc[e + 3] += p.w;
      }
    }
    if constexpr (GATE) {
      float gv[V];
      unpack16<DT>(ldg_nc_16(gate + bag * d + (int64_t)ch * V), gv);
#pragma unroll
      for (int e = 0; e < V; ++e) acc[e] *= gv[e];
    }
    *reinterpret_cast<uint4*>(out + bag * d + (int64_t)ch * V) = pack16<DT>(acc);
  }
}

size_t embbag_split_workspace(int64_t n_bags, int B, int d) {
  const int groups = (B + kGroupRows - 1) / kGroupRows;
  return (size_t)(n_bags > 0 ? n_bags : 0) * groups * d * sizeof(float);
}

template <pkm_dtype DT>
static cudaError_t launch_split_t(const void* table, int64_t n_rows, int d, const int32_t* idx,
                                  const float* w, int64_t n_bags, int B, const void* gate,
                                  void* out, float* part, int32_t* status, cudaStream_t stream,
                                  bool pdl) {
  using T = typename Elem<DT>::T;
  const int groups = (B + kGroupRows - 1) / kGroupRows;
  const int chunks = d / Elem<DT>::kVec;
  const int threads = min(256, (chunks + 31) / 32 * 32);
  cudaError_t e = launch_maybe_pdl(pdl, embbag_part_kernel<DT>,
                                   dim3((unsigned)n_bags, (unsigned)groups), dim3(threads), 0,
                                   stream, (const T*)table, n_rows, d, idx, w, B, part, status);
  if (e != cudaSuccess) return e;
  if (gate)
    e = launch_maybe_pdl(pdl, embbag_reduce_kernel<DT, true>, dim3((unsigned)n_bags),
                         dim3(threads), 0, stream, (const float*)part, groups, d, (const T*)gate,
                         (T*)out);
  else
    e = launch_maybe_pdl(pdl, embbag_reduce_kernel<DT, false>, dim3((unsigned)n_bags),
                         dim3(threads), 0, stream, (const float*)part, groups, d, (const T*)nullptr,
                         (T*)out);
  note_launch(2);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_embbag_fwd_split(const void* table, int64_t n_rows, int d, pkm_dtype dt,
                                    const int32_t* idx, const float* w, int64_t n_bags, int B,
                                    const void* gate, void* out, float* part, int32_t* status,
                                    cudaStream_t stream, bool pdl) {
  if (n_bags <= 0) return cudaSuccess;
  if (n_bags > 65535) return cudaErrorInvalidValue;
  return dt == PKM_BF16 ? launch_split_t<PKM_BF16>(table, n_rows, d, idx, w, n_bags, B, gate,
                                                   out, part, status, stream, pdl)
                        : launch_split_t<PKM_F32>(table, n_rows, d, idx, w, n_bags, B, gate,
                                                  out, part, status, stream, pdl);
}

}  // namespace pkm
