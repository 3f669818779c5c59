// k_embbag.cu -- the softmax-weighted bag gather.
//
// "Memory Layers at Scale" digest, "병렬 EmbeddingBag 구현": the layer's
// core is a weighted EmbeddingBag and it is bound by memory bandwidth, not
// FLOPs.  out[t] = sum_j w[t,j] * table[idx[t,j]], optionally times a gate
// row ("Memory+ 블록": y ⊙ silu(x W1)).
//
// Layout: each thread owns one 16-byte column chunk of a bag's output and
// walks the bag's rows with kUnroll = 16 independent 16-byte loads in flight
// (64 registers, 4 CTAs of 256 threads per SM), so each gathered row is read
// by consecutive threads in full 128-byte lines.  Measured on B200: 16 loads
// in flight at 4 CTAs/SM beat 8 at 8 CTAs/SM by 4-5%.
// fp32 accumulation in row order, one rounding at the store.
#include "common.cuh"
#include "kernels.h"

namespace pkm {

constexpr int kBagThreads = 256;
constexpr int kUnroll = 16;  // independent 16-byte row loads in flight per thread

template <pkm_dtype DT, bool GATE>
__global__ void __launch_bounds__(kBagThreads, 4) embbag_fwd_kernel(
    const typename Elem<DT>::T* __restrict__ table, int64_t n_rows, int d,
    const int32_t* __restrict__ idx, const float* __restrict__ w, int64_t n_bags, int B,
    const typename Elem<DT>::T* __restrict__ gate, typename Elem<DT>::T* __restrict__ out,
    int bags_per_cta, int32_t* status) {
  constexpr int V = Elem<DT>::kVec;
  extern __shared__ unsigned char smem_raw[];
  int32_t* s_idx = reinterpret_cast<int32_t*>(smem_raw);       // [bags_per_cta][B]
  float* s_w = reinterpret_cast<float*>(s_idx + bags_per_cta * B);
  const int chunks = d / V;                        // 16-byte chunks per row
  const int tpb = kBagThreads / bags_per_cta;      // threads per bag
  const int local = threadIdx.x / tpb;
  const int64_t groups = (n_bags + bags_per_cta - 1) / bags_per_cta;

  // persistent: each CTA walks bag groups blockIdx.x, + gridDim.x, ...
  for (int64_t grp = blockIdx.x; grp < groups; grp += gridDim.x) {
    const int64_t bag0 = grp * bags_per_cta;
    __syncthreads();  // the previous group's ids and weights are consumed
    for (int i = threadIdx.x; i < bags_per_cta * B; i += kBagThreads) {
      const int64_t bag = bag0 + i / B;
      int32_t r = -1;
      float wv = 0.f;
      if (bag < n_bags) {
        r = idx[bag0 * B + i];
        wv = w[bag0 * B + i];
        if (r < 0 || r >= n_rows) {
          set_status(status, PKM_ERR_DEVICE);
          r = -1;
        }
      }
      s_idx[i] = r;
      s_w[i] = wv;
    }
    __syncthreads();

    const int64_t bag = bag0 + local;
    if (bag >= n_bags) continue;
    const int32_t* bi = s_idx + local * B;
    const float* bw = s_w + local * B;

    for (int ch = threadIdx.x % tpb; ch < chunks; ch += tpb) {
      float acc[V];
#pragma unroll
      for (int e = 0; e < V; ++e) acc[e] = 0.f;
      const typename Elem<DT>::T* col = table + (int64_t)ch * V;
      int j = 0;
      for (; j + kUnroll <= B; j += kUnroll) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int32_t r = bi[j + u];
          v[u] = r >= 0 ? ldg_nc_16(col + (int64_t)r * d) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          float f[V];
          unpack16<DT>(v[u], f);
          const float wv = bw[j + u];
#pragma unroll
          for (int e = 0; e < V; ++e) acc[e] = fmaf(wv, f[e], acc[e]);
        }
      }
      for (; j < B; ++j) {
        const int32_t r = bi[j];
        if (r < 0) continue;
        float f[V];
        unpack16<DT>(ldg_nc_16(col + (int64_t)r * d), f);
        const float wv = bw[j];
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = fmaf(wv, f[e], acc[e]);
      }
      if constexpr (GATE) {
        float g[V];
        unpack16<DT>(ldg_nc_16(gate + bag * d + (int64_t)ch * V), g);
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] *= g[e];
      }
      *reinterpret_cast<uint4*>(out + bag * d + (int64_t)ch * V) = pack16<DT>(acc);
    }
  }
}

static int sm_count() {
  static int count[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!count[dev]) {
    int c = 0;
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0)
      c = 148;
    count[dev] = c;
  }
  return count[dev];
}

template <pkm_dtype DT, bool GATE>
static cudaError_t launch_embbag_t(const void* table, int64_t n_rows, int d, const int32_t* idx,
                                   const float* w, int64_t n_bags, int B, const void* gate,
                                   void* out, int ctas_per_sm, int32_t* status,
                                   cudaStream_t stream) {
  using T = typename Elem<DT>::T;
  const int chunks = d / Elem<DT>::kVec;
  // several bags per CTA when a row has fewer 16-byte chunks than threads
  int bags_per_cta = 1;
  while (bags_per_cta * 2 * chunks <= kBagThreads &&
         (size_t)bags_per_cta * 2 * B * 8 <= 32768)
    bags_per_cta *= 2;
  const size_t smem = (size_t)bags_per_cta * B * (sizeof(int32_t) + sizeof(float));
  auto fn = embbag_fwd_kernel<DT, GATE>;
  if (smem > 48 * 1024) {
    cudaError_t e =
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int64_t groups = (n_bags + bags_per_cta - 1) / bags_per_cta;
  const int64_t cap = (int64_t)sm_count() * ctas_per_sm;
  dim3 grid((unsigned)(groups < cap ? groups : cap));
  fn<<<grid, kBagThreads, smem, stream>>>((const T*)table, n_rows, d, idx, w, n_bags, B,
                                          (const T*)gate, (T*)out, bags_per_cta, status);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_embbag_fwd(const void* table, int64_t n_rows, int d, pkm_dtype dt,
                              const int32_t* idx, const float* w, int64_t n_bags, int B,
                              const void* gate, void* out, int32_t* status, cudaStream_t stream,
                              int ctas_per_sm) {
  if (n_bags <= 0) return cudaSuccess;
  if (dt == PKM_BF16)
    return gate ? launch_embbag_t<PKM_BF16, true>(table, n_rows, d, idx, w, n_bags, B, gate,
                                                  out, ctas_per_sm, status, stream)
                : launch_embbag_t<PKM_BF16, false>(table, n_rows, d, idx, w, n_bags, B, nullptr,
                                                   out, ctas_per_sm, status, stream);
  return gate ? launch_embbag_t<PKM_F32, true>(table, n_rows, d, idx, w, n_bags, B, gate, out,
                                               ctas_per_sm, status, stream)
              : launch_embbag_t<PKM_F32, false>(table, n_rows, d, idx, w, n_bags, B, nullptr,
                                                out, ctas_per_sm, status, stream);
}

}  // namespace pkm
