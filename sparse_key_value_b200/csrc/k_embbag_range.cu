// k_embbag_range.cu -- partial bags over one shard of a value table sharded
// by rows across GPUs ("Memory Layers at Scale" digest: memories of 64B and
// 128B parameters exceed one GPU).  The shard's owner sums, for the tokens of
// every rank, the selected rows it holds; a reduce-scatter over tokens adds
// the shards' partials (sparse_key_value_b200/sharded.py).
#include "common.cuh"
#include "kernels.h"

namespace pkm {

namespace {

constexpr int kBagThreads = 256;
constexpr int kUnroll = 8;  // independent 16-byte row loads in flight per thread

int sm_count_range() {
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

}  // namespace

// The partial bag of one shard of a row-sharded table: only the rows in
// [row_lo, row_lo + n_local) contribute, read from the shard's own table at
// r - row_lo; the others are skipped (another shard holds them).  fp32
// output, so that the shards' partials can be summed without an extra
// rounding.  One CTA per bag (persistent): the first warp compacts the
// bag's entries held here into shared memory (ballot, j order kept), then
// every thread sums its 16-byte column over them with 8 row loads in
// flight.
template <pkm_dtype DT>
__global__ void __launch_bounds__(kBagThreads, 4) embbag_range_kernel(
    const typename Elem<DT>::T* __restrict__ table, int64_t row_lo, int64_t n_local, int d,
    const int32_t* __restrict__ idx, const float* __restrict__ w, int64_t n_bags, int B,
    float* __restrict__ out) {
  constexpr int V = Elem<DT>::kVec;
  extern __shared__ unsigned char smem_raw[];
  int32_t* s_idx = reinterpret_cast<int32_t*>(smem_raw);  // [B] the bag's rows held here, in j order
  float* s_w = reinterpret_cast<float*>(s_idx + B);
  __shared__ int s_count;
  const int chunks = d / V;
  for (int64_t bag = blockIdx.x; bag < n_bags; bag += gridDim.x) {
    __syncthreads();  // the previous bag's list is consumed
    if (threadIdx.x < 32) {
      // the first warp keeps, in j order, the entries whose row this shard holds
      const int lane = threadIdx.x;
      int base = 0;
      for (int i0 = 0; i0 < B; i0 += 32) {
        const int i = i0 + lane;
        int64_t r = -1;
        float wv = 0.f;
        if (i < B) {
          r = (int64_t)idx[bag * B + i] - row_lo;
          wv = w[bag * B + i];
        }
        const bool mine = i < B && r >= 0 && r < n_local;
        const unsigned m = __ballot_sync(0xffffffffu, mine);
        if (mine) {
          const int pos = base + __popc(m & ((1u << lane) - 1u));
          s_idx[pos] = (int32_t)r;
          s_w[pos] = wv;
        }
        base += __popc(m);
      }
      if (lane == 0) s_count = base;
    }
    __syncthreads();
    const int cnt = s_count;
    for (int ch = threadIdx.x; ch < chunks; ch += kBagThreads) {
      float acc[V];
#pragma unroll
      for (int e = 0; e < V; ++e) acc[e] = 0.f;
      const typename Elem<DT>::T* col = table + (int64_t)ch * V;
      for (int j = 0; j < cnt; j += kUnroll) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
          v[u] = j + u < cnt ? ldg_nc_16(col + (int64_t)s_idx[j + u] * d) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          if (j + u >= cnt) break;
          float f[V];
          unpack16<DT>(v[u], f);
          const float wv = s_w[j + u];
#pragma unroll
          for (int e = 0; e < V; ++e) acc[e] = fmaf(wv, f[e], acc[e]);
        }
      }
      float* o = out + bag * d + (int64_t)ch * V;
#pragma unroll
      for (int e = 0; e < V; e += 4)
        __stcs(reinterpret_cast<float4*>(o + e), make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]));
    }
  }
}

cudaError_t launch_embbag_range(const void* table, int64_t row_lo, int64_t n_local, int d,
                                pkm_dtype dt, const int32_t* idx, const float* w, int64_t n_bags,
                                int B, float* out, cudaStream_t stream) {
  if (n_bags <= 0) return cudaSuccess;
  const size_t smem = (size_t)B * (sizeof(int32_t) + sizeof(float));
  const int64_t cap = (int64_t)sm_count_range() * 4;
  dim3 grid((unsigned)(n_bags < cap ? n_bags : cap));
  if (dt == PKM_BF16) {
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(embbag_range_kernel<PKM_BF16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return cudaErrorInvalidValue;
    embbag_range_kernel<PKM_BF16><<<grid, kBagThreads, smem, stream>>>(
        (const __nv_bfloat16*)table, row_lo, n_local, d, idx, w, n_bags, B, out);
  } else {
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(embbag_range_kernel<PKM_F32>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return cudaErrorInvalidValue;
    embbag_range_kernel<PKM_F32><<<grid, kBagThreads, smem, stream>>>(
        (const float*)table, row_lo, n_local, d, idx, w, n_bags, B, out);
  }
  note_launch();
  return cudaGetLastError();
}

}  // namespace pkm
