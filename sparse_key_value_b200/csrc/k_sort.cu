// k_sort.cu -- stable LSD radix sort of (key, value) pairs and an exclusive
// scan, the deterministic ordering step behind the sparse gradient
// reductions (value rows and sub-key rows are summed in sorted order, never
// with atomics).
//
// Per 8-bit digit: (1) per-block digit histograms, (2) one exclusive scan
// over [digit][block], (3) a stable scatter: each block walks its keys in
// order, 256 at a time; within a warp, __match_any_sync finds the lanes with
// the same digit and the lane's rank among them; per-warp counts are
// prefixed in warp order, so equal digits keep their input order.
#include "common.cuh"
#include "kernels.h"

namespace pkm {

namespace {
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRounds = 16;
constexpr int kBlockKeys = kThreads * kRounds;  // 4096 keys per block
constexpr int kRadix = 256;
}  // namespace

__global__ void __launch_bounds__(kThreads) radix_hist_kernel(const uint32_t* __restrict__ keys,
                                                              int64_t n, int shift, int nblocks,
                                                              uint32_t* __restrict__ hist) {
  __shared__ uint32_t h[kRadix];
  h[threadIdx.x] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kBlockKeys;
  for (int r = 0; r < kRounds; ++r) {
    const int64_t i = base + r * kThreads + threadIdx.x;
    if (i < n) atomicAdd(&h[(keys[i] >> shift) & (kRadix - 1)], 1u);
  }
  __syncthreads();
  hist[(int64_t)threadIdx.x * nblocks + blockIdx.x] = h[threadIdx.x];
}

// Exclusive scan of data[0..len) in place by one CTA of 1024 threads;
// *total (optional) receives the sum.  Each thread scans a contiguous run.
__global__ void __launch_bounds__(1024) scan_exclusive_kernel(uint32_t* __restrict__ data,
                                                              int64_t len,
                                                              uint32_t* __restrict__ total,
                                                              int64_t* __restrict__ total64) {
  __shared__ uint32_t warp_sums[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t per = (len + 1023) / 1024;
  const int64_t b = tid * per, e = min(len, b + per);
  uint32_t s = 0;
  for (int64_t i = b; i < e; ++i) s += data[i];
  // block-wide exclusive scan of the per-thread sums
  uint32_t x = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  uint32_t run = x - s + (warp > 0 ? warp_sums[warp - 1] : 0u);
  for (int64_t i = b; i < e; ++i) {
    const uint32_t v = data[i];
    data[i] = run;
    run += v;
  }
  if (tid == 1023) {
    if (total) *total = run;
    if (total64) *total64 = (int64_t)run;
  }
}

__global__ void __launch_bounds__(kThreads) radix_scatter_kernel(
    const uint32_t* __restrict__ keys_in, const uint32_t* __restrict__ vals_in, int64_t n,
    int shift, int nblocks, const uint32_t* __restrict__ offs, uint32_t* __restrict__ keys_out,
    uint32_t* __restrict__ vals_out) {
  __shared__ uint32_t cnt[kRadix];
  __shared__ uint32_t wh[kWarps][kRadix];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  cnt[tid] = offs[(int64_t)tid * nblocks + blockIdx.x];
  const int64_t base = (int64_t)blockIdx.x * kBlockKeys;
  const unsigned lt = (1u << lane) - 1u;
  for (int r = 0; r < kRounds; ++r) {
    for (int w = 0; w < kWarps; ++w) wh[w][tid] = 0;
    __syncthreads();
    const int64_t i = base + r * kThreads + tid;
    const bool valid = i < n;
    uint32_t key = 0, val = 0, d = kRadix;  // invalid lanes form their own group
    if (valid) {
      key = keys_in[i];
      val = vals_in[i];
      d = (key >> shift) & (kRadix - 1);
    }
    const unsigned peers = __match_any_sync(0xffffffffu, d);
    const uint32_t rank = __popc(peers & lt);
    if (valid && rank == 0) wh[warp][d] = __popc(peers);
    __syncthreads();
    {  // prefix over warps, digit `tid`
      uint32_t run = cnt[tid];
      for (int w = 0; w < kWarps; ++w) {
        const uint32_t c = wh[w][tid];
        wh[w][tid] = run;
        run += c;
      }
      cnt[tid] = run;
    }
    __syncthreads();
    if (valid) {
      const uint32_t dst = wh[warp][d] + rank;
      keys_out[dst] = key;
      vals_out[dst] = val;
    }
    __syncthreads();
  }
}

size_t radix_sort_workspace(int64_t n) {
  const int64_t nblocks = (n + kBlockKeys - 1) / kBlockKeys;
  // histogram/offsets + two key and two value buffers
  return (size_t)(kRadix * nblocks + 64) * 4 + (size_t)n * 4 * 4 + 4 * 256;
}

// Sorts (keys_in, vals_in) into (keys_out, vals_out).  The inputs are not
// modified; the workspace holds the ping-pong buffers.
cudaError_t launch_radix_sort(const uint32_t* keys_in, const uint32_t* vals_in, int64_t n,
                              int key_bits, uint32_t* keys_out, uint32_t* vals_out,
                              void* workspace, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const int nblocks = (int)((n + kBlockKeys - 1) / kBlockKeys);
  char* ws = static_cast<char*>(workspace);
  uint32_t* hist = reinterpret_cast<uint32_t*>(ws);
  size_t off = ((size_t)(kRadix * nblocks + 64) * 4 + 255) / 256 * 256;
  uint32_t* ka = reinterpret_cast<uint32_t*>(ws + off);
  uint32_t* va = ka + n;
  uint32_t* kb = va + n;
  uint32_t* vb = kb + n;
  const int passes = (key_bits + 7) / 8;
  const uint32_t* src_k = keys_in;
  const uint32_t* src_v = vals_in;
  for (int p = 0; p < passes; ++p) {
    const bool last = p == passes - 1;
    uint32_t* dk = last ? keys_out : ((p & 1) ? kb : ka);
    uint32_t* dv = last ? vals_out : ((p & 1) ? vb : va);
    radix_hist_kernel<<<nblocks, kThreads, 0, stream>>>(src_k, n, p * 8, nblocks, hist);
    scan_exclusive_kernel<<<1, 1024, 0, stream>>>(hist, (int64_t)kRadix * nblocks, nullptr,
                                                  nullptr);
    radix_scatter_kernel<<<nblocks, kThreads, 0, stream>>>(src_k, src_v, n, p * 8, nblocks, hist,
                                                           dk, dv);
    note_launch(3);
    src_k = dk;
    src_v = dv;
  }
  return cudaGetLastError();
}

cudaError_t launch_scan_exclusive(uint32_t* data, int64_t len, uint32_t* total, int64_t* total64,
                                  cudaStream_t stream) {
  if (len <= 0) return cudaSuccess;
  scan_exclusive_kernel<<<1, 1024, 0, stream>>>(data, len, total, total64);
  note_launch();
  return cudaGetLastError();
}

}  // namespace pkm
