// k_sort.cu -- stable LSD radix sort of (key, value) pairs and an exclusive
// scan, the deterministic ordering step behind the sparse gradient
// reductions (value rows and sub-key rows are summed in sorted order, never
// with atomics).
//
// Per 8-bit digit: (1) per-block digit histograms, (2) an exclusive scan of
// each digit's row of block counts (one CTA per digit) and of the digit
// totals, (3) a stable scatter: each block walks its keys in
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

// Exclusive scan of data[0..len) in place by one CTA of 1024 threads, in
// coalesced tiles of 4096 (four consecutive values per thread); *total /
// *total64 (optional) receive the sum.
__device__ __forceinline__ uint32_t block_exclusive_scan_1024(uint32_t x, uint32_t* warp_sums,
                                                              uint32_t& block_total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t v = lane < (int)(blockDim.x >> 5) ? warp_sums[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    warp_sums[lane] = v;  // inclusive over warps
  }
  __syncthreads();
  block_total = warp_sums[(blockDim.x >> 5) - 1];
  const uint32_t before = warp > 0 ? warp_sums[warp - 1] : 0u;
  __syncthreads();  // warp_sums is reused by the next call
  return before + incl - x;
}

__global__ void __launch_bounds__(1024) scan_exclusive_kernel(uint32_t* __restrict__ data,
                                                              int64_t len,
                                                              uint32_t* __restrict__ total,
                                                              int64_t* __restrict__ total64) {
  __shared__ uint32_t warp_sums[32];
  uint32_t carry = 0;
  for (int64_t base = 0; base < len; base += 4096) {
    const int64_t i0 = base + (int64_t)threadIdx.x * 4;
    uint32_t v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = i0 + e < len ? data[i0 + e] : 0u;
    const uint32_t sum = v[0] + v[1] + v[2] + v[3];
    uint32_t tile_total;
    uint32_t run = carry + block_exclusive_scan_1024(sum, warp_sums, tile_total);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (i0 + e < len) data[i0 + e] = run;
      run += v[e];
    }
    carry += tile_total;
  }
  if (threadIdx.x == 0) {
    if (total) *total = carry;
    if (total64) *total64 = (int64_t)carry;
  }
}

// Per-digit scan of the block histograms hist[d][0..nblocks): CTA d replaces
// its row by the exclusive prefix over blocks and writes the digit total.
__global__ void __launch_bounds__(1024) radix_digit_scan_kernel(uint32_t* __restrict__ hist,
                                                                int nblocks,
                                                                uint32_t* __restrict__ totals) {
  __shared__ uint32_t warp_sums[32];
  uint32_t* row = hist + (int64_t)blockIdx.x * nblocks;
  uint32_t carry = 0;
  for (int base = 0; base < nblocks; base += 1024) {
    const int i = base + threadIdx.x;
    const uint32_t v = i < nblocks ? row[i] : 0u;
    uint32_t tile_total;
    const uint32_t ex = block_exclusive_scan_1024(v, warp_sums, tile_total);
    if (i < nblocks) row[i] = carry + ex;
    carry += tile_total;
  }
  if (threadIdx.x == 0) totals[blockIdx.x] = carry;
}

// Exclusive scan of the kRadix digit totals (in place).
__global__ void __launch_bounds__(kRadix) radix_base_scan_kernel(uint32_t* __restrict__ totals) {
  __shared__ uint32_t t[kRadix];
  t[threadIdx.x] = totals[threadIdx.x];
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t run = 0;
    for (int d = 0; d < kRadix; ++d) {
      const uint32_t v = t[d];
      t[d] = run;
      run += v;
    }
  }
  __syncthreads();
  totals[threadIdx.x] = t[threadIdx.x];
}

__global__ void __launch_bounds__(kThreads) radix_scatter_kernel(
    const uint32_t* __restrict__ keys_in, const uint32_t* __restrict__ vals_in, int64_t n,
    int shift, int nblocks, const uint32_t* __restrict__ offs,
    const uint32_t* __restrict__ digit_base, uint32_t* __restrict__ keys_out,
    uint32_t* __restrict__ vals_out) {
  __shared__ uint32_t cnt[kRadix];
  __shared__ uint32_t wh[kWarps][kRadix];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  cnt[tid] = digit_base[tid] + offs[(int64_t)tid * nblocks + blockIdx.x];
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
  // histogram/offsets, digit bases, two key and two value buffers
  return (size_t)(kRadix * nblocks + 64) * 4 + 256 + kRadix * 4 + (size_t)n * 4 * 4 + 4 * 256;
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
  uint32_t* dbase = reinterpret_cast<uint32_t*>(ws + off);
  off += (kRadix * 4 + 255) / 256 * 256;
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
    radix_digit_scan_kernel<<<kRadix, 1024, 0, stream>>>(hist, nblocks, dbase);
    radix_base_scan_kernel<<<1, kRadix, 0, stream>>>(dbase);
    radix_scatter_kernel<<<nblocks, kThreads, 0, stream>>>(src_k, src_v, n, p * 8, nblocks, hist,
                                                           dbase, dk, dv);
    note_launch(4);
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
