// k_combine.cu -- k x k candidate combine, final top-k and softmax.
//
// "모델 안의 메모리", "작동 방식": the best half-keys of each half are combined
// (1,000 x 1,000 cells searched with 2,000 comparisons); figure D shows the
// same on an 8 x 8 grid.  The full score of cell (a, b) is s1[a] + s2[b]
// and its value row is a * n_sub + b.  The weights are a softmax over the k
// kept scores ("작동 방식": a weighted average of the values read).
//
// One warp per (token, head).  Both candidate sets are walks over sorted
// queues: queue i yields its entries best first, and the warp repeatedly
// takes the best queue head (a k-way merge), so no k^2 buffer is formed.
#include <math.h>

#include "kernels.h"
#include "warp_topk.cuh"

namespace pkm {

// warp-wide best of (s, id) pairs; returns the winning lane
__device__ __forceinline__ int warp_best(float& s, int32_t& id) {
  const int lane = threadIdx.x & 31;
  int who = lane;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    int32_t i2 = __shfl_xor_sync(0xffffffffu, id, o);
    int w2 = __shfl_xor_sync(0xffffffffu, who, o);
    if (better(s2, i2, s, id)) {
      s = s2;
      id = i2;
      who = w2;
    }
  }
  return who;
}

constexpr int kCombWarps = 8;

// lists: smem per warp: l1v/l1i (half 1), l2v/l2i (half 2), k entries each
__global__ void __launch_bounds__(kCombWarps * 32) combine_kernel(
    const float* __restrict__ hv, const int32_t* __restrict__ hi, int splits, int64_t T, int H,
    int n, int k, int32_t* __restrict__ idx, float* __restrict__ wout) {
  __shared__ float lv[kCombWarps][2][64];
  __shared__ int32_t li[kCombWarps][2][64];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t th = (int64_t)blockIdx.x * kCombWarps + warp;  // t * H + h
  if (th >= T * H) return;
  const int64_t TH2 = T * H * 2;

  // 1. per half: the k best over the split lists (a walk over `splits` queues)
  for (int c = 0; c < 2; ++c) {
    const int64_t row = th * 2 + c;
    if (splits == 1) {
      for (int j = lane; j < k; j += 32) {
        lv[warp][c][j] = hv[row * k + j];
        li[warp][c][j] = hi[row * k + j];
      }
    } else {
      int p = 0;  // this lane's position in its split list (lane < splits)
      for (int r = 0; r < k; ++r) {
        float s = -INFINITY;
        int32_t id = 0x7fffffff;
        if (lane < splits && p < k) {
          const int64_t off = ((int64_t)lane * TH2 + row) * k + p;
          s = hv[off];
          id = hi[off];
        }
        int who = warp_best(s, id);
        if (lane == 0) {
          lv[warp][c][r] = s;
          li[warp][c][r] = id;
        }
        if (lane == who) ++p;
      }
    }
  }
  __syncwarp();

  // 2. k x k combine: queue i (lane i and lane i + 32) walks b over half 2
  float s1a = -INFINITY, s1b = -INFINITY;
  int32_t a1a = 0, a1b = 0;
  if (lane < k) { s1a = lv[warp][0][lane]; a1a = li[warp][0][lane]; }
  if (lane + 32 < k) { s1b = lv[warp][0][lane + 32]; a1b = li[warp][0][lane + 32]; }
  int pa = 0, pb = 0;
  float outS0 = 0.f, outS1 = 0.f;
  int32_t outI0 = 0, outI1 = 0;
  for (int r = 0; r < k; ++r) {
    float sa = -INFINITY, sb = -INFINITY;
    int32_t ia = 0x7fffffff, ib = 0x7fffffff;
    if (lane < k && pa < k) {
      sa = s1a + lv[warp][1][pa];
      ia = a1a * n + li[warp][1][pa];
    }
    if (lane + 32 < k && pb < k) {
      sb = s1b + lv[warp][1][pb];
      ib = a1b * n + li[warp][1][pb];
    }
    const bool takeb = better(sb, ib, sa, ia);
    float s = takeb ? sb : sa;
    int32_t id = takeb ? ib : ia;
    int who = warp_best(s, id);
    if (lane == who) {
      if (takeb) ++pb; else ++pa;
    }
    if (lane == (r & 31)) {
      if (r < 32) { outS0 = s; outI0 = id; } else { outS1 = s; outI1 = id; }
    }
  }

  // 3. softmax over the k kept scores (entry 0 is the maximum)
  const float m = __shfl_sync(0xffffffffu, outS0, 0);
  float e0 = lane < k ? expf(outS0 - m) : 0.f;
  float e1 = lane + 32 < k ? expf(outS1 - m) : 0.f;
  const float z = warp_sum(e0 + e1);
  const float inv = 1.0f / z;
  if (lane < k) {
    idx[th * k + lane] = outI0;
    wout[th * k + lane] = e0 * inv;
  }
  if (lane + 32 < k) {
    idx[th * k + lane + 32] = outI1;
    wout[th * k + lane + 32] = e1 * inv;
  }
}

cudaError_t launch_combine(const float* hv, const int32_t* hi, int splits, int64_t T, int H,
                           int n, int k, int32_t* idx, float* w, cudaStream_t stream) {
  const int64_t TH = T * H;
  if (TH <= 0) return cudaSuccess;
  dim3 grid((unsigned)((TH + kCombWarps - 1) / kCombWarps));
  combine_kernel<<<grid, kCombWarps * 32, 0, stream>>>(hv, hi, splits, T, H, n, k, idx, w);
  note_launch();
  return cudaGetLastError();
}

}  // namespace pkm
