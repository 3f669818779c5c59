// warp_sort32.cuh -- 32 candidates held one per lane of a warp (an fp32
// score and a 32-bit id), sorted and merged by bitonic exchange networks
// across the lanes, and the k x k combine of two such sorted lists.
//
// "Memory Layers at Scale" digest, "Product-key 검색", and "모델 안의 메모리",
// "작동 방식": the best sub-keys of the two halves are combined; a full key's
// score is the sum of its halves' scores.
//
// Exactly equal scores are ties and may come out in either order.
#pragma once

#include <math.h>

#include "common.cuh"

namespace pkm {

// exchange with lane ^ partner_mask keeping the larger (keep_max) or the
// smaller score; the id moves when the score does.  Written as fp32 max /
// min and two selects: the form that compiles to straight-line code (a
// comparison chosen per lane measured 8x slower per sort on B200).
__device__ __forceinline__ void warp_cas(float& v, uint32_t& id, int partner_mask,
                                         bool keep_max) {
  const float o = __shfl_xor_sync(0xffffffffu, v, partner_mask);
  const uint32_t oi = __shfl_xor_sync(0xffffffffu, id, partner_mask);
  const float nv = keep_max ? fmaxf(v, o) : fminf(v, o);
  id = nv != v ? oi : id;
  v = nv;
}

// 32 keys, one per lane, sorted descending across the warp
__device__ __forceinline__ void warp_sort32_desc(float& v, uint32_t& id) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
    const bool desc = (lane & size) == 0;
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1)
      warp_cas(v, id, stride, ((lane & stride) == 0) == desc);
  }
}

// (v, id) <- top 32 of (v, id) u (w, wi), both sorted descending across the
// warp: the larger of v[l] and w[31 - l] is a bitonic sequence holding the
// top 32, five exchange stages sort it
__device__ __forceinline__ void warp_merge32_desc(float& v, uint32_t& id, float w,
                                                  uint32_t wi) {
  const int lane = threadIdx.x & 31;
  const float r = __shfl_sync(0xffffffffu, w, 31 - lane);
  const uint32_t ri = __shfl_sync(0xffffffffu, wi, 31 - lane);
  const float nv = fmaxf(v, r);
  id = nv != v ? ri : id;
  v = nv;
#pragma unroll
  for (int stride = 16; stride > 0; stride >>= 1) warp_cas(v, id, stride, (lane & stride) == 0);
}

// The cells (i, j) of a k x k grid with (i+1)(j+1) <= k, row-major, as
// i << 8 | j; slot e of 128 (0xffff past the last: at most 119 cells for
// k <= 32).
__device__ __forceinline__ uint16_t topk_cell(int e, int k) {
  int rem = e, i = 0;
  for (; i < k; ++i) {
    const int m = k / (i + 1);
    if (rem < m) break;
    rem -= m;
  }
  return i < k ? (uint16_t)((i << 8) | rem) : (uint16_t)0xffffu;
}

// One warp per (token, head).  Lane l holds entry l of each half's sorted
// list of the k best (v1, a1: scores and positions of the first half; v2, b2
// of the second; entries past k are -inf).  In the k x k grid
// S[i][j] = v1[i] + v2[j] (non-increasing along rows and columns) cell
// (i, j) is beaten by the (i+1)(j+1) - 1 cells above and left of it, so only
// the cells with (i+1)(j+1) <= k can be among the k best.  Lane l takes
// cells l, l+32, l+64, l+96 of `cells`; each group of 32 is sorted across
// the warp, the four groups are merged keeping the top 32, and lane l < k
// writes the l-th best: row id a*n + b and its softmax weight over the k
// kept scores.  With k = 32 the first group is the grid's first row
// v1[0] + v2[j], j = 0..31, already in order (fp32 addition of a common
// term keeps the order of the v2[j]): its sort is skipped.
template <bool K32 = false>
__device__ __forceinline__ void combine_lists_warp(float v1, uint32_t a1, float v2, uint32_t b2,
                                                   const uint16_t* cells, int n, int k,
                                                   int32_t* __restrict__ idx_out,
                                                   float* __restrict__ w_out) {
  const int lane = threadIdx.x & 31;
  float v[4];
  uint32_t id[4];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const uint32_t cell = cells[lane + 32 * g];
    const bool valid = cell != 0xffffu;
    const int i = valid ? (int)(cell >> 8) : 0, j = valid ? (int)(cell & 255u) : 0;
    const float si = __shfl_sync(0xffffffffu, v1, i);
    const float sj = __shfl_sync(0xffffffffu, v2, j);
    const uint32_t ai = __shfl_sync(0xffffffffu, a1, i);
    const uint32_t bj = __shfl_sync(0xffffffffu, b2, j);
    v[g] = valid ? (si + sj) + 0.0f : -INFINITY;  // + 0: -0 -> +0
    id[g] = valid ? ai * (uint32_t)n + bj : 0xffffffffu;
  }
#pragma unroll
  for (int g = K32 ? 1 : 0; g < 4; ++g) warp_sort32_desc(v[g], id[g]);
  warp_merge32_desc(v[0], id[0], v[1], id[1]);
  warp_merge32_desc(v[2], id[2], v[3], id[3]);
  warp_merge32_desc(v[0], id[0], v[2], id[2]);
  // softmax over the k kept scores; lane 0 holds the maximum
  const float mx = __shfl_sync(0xffffffffu, v[0], 0);
  const float e = lane < k ? expf(v[0] - mx) : 0.f;
  float z = e;
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) z += __shfl_xor_sync(0xffffffffu, z, m);
  if (lane < k) {
    idx_out[lane] = (int32_t)id[0];
    w_out[lane] = e / z;
  }
}

}  // namespace pkm
