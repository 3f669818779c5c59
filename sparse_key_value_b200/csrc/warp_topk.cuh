// warp_topk.cuh -- a sorted top-k list (k <= 64) held by one warp in
// registers: lane l owns entries l and l + 32.  Order: larger score first,
// equal scores -> smaller id first.
#pragma once

#include "common.cuh"

namespace pkm {

struct WarpTopK {
  float v0, v1;  // scores of entries lane, lane + 32
  int32_t i0, i1;
  int cnt;       // valid entries (<= k)
  int k;

  __device__ __forceinline__ void init(int k_) {
    k = k_;
    cnt = 0;
    v0 = v1 = -INFINITY;
    i0 = i1 = 0x7fffffff;
  }

  // entry k-1 (meaningful when cnt == k)
  __device__ __forceinline__ void last(float& v, int32_t& i) const {
    int src = (k - 1) & 31;
    float a = __shfl_sync(0xffffffffu, v0, src), b = __shfl_sync(0xffffffffu, v1, src);
    int32_t ia = __shfl_sync(0xffffffffu, i0, src), ib = __shfl_sync(0xffffffffu, i1, src);
    bool hi = (k - 1) >= 32;
    v = hi ? b : a;
    i = hi ? ib : ia;
  }

  // would (s, id) enter the list?  (uniform across the warp given uniform args)
  __device__ __forceinline__ bool admits(float s, int32_t id, float lv, int32_t li) const {
    return cnt < k || better(s, id, lv, li);
  }

  // Insert (s, id), which every lane passes identically.
  __device__ __forceinline__ void insert(float s, int32_t id) {
    const int lane = threadIdx.x & 31;
    bool b0 = lane < cnt && better(v0, i0, s, id);
    bool b1 = lane + 32 < cnt && better(v1, i1, s, id);
    int pos = __popc(__ballot_sync(0xffffffffu, b0)) + __popc(__ballot_sync(0xffffffffu, b1));
    if (pos >= k) return;
    float pv0 = __shfl_up_sync(0xffffffffu, v0, 1), pv1 = __shfl_up_sync(0xffffffffu, v1, 1);
    int32_t pi0 = __shfl_up_sync(0xffffffffu, i0, 1), pi1 = __shfl_up_sync(0xffffffffu, i1, 1);
    float w31 = __shfl_sync(0xffffffffu, v0, 31);
    int32_t j31 = __shfl_sync(0xffffffffu, i0, 31);
    if (lane == 0) {
      pv1 = w31;
      pi1 = j31;
    }
    const int e0 = lane, e1 = lane + 32;
    if (e0 > pos) { v0 = pv0; i0 = pi0; } else if (e0 == pos) { v0 = s; i0 = id; }
    if (e1 > pos) { v1 = pv1; i1 = pi1; } else if (e1 == pos) { v1 = s; i1 = id; }
    cnt = cnt + 1 < k ? cnt + 1 : k;
  }

  // Offer one candidate per lane (valid[lane] says whether it exists); all
  // admitted candidates are inserted.  The result does not depend on the
  // order of insertion because the order is total.
  __device__ __forceinline__ void offer(bool valid, float s, int32_t id) {
    float lv;
    int32_t li;
    last(lv, li);
    unsigned m = __ballot_sync(0xffffffffu, valid && admits(s, id, lv, li));
    while (m) {
      int src = __ffs(m) - 1;
      m &= m - 1;
      float cs = __shfl_sync(0xffffffffu, s, src);
      int32_t ci = __shfl_sync(0xffffffffu, id, src);
      insert(cs, ci);
    }
  }

  // write entries 0..k-1
  __device__ __forceinline__ void store(float* v, int32_t* ids) const {
    const int lane = threadIdx.x & 31;
    if (lane < k) { v[lane] = v0; ids[lane] = i0; }
    if (lane + 32 < k) { v[lane + 32] = v1; ids[lane + 32] = i1; }
  }
};

}  // namespace pkm
