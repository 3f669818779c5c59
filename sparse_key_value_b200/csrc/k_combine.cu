// k_combine.cu -- k x k candidate combine, final top-k and softmax.
//
// "모델 안의 메모리", "작동 방식": the best half-keys of each half are combined
// (1,000 x 1,000 cells searched with 2,000 comparisons); figure D shows the
// same on an 8 x 8 grid.  The full score of cell (a, b) is s1[a] + s2[b]
// and its value row is a * n_sub + b.  The weights are a softmax over the k
// kept scores ("작동 방식": a weighted average of the values read).
//
// One warp per (token, head).  With both half lists sorted best first, cell
// (i, j) of the k x k grid is beaten by every cell (i', j') with i' <= i and
// j' <= j, so only the cells with (i+1)(j+1) <= k can be among the k best
// (119 cells for k = 32; all cells when k <= 3).  The warp packs those cells
// as 64-bit keys (order-preserving score bits, then the complemented row
// id, so equal scores favour the smaller id), sorts them with a bitonic
// network spread over its lanes, and keeps the first k.  When the per-half
// lists come in several column splits (each sorted), the warp first merges
// each half's splits pairwise in a binary tree of bitonic merges.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace pkm {

namespace {

constexpr int kCombWarps = 8;

__device__ __forceinline__ uint32_t ordf(float s) {
  uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float unordf(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}
__device__ __forceinline__ uint64_t key_of(float s, int32_t id) {
  return ((uint64_t)ordf(s) << 32) | (uint64_t)(0xffffffffu - (uint32_t)id);
}

__device__ __forceinline__ uint64_t shfl_xor64(uint64_t v, int m) {
  uint32_t lo = (uint32_t)v, hi = (uint32_t)(v >> 32);
  lo = __shfl_xor_sync(0xffffffffu, lo, m);
  hi = __shfl_xor_sync(0xffffffffu, hi, m);
  return ((uint64_t)hi << 32) | lo;
}

// Bitonic sort, descending, of the 32*S keys held as v[s] on lane l at
// position p = s * 32 + l.  S is a power of two.
template <int S>
__device__ __forceinline__ void warp_sort_desc(uint64_t (&v)[S]) {
  const int lane = threadIdx.x & 31;
  constexpr int NT = 32 * S;
#pragma unroll
  for (int size = 2; size <= NT; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride >= 32) {  // partner in another slot of the same lane
        const int ds = stride >> 5;
#pragma unroll
        for (int s = 0; s < S; ++s) {
          if ((s & ds) == 0) {
            const int p = s * 32 + lane;
            const bool desc = (p & size) == 0;
            uint64_t a = v[s], b = v[s + ds];
            const bool sw = desc ? (a < b) : (a > b);
            v[s] = sw ? b : a;
            v[s + ds] = sw ? a : b;
          }
        }
      } else {  // partner on lane ^ stride
#pragma unroll
        for (int s = 0; s < S; ++s) {
          const int p = s * 32 + lane;
          const bool desc = (p & size) == 0;
          const bool lower = (lane & stride) == 0;
          const uint64_t o = shfl_xor64(v[s], stride);
          // the lower position keeps the larger key in a descending block
          const bool keep_max = (lower == desc);
          const uint64_t mx = v[s] > o ? v[s] : o, mn = v[s] > o ? o : v[s];
          v[s] = keep_max ? mx : mn;
        }
      }
    }
  }
}

// a (sorted desc, one key per lane) <- the 32 largest keys of a and b (b also
// sorted desc, one key per lane): the lane-wise maximum of a and reversed b
// is bitonic, and five exchange stages sort it.
__device__ __forceinline__ uint64_t warp_merge_top32(uint64_t a, uint64_t b) {
  const int lane = threadIdx.x & 31;
  uint32_t lo = (uint32_t)b, hi = (uint32_t)(b >> 32);
  lo = __shfl_sync(0xffffffffu, lo, 31 - lane);
  hi = __shfl_sync(0xffffffffu, hi, 31 - lane);
  const uint64_t br = ((uint64_t)hi << 32) | lo;
  uint64_t v = a > br ? a : br;
#pragma unroll
  for (int stride = 16; stride > 0; stride >>= 1) {
    const uint64_t o = shfl_xor64(v, stride);
    const bool lower = (lane & stride) == 0;
    v = lower ? (v > o ? v : o) : (v > o ? o : v);
  }
  return v;
}

// number of candidate cells (i, j), i, j < k, with (i+1)(j+1) <= k
__host__ __device__ __forceinline__ int pruned_cells(int k) {
  int c = 0;
  for (int i = 1; i <= k; ++i) c += k / i;
  return c;
}

// MS: a power of two >= the number of column splits (k <= 32 here).
template <int MS>
__global__ void __launch_bounds__(kCombWarps * 32) combine_kernel(
    const float* __restrict__ hv, const int32_t* __restrict__ hi, int splits, int64_t T, int H,
    int n, int k, int32_t* __restrict__ idx, float* __restrict__ wout) {
  constexpr int S = 4;  // 128 sort slots: the (i+1)(j+1) <= k cells, k <= 32
  __shared__ float lv[kCombWarps][2][32];
  __shared__ int32_t li[kCombWarps][2][32];
  __shared__ uint8_t cell_i[32 * S];
  __shared__ uint8_t cell_j[32 * S];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t th = (int64_t)blockIdx.x * kCombWarps + warp;  // t * H + h
  const int64_t TH2 = T * H * 2;

  // candidate cells (i, j) with (i+1)(j+1) <= k, row-major, shared by the CTA
  const int ncells = pruned_cells(k);
  for (int p = threadIdx.x; p < ncells; p += blockDim.x) {
    int i = 0, acc = 0;
    while (acc + k / (i + 1) <= p) {
      acc += k / (i + 1);
      ++i;
    }
    cell_i[p] = (uint8_t)i;
    cell_j[p] = (uint8_t)(p - acc);
  }
  __syncthreads();
  if (th >= T * H) return;

  // 1. each half's k best: the splits' sorted lists (one key per lane),
  // merged pairwise in a binary tree
  for (int c = 0; c < 2; ++c) {
    const int64_t row = th * 2 + c;
    uint64_t v[MS];
#pragma unroll
    for (int sp = 0; sp < MS; ++sp) {
      v[sp] = 0;
      if (sp < splits && lane < k) {
        const int64_t off = ((int64_t)sp * TH2 + row) * k + lane;
        const int32_t iv = hi[off];
        if (iv != 0x7fffffff) v[sp] = key_of(hv[off], iv);
      }
    }
#pragma unroll
    for (int width = 1; width < MS; width <<= 1) {
#pragma unroll
      for (int a = 0; a + width < MS; a += 2 * width)
        if (a + width < splits) v[a] = warp_merge_top32(v[a], v[a + width]);
    }
    if (lane < k) {
      lv[warp][c][lane] = unordf((uint32_t)(v[0] >> 32));
      li[warp][c][lane] = (int32_t)(0xffffffffu - (uint32_t)v[0]);
    }
  }
  __syncwarp();

  // 2. pack the candidate cells and sort them
  uint64_t v[S];
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const int p = s * 32 + lane;
    v[s] = 0;
    if (p < ncells) {
      const int i = cell_i[p], j = cell_j[p];
      const float Sc = lv[warp][0][i] + lv[warp][1][j];
      const int32_t id = li[warp][0][i] * n + li[warp][1][j];
      v[s] = key_of(Sc, id);
    }
  }
  warp_sort_desc<S>(v);

  // 3. softmax over the k kept scores (entry 0 is the maximum)
  const float S0 = unordf((uint32_t)(v[0] >> 32));  // lane's entry `lane`
  const float m = __shfl_sync(0xffffffffu, S0, 0);
  const float e0 = lane < k ? expf(S0 - m) : 0.f;
  const float z = warp_sum(e0);
  const float inv = 1.0f / z;
  if (lane < k) {
    idx[th * k + lane] = (int32_t)(0xffffffffu - (uint32_t)v[0]);
    wout[th * k + lane] = e0 * inv;
  }
}

// One thread per (token, head), used when each half has a single list.  The
// k x k grid S[i][j] = s1[i] + s2[j] decreases along rows and columns, so its
// cells can be taken best first with a max-heap frontier: start at (0, 0);
// taking (i, j) admits (i, j+1) and, on the first column, (i+1, 0).
// Heap entries are the order-preserving score bits and the cell (i, j); two
// cells with the same score are ordered by their row ids a1[i]*n + b2[j]
// (smaller id first), computed only on such ties.  The CTA's lists form one
// contiguous block of hv / hi and its outputs one contiguous block of idx /
// w: both move through shared memory with coalesced accesses.  Per-thread
// arrays are stored [slot][thread] with a padded row (conflict-free).
constexpr int kThreadCombine = 64;
constexpr int kTcPad = kThreadCombine + 1;  // row stride of the [slot][thread] arrays

__global__ void __launch_bounds__(kThreadCombine) combine_thread_kernel(
    const float* __restrict__ hv, const int32_t* __restrict__ hi, int64_t TH, int n, int k,
    int32_t* __restrict__ idx, float* __restrict__ wout) {
  extern __shared__ unsigned char sm[];
  const int tid = threadIdx.x;
  constexpr int P = kTcPad;
  float* s12 = reinterpret_cast<float*>(sm);                           // [2k][P]: s1, s2
  uint32_t* hk = reinterpret_cast<uint32_t*>(s12 + 2 * k * P);         // heap scores [k+2][P]
  float* mz = reinterpret_cast<float*>(hk + (k + 2) * P);              // [2][P]: max, 1/sum
  uint16_t* ab = reinterpret_cast<uint16_t*>(mz + 2 * P);              // [2k][P]: a1, b2
  uint16_t* hc = ab + 2 * k * P;                                       // heap cells [k+2][P]
  uint16_t* rec = hc + (k + 2) * P;                                    // taken cells [k][P]
  const int64_t th0 = (int64_t)blockIdx.x * kThreadCombine;
  const int nth = (int)min((int64_t)kThreadCombine, TH - th0);  // (t, h) pairs of this CTA

  // 1. the CTA's 2k-long list rows, element e = t_local * 2k + c * k + j
  {
    const int total = nth * 2 * k;
    const float* gv = hv + th0 * 2 * k;
    const int32_t* gi = hi + th0 * 2 * k;
    const bool vec = ((reinterpret_cast<uintptr_t>(gv) | reinterpret_cast<uintptr_t>(gi)) & 15u) == 0;
    const int nvec = vec ? total / 4 : 0;
    for (int q = tid; q < nvec; q += kThreadCombine) {
      const float4 v = reinterpret_cast<const float4*>(gv)[q];
      const int4 w = reinterpret_cast<const int4*>(gi)[q];
      const float vs[4] = {v.x, v.y, v.z, v.w};
      const int32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = 4 * q + u;
        const int tl = e / (2 * k), r = e - tl * 2 * k;
        s12[r * P + tl] = vs[u];
        ab[r * P + tl] = (uint16_t)ws[u];
      }
    }
    for (int e = nvec * 4 + tid; e < total; e += kThreadCombine) {
      const int tl = e / (2 * k), r = e - tl * 2 * k;
      s12[r * P + tl] = gv[e];
      ab[r * P + tl] = (uint16_t)gi[e];
    }
  }
  __syncthreads();

  const float* s1 = s12;
  const float* s2 = s12 + k * P;
  const uint16_t* a1 = ab;
  const uint16_t* b2 = ab + k * P;
  if (tid < nth) {
    auto id_of = [&](int cell) {
      return (int32_t)a1[(cell >> 6) * P + tid] * n + (int32_t)b2[(cell & 63) * P + tid];
    };
    // is entry (s, c) ahead of entry (t, d)?
    auto ahead = [&](uint32_t s, int c, uint32_t t, int d) {
      return s != t ? s > t : id_of(c) < id_of(d);
    };
    auto score_at = [&](int i, int j) { return ordf(s1[i * P + tid] + s2[j * P + tid]); };
    int size = 0;
    auto push = [&](uint32_t key, int cell) {
      int pos = ++size;
      while (pos > 1) {
        const int par = pos >> 1;
        const uint32_t pk = hk[par * P + tid];
        const int pc = hc[par * P + tid];
        if (!ahead(key, cell, pk, pc)) break;
        hk[pos * P + tid] = pk;
        hc[pos * P + tid] = (uint16_t)pc;
        pos = par;
      }
      hk[pos * P + tid] = key;
      hc[pos * P + tid] = (uint16_t)cell;
    };
    push(score_at(0, 0), 0);
    for (int r = 0; r < k; ++r) {
      const int cell = hc[1 * P + tid];
      // pop
      const uint32_t lk = hk[size * P + tid];
      const int lc = hc[size * P + tid];
      --size;
      int pos = 1;
      while (true) {
        int ch = pos * 2;
        if (ch > size) break;
        uint32_t ck = hk[ch * P + tid];
        int cc = hc[ch * P + tid];
        if (ch < size) {
          const uint32_t k2 = hk[(ch + 1) * P + tid];
          const int c2 = hc[(ch + 1) * P + tid];
          if (ahead(k2, c2, ck, cc)) {
            ck = k2;
            cc = c2;
            ++ch;
          }
        }
        if (!ahead(ck, cc, lk, lc)) break;
        hk[pos * P + tid] = ck;
        hc[pos * P + tid] = (uint16_t)cc;
        pos = ch;
      }
      if (size > 0 || pos > 1) {
        hk[pos * P + tid] = lk;
        hc[pos * P + tid] = (uint16_t)lc;
      }
      rec[r * P + tid] = (uint16_t)cell;
      const int i = cell >> 6, j = cell & 63;
      if (j + 1 < k) push(score_at(i, j + 1), i * 64 + j + 1);
      if (j == 0 && i + 1 < k) push(score_at(i + 1, 0), (i + 1) * 64);
    }
    // softmax normaliser over the k kept scores (the first is the maximum)
    const int c0 = rec[tid];
    const float m = s1[(c0 >> 6) * P + tid] + s2[(c0 & 63) * P + tid];
    float z = 0.f;
    for (int r = 0; r < k; ++r) {
      const int c = rec[r * P + tid];
      z += expf(s1[(c >> 6) * P + tid] + s2[(c & 63) * P + tid] - m);
    }
    mz[tid] = m;
    mz[P + tid] = 1.0f / z;
  }
  __syncthreads();

  // 2. the CTA's outputs, element e = t_local * k + r
  {
    const int total = nth * k;
    int32_t* gi = idx + th0 * k;
    float* gw = wout + th0 * k;
    for (int e = tid; e < total; e += kThreadCombine) {
      const int tl = e / k, r = e - tl * k;
      const int c = rec[r * P + tl];
      const int i = c >> 6, j = c & 63;
      const float sc = s1[i * P + tl] + s2[j * P + tl];
      gi[e] = (int32_t)a1[i * P + tl] * n + (int32_t)b2[j * P + tl];
      gw[e] = expf(sc - mz[tl]) * mz[P + tl];
    }
  }
}

}  // namespace

cudaError_t launch_combine(const float* hv, const int32_t* hi, int splits, int64_t T, int H,
                           int n, int k, int32_t* idx, float* w, cudaStream_t stream) {
  const int64_t TH = T * H;
  if (TH <= 0) return cudaSuccess;
  if (splits == 1) {
    const size_t smem = (size_t)kTcPad * ((size_t)k * 8 + (size_t)(k + 2) * 4 + 8 +
                                          (size_t)k * 4 + (size_t)(k + 2) * 2 + (size_t)k * 2);
    if (n > 65536) return cudaErrorInvalidValue;  // sub-key ids are held as 16 bits
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(combine_thread_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return cudaErrorInvalidValue;
    combine_thread_kernel<<<(unsigned)((TH + kThreadCombine - 1) / kThreadCombine),
                            kThreadCombine, smem, stream>>>(hv, hi, TH, n, k, idx, w);
    note_launch();
    return cudaGetLastError();
  }
  // several column splits (tensor-core scoring, k <= 32)
  if (k > 32 || splits > 32) return cudaErrorInvalidValue;
  dim3 grid((unsigned)((TH + kCombWarps - 1) / kCombWarps));
  const int threads = kCombWarps * 32;
  if (splits <= 2)
    combine_kernel<2><<<grid, threads, 0, stream>>>(hv, hi, splits, T, H, n, k, idx, w);
  else if (splits <= 4)
    combine_kernel<4><<<grid, threads, 0, stream>>>(hv, hi, splits, T, H, n, k, idx, w);
  else if (splits <= 8)
    combine_kernel<8><<<grid, threads, 0, stream>>>(hv, hi, splits, T, H, n, k, idx, w);
  else if (splits <= 16)
    combine_kernel<16><<<grid, threads, 0, stream>>>(hv, hi, splits, T, H, n, k, idx, w);
  else
    combine_kernel<32><<<grid, threads, 0, stream>>>(hv, hi, splits, T, H, n, k, idx, w);
  note_launch();
  return cudaGetLastError();
}

}  // namespace pkm
