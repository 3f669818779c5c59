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
// lists come in several column splits, the warp first merges each half's
// splits the same way.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace pkm {

namespace {

constexpr int kCombWarps = 8;
constexpr int kMaxSlots = 16;  // keys per lane: up to 512 candidates per warp

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
// position p = s * 32 + l.  S is a power of two <= kMaxSlots.
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

// number of candidate cells (i, j), i, j < k, with (i+1)(j+1) <= k
__host__ __device__ __forceinline__ int pruned_cells(int k) {
  int c = 0;
  for (int i = 1; i <= k; ++i) c += k / i;
  return c;
}

template <int S>
__global__ void __launch_bounds__(kCombWarps * 32) combine_kernel(
    const float* __restrict__ hv, const int32_t* __restrict__ hi, int splits, int64_t T, int H,
    int n, int k, int32_t* __restrict__ idx, float* __restrict__ wout) {
  __shared__ float lv[kCombWarps][2][64];
  __shared__ int32_t li[kCombWarps][2][64];
  __shared__ uint8_t cell_i[32 * kMaxSlots];
  __shared__ uint8_t cell_j[32 * kMaxSlots];
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

  // 1. each half's k best, merging the column splits when there are several
  for (int c = 0; c < 2; ++c) {
    const int64_t row = th * 2 + c;
    if (splits == 1) {
      for (int j = lane; j < k; j += 32) {
        lv[warp][c][j] = hv[row * k + j];
        li[warp][c][j] = hi[row * k + j];
      }
    } else {
      uint64_t v[S];
#pragma unroll
      for (int s = 0; s < S; ++s) {
        const int p = s * 32 + lane;
        const int sp = p / k, j = p - sp * k;
        v[s] = 0;
        if (sp < splits) {
          const int64_t off = ((int64_t)sp * TH2 + row) * k + j;
          const int32_t iv = hi[off];
          if (iv != 0x7fffffff) v[s] = key_of(hv[off], iv);
        }
      }
      warp_sort_desc<S>(v);
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const int p = s * 32 + lane;
        if (p < k) {
          lv[warp][c][p] = unordf((uint32_t)(v[s] >> 32));
          li[warp][c][p] = (int32_t)(0xffffffffu - (uint32_t)v[s]);
        }
      }
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
  const float S1 = unordf((uint32_t)(v[1] >> 32));  // entry `lane + 32`
  const float m = __shfl_sync(0xffffffffu, S0, 0);
  const float e0 = lane < k ? expf(S0 - m) : 0.f;
  const float e1 = lane + 32 < k ? expf(S1 - m) : 0.f;
  const float z = warp_sum(e0 + e1);
  const float inv = 1.0f / z;
  if (lane < k) {
    idx[th * k + lane] = (int32_t)(0xffffffffu - (uint32_t)v[0]);
    wout[th * k + lane] = e0 * inv;
  }
  if (lane + 32 < k) {
    idx[th * k + lane + 32] = (int32_t)(0xffffffffu - (uint32_t)v[1]);
    wout[th * k + lane + 32] = e1 * inv;
  }
}

// One thread per (token, head), used when each half has a single list.  The
// k x k grid S[i][j] = s1[i] + s2[j] decreases along rows and columns, so its
// cells can be taken best first with a max-heap frontier: start at (0, 0);
// taking (i, j) admits (i, j+1) and, on the first column, (i+1, 0).  Lists
// and heap live in shared memory as [slot][thread] (conflict-free).
constexpr int kThreadCombine = 64;

__global__ void __launch_bounds__(kThreadCombine) combine_thread_kernel(
    const float* __restrict__ hv, const int32_t* __restrict__ hi, int64_t TH, int n, int k,
    int32_t* __restrict__ idx, float* __restrict__ wout) {
  extern __shared__ unsigned char sm[];
  const int tid = threadIdx.x;
  constexpr int B = kThreadCombine;
  float* s1 = reinterpret_cast<float*>(sm);          // [k][B]
  float* s2 = s1 + k * B;                            // [k][B]
  int32_t* a1 = reinterpret_cast<int32_t*>(s2 + k * B);
  int32_t* b2 = a1 + k * B;
  uint64_t* hk = reinterpret_cast<uint64_t*>(b2 + k * B);  // heap keys [k+2][B]
  uint16_t* hc = reinterpret_cast<uint16_t*>(hk + (k + 2) * B);  // heap cells
  float* outS = reinterpret_cast<float*>(hc + (k + 2) * B);      // [k][B]
  const int64_t th = (int64_t)blockIdx.x * B + tid;
  if (th >= TH) return;
  for (int j = 0; j < k; ++j) {
    s1[j * B + tid] = hv[(th * 2) * k + j];
    a1[j * B + tid] = hi[(th * 2) * k + j];
    s2[j * B + tid] = hv[(th * 2 + 1) * k + j];
    b2[j * B + tid] = hi[(th * 2 + 1) * k + j];
  }
  auto key_at = [&](int i, int j) {
    return key_of(s1[i * B + tid] + s2[j * B + tid], a1[i * B + tid] * n + b2[j * B + tid]);
  };
  int size = 0;
  auto push = [&](uint64_t key, int cell) {
    int pos = ++size;
    while (pos > 1) {
      const int par = pos >> 1;
      const uint64_t pk = hk[par * B + tid];
      if (pk >= key) break;
      hk[pos * B + tid] = pk;
      hc[pos * B + tid] = hc[par * B + tid];
      pos = par;
    }
    hk[pos * B + tid] = key;
    hc[pos * B + tid] = (uint16_t)cell;
  };
  push(key_at(0, 0), 0);
  for (int r = 0; r < k; ++r) {
    const uint64_t top = hk[1 * B + tid];
    const int cell = hc[1 * B + tid];
    // pop
    const uint64_t lk = hk[size * B + tid];
    const uint16_t lc = hc[size * B + tid];
    --size;
    int pos = 1;
    while (true) {
      int ch = pos * 2;
      if (ch > size) break;
      uint64_t ck = hk[ch * B + tid];
      if (ch < size) {
        const uint64_t rk2 = hk[(ch + 1) * B + tid];
        if (rk2 > ck) {
          ck = rk2;
          ++ch;
        }
      }
      if (ck <= lk) break;
      hk[pos * B + tid] = ck;
      hc[pos * B + tid] = hc[ch * B + tid];
      pos = ch;
    }
    if (size > 0 || pos > 1) {
      hk[pos * B + tid] = lk;
      hc[pos * B + tid] = lc;
    }
    // emit
    idx[th * k + r] = (int32_t)(0xffffffffu - (uint32_t)top);
    outS[r * B + tid] = unordf((uint32_t)(top >> 32));
    const int i = cell >> 6, j = cell & 63;
    if (j + 1 < k) push(key_at(i, j + 1), i * 64 + j + 1);
    if (j == 0 && i + 1 < k) push(key_at(i + 1, 0), (i + 1) * 64);
  }
  // softmax over the k kept scores (entry 0 is the maximum)
  const float m = outS[tid];
  float z = 0.f;
  for (int r = 0; r < k; ++r) z += expf(outS[r * B + tid] - m);
  const float inv = 1.0f / z;
  for (int r = 0; r < k; ++r) wout[th * k + r] = expf(outS[r * B + tid] - m) * inv;
}

}  // namespace

cudaError_t launch_combine(const float* hv, const int32_t* hi, int splits, int64_t T, int H,
                           int n, int k, int32_t* idx, float* w, cudaStream_t stream) {
  const int64_t TH = T * H;
  if (TH <= 0) return cudaSuccess;
  if (splits == 1) {
    const size_t smem = (size_t)kThreadCombine *
                        ((size_t)k * 16 + (size_t)(k + 2) * 10 + (size_t)k * 4);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(combine_thread_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return cudaErrorInvalidValue;
    combine_thread_kernel<<<(unsigned)((TH + kThreadCombine - 1) / kThreadCombine),
                            kThreadCombine, smem, stream>>>(hv, hi, TH, n, k, idx, w);
    note_launch();
    return cudaGetLastError();
  }
  const int need = max(pruned_cells(k), splits > 1 ? splits * k : 0);
  dim3 grid((unsigned)((TH + kCombWarps - 1) / kCombWarps));
  const int threads = kCombWarps * 32;
  if (need <= 64)
    combine_kernel<2><<<grid, threads, 0, stream>>>(hv, hi, splits, T, H, n, k, idx, w);
  else if (need <= 128)
    combine_kernel<4><<<grid, threads, 0, stream>>>(hv, hi, splits, T, H, n, k, idx, w);
  else if (need <= 256)
    combine_kernel<8><<<grid, threads, 0, stream>>>(hv, hi, splits, T, H, n, k, idx, w);
  else if (need <= 512)
    combine_kernel<16><<<grid, threads, 0, stream>>>(hv, hi, splits, T, H, n, k, idx, w);
  else
    return cudaErrorInvalidValue;
  note_launch();
  return cudaGetLastError();
}

}  // namespace pkm
