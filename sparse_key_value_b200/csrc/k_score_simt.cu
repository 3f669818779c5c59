// k_score_simt.cu -- qk-normalisation factors and the SIMT-core sub-key
// scoring with fused per-half top-k.
//
// "Memory Layers at Scale" digest, "Memory+ 블록": qk-normalization, read
// here as L2 normalisation of every query half and sub-key row (clamped at
// 1e-12).  "모델 안의 메모리", "작동 방식": each half of the query is compared
// with every half-key of its table and the best are kept.
//
// The SIMT path serves fp32 inputs and k > 32; bf16 with k <= 32 runs on the
// tensor cores (k_score_tc.cu).  Scores are formed exactly as
//   s = sqrt(d_half) * rq * rk[a] * <q_c, K_c[a]>
// with the raw (unnormalised) inputs in the dot product and fp32 throughout.
#include <math.h>

#include "kernels.h"
#include "warp_topk.cuh"

namespace pkm {

// One warp per ROWS consecutive rows of at most 32 * NVL 16-byte vectors:
// every lane issues its loads for all ROWS rows before reducing, so about
// eight 16-byte loads per lane are in flight.
template <pkm_dtype DT, int NVL, int ROWS>
__global__ void __launch_bounds__(256) row_rnorm_kernel(const typename Elem<DT>::T* __restrict__ x,
                                                        int64_t rows, int d,
                                                        float* __restrict__ r) {
  constexpr int V = Elem<DT>::kVec;
  const int lane = threadIdx.x & 31;
  const int64_t row0 = ((int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32) * ROWS;
  if (row0 >= rows) return;
  const int nv = d / V;  // vectors per row
  uint4 v[ROWS][NVL];
#pragma unroll
  for (int q = 0; q < ROWS; ++q)
#pragma unroll
    for (int u = 0; u < NVL; ++u) {
      const int c = lane + 32 * u;
      if (row0 + q < rows && c < nv) v[q][u] = ldg_nc_16(x + (row0 + q) * d + (int64_t)c * V);
    }
#pragma unroll
  for (int q = 0; q < ROWS; ++q) {
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < NVL; ++u) {
      const int c = lane + 32 * u;
      if (row0 + q < rows && c < nv) {
        float f[V];
        unpack16<DT>(v[q][u], f);
#pragma unroll
        for (int e = 0; e < V; ++e) ss = fmaf(f[e], f[e], ss);
      }
    }
    ss = warp_sum(ss);
    if (lane == 0 && row0 + q < rows) r[row0 + q] = 1.0f / fmaxf(sqrtf(ss), kNormEps);
  }
}

template <pkm_dtype DT, int NVL>
static void launch_rnorm_t(const void* x, int64_t rows, int d, float* r, cudaStream_t stream) {
  constexpr int ROWS = NVL >= 8 ? 1 : 8 / NVL;
  const int warps = 8;
  const int64_t groups = (rows + ROWS - 1) / ROWS;
  dim3 grid((unsigned)((groups + warps - 1) / warps));
  row_rnorm_kernel<DT, NVL, ROWS><<<grid, warps * 32, 0, stream>>>(
      (const typename Elem<DT>::T*)x, rows, d, r);
}

// d <= 2048 (bf16) / 1024 (fp32): the forward and backward validate d_half.
cudaError_t launch_row_rnorm(const void* x, pkm_dtype dt, int64_t rows, int d, float* r,
                             cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const int V = dt == PKM_BF16 ? 8 : 4;
  const int nvl = (d / V + 31) / 32;
  if (nvl > 16) return cudaErrorInvalidValue;
#define PKM_RNORM(T_)                                            \
  if (nvl <= 1) launch_rnorm_t<T_, 1>(x, rows, d, r, stream);   \
  else if (nvl <= 2) launch_rnorm_t<T_, 2>(x, rows, d, r, stream); \
  else if (nvl <= 4) launch_rnorm_t<T_, 4>(x, rows, d, r, stream); \
  else if (nvl <= 8) launch_rnorm_t<T_, 8>(x, rows, d, r, stream); \
  else launch_rnorm_t<T_, 16>(x, rows, d, r, stream)
  if (dt == PKM_BF16) {
    PKM_RNORM(PKM_BF16);
  } else {
    PKM_RNORM(PKM_F32);
  }
#undef PKM_RNORM
  note_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------------
// CTA = 8 warps = 8 tokens of one (head, half).  The 256 threads score 256
// sub-keys at a time against the 8 query halves staged in shared memory;
// each warp then folds its token's 256 new scores into its top-k list.
constexpr int kSimtTok = 8;
constexpr int kSimtCols = 256;

template <pkm_dtype DT>
__global__ void __launch_bounds__(256) score_topk_simt_kernel(
    const typename Elem<DT>::T* __restrict__ q, const typename Elem<DT>::T* __restrict__ K,
    int64_t T, int H, int dh, int n, int k, const float* __restrict__ rq,
    const float* __restrict__ rk, float* __restrict__ hv, int32_t* __restrict__ hi) {
  constexpr int V = Elem<DT>::kVec;
  extern __shared__ float smem[];
  float* qs = smem;                          // [8][dh]
  float* sc = smem + kSimtTok * dh;          // [8][256]
  const int hc = blockIdx.y;                 // h * 2 + c
  const int h = hc >> 1;
  const int64_t t0 = (int64_t)blockIdx.x * kSimtTok;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float scale = sqrtf((float)dh);

  // stage the 8 query halves as fp32
  for (int i = threadIdx.x; i < kSimtTok * dh; i += blockDim.x) {
    int tt = i / dh, e = i - tt * dh;
    int64_t t = t0 + tt;
    float v = 0.f;
    if (t < T) {
      const typename Elem<DT>::T* p = q + ((t * H) * 2 + hc) * (int64_t)dh + e;
      if constexpr (DT == PKM_BF16) v = __bfloat162float(*p); else v = *p;
    }
    qs[i] = v;
  }
  float rowf[kSimtTok];
#pragma unroll
  for (int i = 0; i < kSimtTok; ++i) {
    int64_t t = t0 + i;
    rowf[i] = t < T ? scale * rq[(t * H) * 2 + hc] : 0.f;
  }
  __syncthreads();

  WarpTopK top;
  top.init(k);
  const typename Elem<DT>::T* Kc = K + (int64_t)hc * n * dh;
  const float* rkc = rk + (int64_t)hc * n;

  for (int a0 = 0; a0 < n; a0 += kSimtCols) {
    const int a = a0 + threadIdx.x;
    float acc[kSimtTok];
#pragma unroll
    for (int i = 0; i < kSimtTok; ++i) acc[i] = 0.f;
    if (a < n) {
      const typename Elem<DT>::T* kr = Kc + (int64_t)a * dh;
      for (int e = 0; e < dh; e += V) {
        float f[V];
        unpack16<DT>(*reinterpret_cast<const uint4*>(kr + e), f);
#pragma unroll
        for (int i = 0; i < kSimtTok; ++i) {
#pragma unroll
          for (int u = 0; u < V; ++u) acc[i] = fmaf(f[u], qs[i * dh + e + u], acc[i]);
        }
      }
      const float rka = rkc[a];
#pragma unroll
      for (int i = 0; i < kSimtTok; ++i) sc[i * kSimtCols + threadIdx.x] = acc[i] * rka * rowf[i];
    }
    __syncthreads();
    // warp `warp` folds token warp's scores into its list
    for (int j = 0; j < kSimtCols; j += 32) {
      int col = a0 + j + lane;
      bool valid = col < n;
      float s = valid ? sc[warp * kSimtCols + j + lane] : -INFINITY;
      top.offer(valid, s, col);
    }
    __syncthreads();
  }
  const int64_t t = t0 + warp;
  if (t < T) {
    const int64_t row = (t * H) * 2 + hc;
    top.store(hv + row * k, hi + row * k);
  }
  (void)h;
}

cudaError_t launch_score_topk_simt(const void* q, const void* K, pkm_dtype dt, int64_t T,
                                   int H, int dh, int n, int k, const float* rq,
                                   const float* rk, float* hv, int32_t* hi,
                                   cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  dim3 grid((unsigned)((T + kSimtTok - 1) / kSimtTok), (unsigned)(H * 2));
  size_t smem = sizeof(float) * (size_t)kSimtTok * (dh + kSimtCols);
  cudaError_t e;
  if (dt == PKM_BF16) {
    auto fn = score_topk_simt_kernel<PKM_BF16>;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    fn<<<grid, 256, smem, stream>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)K, T, H, dh,
                                    n, k, rq, rk, hv, hi);
    note_launch();
  } else {
    auto fn = score_topk_simt_kernel<PKM_F32>;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    fn<<<grid, 256, smem, stream>>>((const float*)q, (const float*)K, T, H, dh, n, k, rq, rk,
                                    hv, hi);
    note_launch();
  }
  return cudaGetLastError();
}

}  // namespace pkm
