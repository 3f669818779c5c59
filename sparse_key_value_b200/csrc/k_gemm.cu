// k_gemm.cu -- dense pieces of the Memory+ block ("Memory Layers at
// Scale" digest, "Memory+ 블록": out = (y ⊙ silu(x W1)) W2).
//
// The GEMM runs on the tensor cores (k_gemm_tc.cu) when the shape allows it,
// else on this SIMT kernel; both read every operand in the layout the caller
// holds it (K-major, or MN-major for a weight [d_in, d_out] used as x W and
// for the tokens of a weight gradient x^T dy).  The transpose kernel serves
// the backward's small steps that want a transposed copy.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace pkm {

// dst[c][r] = src[r][c] for a rows x cols bf16 matrix, dst rows ld long
// (ld >= rows; entries rows..ld-1 are written as zeros).  64 x 64 tiles: rows
// are read and written as 16-byte vectors (coalesced 128-byte segments), the
// transpose itself happens element-wise in shared memory.
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const __nv_bfloat16* __restrict__ src,
                                                             int rows, int cols,
                                                             __nv_bfloat16* __restrict__ dst,
                                                             int ld) {
  __shared__ uint16_t tile[64][65];
  const int c0 = blockIdx.x * 64, r0 = blockIdx.y * 64;
  const int tid = threadIdx.x;
  const uint16_t* s16 = reinterpret_cast<const uint16_t*>(src);
  const bool vec_src = (cols % 8) == 0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = (tid >> 3) + 32 * h;  // tile row: source row r0 + i
    const int q = tid & 7;              // 16-byte vector of the row
    const int r = r0 + i, c = c0 + 8 * q;
    uint16_t v[8];
    if (r < rows && vec_src && c + 8 <= cols) {
      const uint4 u = *reinterpret_cast<const uint4*>(s16 + (int64_t)r * cols + c);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[2 * e] = (uint16_t)(w[e] & 0xffffu);
        v[2 * e + 1] = (uint16_t)(w[e] >> 16);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e)
        v[e] = (r < rows && c + e < cols) ? s16[(int64_t)r * cols + c + e] : (uint16_t)0;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) tile[i][8 * q + e] = v[e];
  }
  __syncthreads();
  const bool vec_dst = (ld % 8) == 0;
  uint16_t* d16 = reinterpret_cast<uint16_t*>(dst);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int j = (tid >> 3) + 32 * h;  // tile column: destination row c0 + j
    const int q = tid & 7;
    const int c = c0 + j, r = r0 + 8 * q;
    if (c >= cols) continue;
    uint16_t v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = tile[8 * q + e][j];
    uint16_t* d = d16 + (int64_t)c * ld + r;
    if (vec_dst && r + 8 <= ld) {
      *reinterpret_cast<uint4*>(d) =
          make_uint4(v[0] | ((uint32_t)v[1] << 16), v[2] | ((uint32_t)v[3] << 16),
                     v[4] | ((uint32_t)v[5] << 16), v[6] | ((uint32_t)v[7] << 16));
    } else {
      for (int e = 0; e < 8 && r + e < ld; ++e) d[e] = v[e];
    }
  }
}

cudaError_t launch_transpose_bf16(const void* src, int rows, int cols, void* dst,
                                  cudaStream_t stream, int ld) {
  if (ld <= 0) ld = rows;
  if (rows <= 0 || cols <= 0 || ld < rows) return rows <= 0 || cols <= 0 ? cudaSuccess
                                                                          : cudaErrorInvalidValue;
  dim3 grid((unsigned)((cols + 63) / 64), (unsigned)((ld + 63) / 64));
  transpose_bf16_kernel<<<grid, 256, 0, stream>>>((const __nv_bfloat16*)src, rows, cols,
                                                  (__nv_bfloat16*)dst, ld);
  note_launch();
  return cudaGetLastError();
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + expf(-z)); }

// C[M,N] = epi(sum_k A[m,k] B[n,k]); 64x64 tile, 256 threads, 4x4 each.
// out_mode: 0 bf16 (epi applied), 1 fp32, 2 fp32 accumulate.  a_mn / b_mn:
// A held as [K][M] / B as [K][N].
__global__ void __launch_bounds__(256) gemm_simt_kernel(const __nv_bfloat16* __restrict__ A,
                                                        const __nv_bfloat16* __restrict__ B,
                                                        int64_t M, int N, int K, int epi,
                                                        int out_mode, bool a_mn, bool b_mn,
                                                        void* __restrict__ Cv) {
  __shared__ float As[16][64 + 1];
  __shared__ float Bs[16][64 + 1];
  const int64_t m0 = (int64_t)blockIdx.y * 64;
  const int n0 = blockIdx.x * 64;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 64 * 16; i += 256) {
      int r = i / 16, kk = i % 16;
      int64_t m = m0 + r;
      int nn = n0 + r;
      const int64_t kq = k0 + kk;
      As[kk][r] = (m < M && kq < K) ? __bfloat162float(A[a_mn ? kq * M + m : m * K + kq]) : 0.f;
      Bs[kk][r] = (nn < N && kq < K) ? __bfloat162float(B[b_mn ? kq * N + nn : (int64_t)nn * K + kq])
                                     : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int64_t m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int nn = n0 + tx * 4 + j;
      if (nn >= N) continue;
      float v = acc[i][j];
      if (out_mode == 0) {
        if (epi == 1) v = silu_f(v);
        static_cast<__nv_bfloat16*>(Cv)[m * N + nn] = __float2bfloat16_rn(v);
      } else {
        float* c = static_cast<float*>(Cv) + m * N + nn;
        *c = out_mode == 2 ? *c + v : v;
      }
    }
  }
}

cudaError_t launch_gemm_simt(const void* A, const void* B, int64_t M, int N, int K, int epi,
                             int out_mode, void* C, cudaStream_t stream, bool a_mn, bool b_mn) {
  dim3 grid((N + 63) / 64, (unsigned)((M + 63) / 64));
  gemm_simt_kernel<<<grid, 256, 0, stream>>>((const __nv_bfloat16*)A, (const __nv_bfloat16*)B,
                                             M, N, K, epi, out_mode, a_mn, b_mn, C);
  note_launch();
  return cudaGetLastError();
}
cudaError_t launch_gemm_tc(const void* A, const void* B, int64_t M, int N, int K, int epi,
                           int out_mode, void* C, int32_t* status, cudaStream_t stream,
                           int splits, int64_t c_split, bool a_mn, bool b_mn, int pdl_mode = 0);

// Shapes the tensor-core GEMM takes: the TMA rows of every operand are a
// multiple of 16 bytes (K for a K-major operand, M / N for an MN-major one).
static bool tc_ok(int64_t M, int N, int K, bool a_mn, bool b_mn) {
  if (M < 1 || N < 16 || K < 64 || N % 8) return false;
  if ((!a_mn || !b_mn) && K % 8) return false;
  return !a_mn || M % 8 == 0;
}

// Few rows (decode batches): C[M,N] = epi(A[M,K] W) with W [K][N] held
// N-contiguous, on the SIMT cores.  A 128-row tensor-core tile would be
// mostly padding, and the work is reading W once, so W is spread over many
// CTAs: each reads an 8-column strip (one 16-byte vector per k) for up to 8
// rows of A.  Its 8 warps split K; lane l takes every 32nd k of its warp's
// range with all of its weight loads in flight at once, and FMAs each vector
// into 8 rows x 8 columns of fp32 partials.  The 32 lanes' partials are
// summed by a butterfly that halves the values a lane holds at each of its
// five exchange steps (lane l ends with outputs 2l and 2l+1), the 8 warps'
// sums in warp order through shared memory: a fixed order, so the result is
// reproducible.  A^T [K][8] is staged in shared memory (one 16-byte load
// gives A[0..7][k]), every 8 k-lines padded by 16 bytes so that the
// staging threads' stores spread over the banks.
constexpr int kSmallM = 8;
constexpr int kSmallCols = 8;
constexpr int kSmallMaxK = 1024;            // A^T fits 18 KiB of static shared memory
constexpr int kSmallWarps = 8;
constexpr int kSmallRowsPerLane = kSmallMaxK / kSmallWarps / 32;  // weight loads in flight

__device__ __forceinline__ int at_index(int k) { return k * kSmallM + (k >> 3) * kSmallM; }

// pdl_mode (programmatic dependent launch): 1 -- A is the previous kernel's
// output, wait for it first; 2 -- the inputs do not depend on the previous
// kernel, wait for it only before finishing (so that this kernel's completion
// still implies that one's); 0 -- ordinary launch.
__global__ void __launch_bounds__(kSmallWarps * 32) gemm_small_m_kernel(
    const __nv_bfloat16* __restrict__ A, const __nv_bfloat16* __restrict__ W, int M, int N, int K,
    int epi, __nv_bfloat16* __restrict__ C, int pdl_mode) {
  __shared__ __align__(16) uint16_t at[kSmallMaxK * kSmallM + kSmallMaxK];  // A^T, padded
  __shared__ float part[kSmallWarps][kSmallM * kSmallCols];
  const int n0 = blockIdx.x * kSmallCols;
  const int m0 = blockIdx.y * kSmallM;
  const int mc = min(kSmallM, M - m0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_launch_dependents();
  // this lane's weight vectors, loaded before anything waits
  const int kw = (K + kSmallWarps - 1) / kSmallWarps;
  const int kb = warp * kw, ke = min(K, kb + kw);
  uint4 wv[kSmallRowsPerLane];
#pragma unroll
  for (int r = 0; r < kSmallRowsPerLane; ++r) {
    const int kk = kb + lane + 32 * r;
    wv[r] = kk < ke ? ldg_nc_16(W + (int64_t)kk * N + n0) : make_uint4(0u, 0u, 0u, 0u);
  }
  if (pdl_mode == 1) pdl_wait();
  // stage A^T: thread kc transposes the 8 x 8 block A[0..7][8 kc .. 8 kc + 7]
  for (int kc = threadIdx.x; kc < K / 8; kc += blockDim.x) {
    uint32_t u[kSmallM][4];
#pragma unroll
    for (int m = 0; m < kSmallM; ++m) {
      const uint4 v = m < mc ? *reinterpret_cast<const uint4*>(A + (int64_t)(m0 + m) * K + kc * 8)
                             : make_uint4(0u, 0u, 0u, 0u);
      u[m][0] = v.x;
      u[m][1] = v.y;
      u[m][2] = v.z;
      u[m][3] = v.w;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        o[q] = __byte_perm(u[2 * q][j >> 1], u[2 * q + 1][j >> 1], (j & 1) ? 0x7632 : 0x5410);
      *reinterpret_cast<uint4*>(at + at_index(kc * 8 + j)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  __syncthreads();
  float acc[kSmallM * kSmallCols];  // [m][c]
#pragma unroll
  for (int i = 0; i < kSmallM * kSmallCols; ++i) acc[i] = 0.f;
#pragma unroll
  for (int r = 0; r < kSmallRowsPerLane; ++r) {
    const int kk = kb + lane + 32 * r;
    if (kk < ke) {
      float wf[8], af[8];
      unpack16<PKM_BF16>(wv[r], wf);
      unpack16<PKM_BF16>(*reinterpret_cast<const uint4*>(at + at_index(kk)), af);
#pragma unroll
      for (int m = 0; m < kSmallM; ++m)
#pragma unroll
        for (int c = 0; c < kSmallCols; ++c) acc[m * kSmallCols + c] = fmaf(af[m], wf[c], acc[m * kSmallCols + c]);
    }
  }
  // butterfly over the lanes: at the step with mask h the lanes with bit h
  // keep the upper half of their values and add their partner's copy of it
#pragma unroll
  for (int h = 16, cnt = kSmallM * kSmallCols; h > 0; h >>= 1, cnt >>= 1) {
    const bool upper = (lane & h) != 0;
#pragma unroll
    for (int i = 0; i < cnt / 2; ++i) {
      const float send = upper ? acc[i] : acc[i + cnt / 2];
      const float keep = upper ? acc[i + cnt / 2] : acc[i];
      acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, h);
    }
  }
  part[warp][2 * lane] = acc[0];
  part[warp][2 * lane + 1] = acc[1];
  __syncthreads();
  if (threadIdx.x < kSmallM * kSmallCols) {
    const int m = threadIdx.x / kSmallCols, c = threadIdx.x % kSmallCols;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kSmallWarps; ++w) v += part[w][threadIdx.x];
    if (epi == 1) v = silu_f(v);
    if (m < mc && n0 + c < N) C[(int64_t)(m0 + m) * N + n0 + c] = __float2bfloat16_rn(v);
  }
  if (pdl_mode == 2) pdl_wait();
}

cudaError_t launch_gemm_bf16(const void* A, const void* B, int64_t M, int N, int K, int epi,
                             void* C, int32_t* status, cudaStream_t stream, bool b_mn,
                             int pdl_mode) {
  if (M <= 0) return cudaSuccess;
  if (b_mn && M <= 64 && K <= kSmallMaxK && K % 8 == 0 && N % 8 == 0) {
    dim3 grid((unsigned)((N + kSmallCols - 1) / kSmallCols), (unsigned)((M + kSmallM - 1) / kSmallM));
    const cudaError_t e = launch_maybe_pdl(
        pdl_mode != 0, gemm_small_m_kernel, grid, dim3(kSmallWarps * 32), 0, stream,
        static_cast<const __nv_bfloat16*>(A), static_cast<const __nv_bfloat16*>(B), (int)M, N, K,
        epi, static_cast<__nv_bfloat16*>(C), pdl_mode);
    note_launch();
    return e != cudaSuccess ? e : cudaGetLastError();
  }
  if (tc_ok(M, N, K, false, b_mn))
    return launch_gemm_tc(A, B, M, N, K, epi, 0, C, status, stream, 1, 0, false, b_mn, pdl_mode);
  return launch_gemm_simt(A, B, M, N, K, epi, 0, C, stream, false, b_mn);
}

cudaError_t launch_gemm_f32(const void* A, const void* B, int64_t M, int N, int K,
                            bool accumulate, float* C, int32_t* status, cudaStream_t stream,
                            bool a_mn, bool b_mn) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  const int mode = accumulate ? 2 : 1;
  if (tc_ok(M, N, K, a_mn, b_mn))
    return launch_gemm_tc(A, B, M, N, K, 0, mode, C, status, stream, 1, 0, a_mn, b_mn);
  return launch_gemm_simt(A, B, M, N, K, 0, mode, C, stream, a_mn, b_mn);
}

// C = sum over s of part[s] (fixed order)
__global__ void sum_slices_kernel(const float* __restrict__ part, int S, int64_t n,
                                  float* __restrict__ C) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < S; ++s) acc += part[(int64_t)s * n + i];
    C[i] = acc;
  }
}

int gemm_splitk_slices(int64_t M, int N, int K) {
  if (M < 1 || N < 16 || K < 64 || N % 8) return 1;
  const int64_t tiles = ((M + 127) / 128) * ((N + 255) / 256);
  const int KB = (K + 63) / 64;
  int s = 1;
  while (s < 8 && tiles * s * 2 <= 148 && KB >= 4 * s * 2) s *= 2;
  return s;
}

size_t gemm_splitk_workspace(int64_t M, int N, int K) {
  const int s = gemm_splitk_slices(M, N, K);
  return s > 1 ? (size_t)s * M * N * sizeof(float) : 0;
}

cudaError_t launch_gemm_f32_splitk(const void* A, const void* B, int64_t M, int N, int K,
                                   float* C, float* part, int32_t* status, cudaStream_t stream,
                                   bool a_mn, bool b_mn) {
  const int S = gemm_splitk_slices(M, N, K);
  if (S <= 1 || !part || !tc_ok(M, N, K, a_mn, b_mn))
    return launch_gemm_f32(A, B, M, N, K, false, C, status, stream, a_mn, b_mn);
  cudaError_t e = launch_gemm_tc(A, B, M, N, K, 0, 1, part, status, stream, S, M * N, a_mn, b_mn);
  if (e != cudaSuccess) return e;
  // the GEMM launcher makes ceil(KB / ceil(KB / S)) slices; with KB >= 8 S this is S
  const int KB = (K + 63) / 64, kbps = (KB + S - 1) / S, nz = (KB + kbps - 1) / kbps;
  const int64_t n = M * N;
  const int64_t blocks = (n + 255) / 256;
  sum_slices_kernel<<<(unsigned)(blocks < 148 * 8 ? blocks : 148 * 8), 256, 0, stream>>>(
      part, nz, n, C);
  note_launch();
  return cudaGetLastError();
}

}  // namespace pkm
