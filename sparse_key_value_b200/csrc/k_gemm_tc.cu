// k_gemm_tc.cu -- the dense GEMMs of the Memory+ block on the tensor cores
// ("Memory Layers at Scale" digest, "Memory+ 블록": out = (y ⊙ silu(x W1)) W2).
//
//   C[M, N] = epi(A[M, K] * B[N, K]^T),  A, B bf16 K-major, C row-major,
//   epi = silu (gate) or identity, fp32 accumulation; C is bf16 (rounded to
//   nearest even), fp32, or fp32 accumulated into (C += A B^T).
//
// One CTA per 128 x 256 output tile:
//   warp 0     TMA producer: 64-wide k-blocks of A [128 x 64] and B [256 x 64]
//              (128-byte swizzle) into a 4-stage ring.
//   warp 1     TMEM owner and MMA issuer: tcgen05.mma kind::f16, M=128, N=256.
//   warps 2-5  epilogue: one thread per output row reads 32 accumulator
//              columns at a time (tcgen05.ld), applies the epilogue, rounds to
//              bf16 (nearest even) and stores 64 contiguous bytes.
// Spin-waits are bounded; on a timeout the CTA records PKM_ERR_TIMEOUT,
// drains what it issued, frees its TMEM and exits.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tmap.h"

namespace pkm {

namespace gm {
constexpr int kM = 128, kN = 256, kKB = 64, kStages = 4;
constexpr int kABytes = kM * kKB * 2, kBBytes = kN * kKB * 2;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 192;
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + 256;
}  // namespace gm

struct GemmCtl {
  uint64_t full[gm::kStages];
  uint64_t empty[gm::kStages];
  uint64_t accf;
  uint64_t drain;
  uint32_t tmem;
  volatile int abort;
};

__device__ __forceinline__ bool gemm_wait(uint64_t* bar, uint32_t parity, GemmCtl* ctl,
                                          int32_t* status) {
  return mbar_wait_or_abort(bar, parity, &ctl->abort, status);
}

// OUT: 0 bf16 store, 1 fp32 store, 2 fp32 accumulate (C += result)
template <int EPI, int OUT>
__global__ void __launch_bounds__(gm::kThreads, 1) gemm_tc_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int64_t M,
    int N, int K, void* __restrict__ Cv, int kb_per_split, int64_t c_split,
    int32_t* status) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* stages = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  GemmCtl* ctl = reinterpret_cast<GemmCtl*>(stages + gm::kStages * gm::kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m0 = (int64_t)blockIdx.x * gm::kM;
  const int n0 = blockIdx.y * gm::kN;
  // split-K (grid.z): this CTA adds k-blocks [kb0, kb0 + KB) into the
  // output slice blockIdx.z (c_split elements apart)
  const int KB_all = (K + gm::kKB - 1) / gm::kKB;
  const int kb0 = kb_per_split > 0 ? (int)blockIdx.z * kb_per_split : 0;
  const int KB = kb_per_split > 0 ? min(kb_per_split, KB_all - kb0) : KB_all;
  Cv = static_cast<char*>(Cv) + (int64_t)blockIdx.z * c_split * (OUT != 0 ? 4 : 2);

  if (threadIdx.x == 0) {
    for (int s = 0; s < gm::kStages; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    mbar_init(&ctl->accf, 1);
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem, gm::kN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t issued_mask = 0, issued_par = 0;
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        const int stage = kb % gm::kStages;
        const uint32_t phase = (uint32_t)(kb / gm::kStages) & 1;
        if (!gemm_wait(&ctl->empty[stage], phase ^ 1, ctl, status)) { ok = false; break; }
        unsigned char* sa = stages + stage * gm::kStageBytes;
        mbar_arrive_expect_tx(&ctl->full[stage], gm::kStageBytes);
        tma_load_2d(sa, &tmA, &ctl->full[stage], (kb0 + kb) * gm::kKB, (int32_t)m0);
        tma_load_2d(sa + gm::kABytes, &tmB, &ctl->full[stage], (kb0 + kb) * gm::kKB, n0);
        issued_mask |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
      }
      if (!ok) {
        for (int s = 0; s < gm::kStages; ++s)
          if (issued_mask & (1u << s))
            for (unsigned long long i = 0; i < kSpinLimit; ++i)
              if (mbar_try_wait(&ctl->full[s], (issued_par >> s) & 1)) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(gm::kM, gm::kN);
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        const int stage = kb % gm::kStages;
        const uint32_t phase = (uint32_t)(kb / gm::kStages) & 1;
        if (!gemm_wait(&ctl->full[stage], phase, ctl, status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = smem_u32(stages + stage * gm::kStageBytes);
        const uint32_t sb = sa + gm::kABytes;
#pragma unroll
        for (int kk = 0; kk < gm::kKB / 16; ++kk)
          tc_mma_f16(tmem, smem_desc_k128(sa + kk * 32), smem_desc_k128(sb + kk * 32), idesc,
                     (kb | kk) != 0);
        tc_commit(&ctl->empty[stage]);
      }
      if (ok) tc_commit(&ctl->accf);
      tc_commit(&ctl->drain);
      for (unsigned long long i = 0; i < kSpinLimit; ++i)
        if (mbar_try_wait(&ctl->drain, 0)) break;
    }
  } else {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int64_t m = m0 + row;
    const bool got = gemm_wait(&ctl->accf, 0, ctl, status);
    if (__all_sync(0xffffffffu, got)) {
      tc_fence_after();
      for (int g = 0; g < gm::kN / 32; ++g) {
        const int col0 = n0 + g * 32;
        if (col0 >= N) break;
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) + g * 32, r);
        tmem_ld_wait();
        if (m < M && OUT != 0) {
          float* dst = static_cast<float*>(Cv) + m * N + col0;
          const int nq = col0 + 32 <= N ? 8 : (N - col0) / 4;  // N % 8 == 0
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (j < nq) {
              float4 v = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                     __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
              if (OUT == 2) {
                const float4 o = reinterpret_cast<const float4*>(dst)[j];
                v.x += o.x;
                v.y += o.y;
                v.z += o.z;
                v.w += o.w;
              }
              reinterpret_cast<float4*>(dst)[j] = v;
            }
          }
        } else if (m < M) {
          uint32_t packed[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            float a = __uint_as_float(r[2 * j]), b = __uint_as_float(r[2 * j + 1]);
            if (EPI == 1) {
              // silu with the fast exponential and division intrinsics (a few
              // ulp in fp32, far below the bf16 rounding that follows; -a
              // large: __expf -> inf, a / inf -> -0)
              a = __fdividef(a, 1.0f + __expf(-a));
              b = __fdividef(b, 1.0f + __expf(-b));
            }
            packed[j] = pack_bf16x2(a, b);
          }
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(Cv) + m * N + col0;
          if (col0 + 32 <= N) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              reinterpret_cast<uint4*>(dst)[j] =
                  make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
          } else {
            for (int j = 0; j < 16 && col0 + 2 * j < N; ++j)
              reinterpret_cast<uint32_t*>(dst)[j] = packed[j];  // N % 8 == 0
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, gm::kN);
  }
}

bool gemm_tc_supported(int64_t M, int N, int K) {
  return M >= 1 && N >= 16 && K >= gm::kKB && N % 8 == 0 && K % 8 == 0;
}

// out_mode: 0 bf16 (epi applied), 1 fp32, 2 fp32 accumulate; epi only with bf16 output.
// splits > 1: split-K into `splits` slices of C, c_split elements apart.
cudaError_t launch_gemm_tc(const void* A, const void* B, int64_t M, int N, int K, int epi,
                           int out_mode, void* C, int32_t* status, cudaStream_t stream,
                           int splits, int64_t c_split) {
  if (M <= 0) return cudaSuccess;
  CUtensorMap tmA, tmB;
  {
    const uint64_t dims[2] = {(uint64_t)K, (uint64_t)M};
    const uint64_t strides[1] = {(uint64_t)K * 2};
    const uint32_t box[2] = {(uint32_t)gm::kKB, (uint32_t)gm::kM};
    if (!make_tmap_bf16(&tmA, A, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {(uint64_t)K, (uint64_t)N};
    const uint64_t strides[1] = {(uint64_t)K * 2};
    const uint32_t box[2] = {(uint32_t)gm::kKB, (uint32_t)gm::kN};
    if (!make_tmap_bf16(&tmB, B, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  const int KB = (K + gm::kKB - 1) / gm::kKB;
  int kbps = 0, nz = 1;
  if (splits > 1) {  // every slice gets at least one k-block
    kbps = (KB + splits - 1) / splits;
    nz = (KB + kbps - 1) / kbps;
  }
  dim3 grid((unsigned)((M + gm::kM - 1) / gm::kM), (unsigned)((N + gm::kN - 1) / gm::kN),
            (unsigned)nz);
  cudaError_t e;
#define PKM_GEMM_TC(E_, O_)                                                                  \
  e = cudaFuncSetAttribute(gemm_tc_kernel<E_, O_>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                           (int)gm::kSmemBytes);                                             \
  if (e != cudaSuccess) return e;                                                            \
  gemm_tc_kernel<E_, O_><<<grid, gm::kThreads, gm::kSmemBytes, stream>>>(tmA, tmB, M, N, K, C, \
                                                                        kbps, c_split, status)
  if (out_mode == 1) {
    PKM_GEMM_TC(0, 1);
  } else if (out_mode == 2) {
    PKM_GEMM_TC(0, 2);
  } else if (epi == 1) {
    PKM_GEMM_TC(1, 0);
  } else {
    PKM_GEMM_TC(0, 0);
  }
#undef PKM_GEMM_TC
  note_launch();
  return cudaGetLastError();
}

}  // namespace pkm
