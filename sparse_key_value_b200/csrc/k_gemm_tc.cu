// k_gemm_tc.cu -- the dense GEMMs of the Memory+ block on the tensor cores
// ("Memory Layers at Scale" digest, "Memory+ 블록": out = (y ⊙ silu(x W1)) W2).
//
//   C[M, N] = epi(A[M, K] * B[N, K]^T), bf16 operands, fp32 accumulation;
//   epi = silu (gate) or identity; C is bf16 (rounded to nearest even), fp32,
//   or fp32 accumulated into (C += A B^T).
// Each operand is read in the layout the caller holds it, so no operand is
// transposed in memory:
//   K-major   A as [M][K] (or B as [N][K]), K contiguous;
//   MN-major  A as [K][M] (or B as [K][N]), M (N) contiguous -- a weight
//             W [d_in, d_out] used as x W, or the tokens' rows used as the
//             contraction of a weight gradient (x^T dy).
// The TMA loads 64-wide k-blocks with the 128-byte swizzle: a K-major tile is
// [rows][64 k] (one 128-byte line per row), an MN-major tile is a stack of
// [64 k][64 rows] boxes (one line per k); the MMA's shared-memory descriptor
// and the instruction descriptor's transpose bit say which.
//
// Persistent: one CTA per SM loops over the output tiles (128 x 256, N
// fastest so neighbouring tiles share their A rows, then split-K slices).
//   warp 0     TMA producer: a 4-stage ring of (A, B) k-blocks, continuing
//              across tiles.
//   warp 1     TMEM owner and MMA issuer: tcgen05.mma kind::f16, M=128,
//              N=256, into one of two 256-column accumulators (TMEM 512).
//   warps 2-5  epilogue: one thread per output row; while it reads and stores
//              one accumulator the MMAs of the next tile fill the other.
// Spin-waits are bounded; on a timeout the CTA records PKM_ERR_TIMEOUT,
// drains what it issued, frees its TMEM and exits.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tmap.h"

namespace pkm {

namespace gm {
constexpr int kM = 128, kN = 256, kKB = 64, kStages = 4, kAcc = 2;
constexpr int kABytes = kM * kKB * 2, kBBytes = kN * kKB * 2;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 192;
constexpr int kBox = 64;  // rows of an MN-major box (128 bytes of bf16)
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + 256;
}  // namespace gm

struct GemmCtl {
  uint64_t full[gm::kStages];
  uint64_t empty[gm::kStages];
  uint64_t accf[gm::kAcc];
  uint64_t acce[gm::kAcc];
  uint64_t drain;
  uint32_t tmem;
  volatile int abort;
};

__device__ __forceinline__ bool gemm_wait(uint64_t* bar, uint32_t parity, GemmCtl* ctl,
                                          int32_t* status) {
  return mbar_wait_or_abort(bar, parity, &ctl->abort, status);
}

// Shared-memory descriptor of an MN-major operand tile with the 128-byte
// swizzle: atoms of 8 k-lines x 64 elements (1024 B); consecutive atoms along
// K are 1024 B apart (stride byte offset), consecutive 64-element groups
// along M/N are one box (8 KiB) apart (leading byte offset).
__device__ __forceinline__ uint64_t smem_desc_mn128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((gm::kBox * 128) >> 4) << 16;  // leading byte offset: next box
  d |= (uint64_t)(1024 >> 4) << 32;              // stride byte offset: next 8 k-lines
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

struct TileCoord {
  int64_t m0;
  int n0, z;
};

__device__ __forceinline__ TileCoord tile_of(int t, int tiles_m, int tiles_n) {
  const int nt = t % tiles_n;
  const int r = t / tiles_n;
  return TileCoord{(int64_t)(r % tiles_m) * gm::kM, nt * gm::kN, r / tiles_m};
}

// OUT: 0 bf16 store, 1 fp32 store, 2 fp32 accumulate (C += result).
// AMN / BMN: the operand is MN-major.
template <int EPI, int OUT, bool AMN, bool BMN>
__global__ void __launch_bounds__(gm::kThreads, 1) gemm_tc_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int64_t M,
    int N, int K, void* __restrict__ Cv, int kb_per_split, int nz, int64_t c_split,
    int32_t* status, int pdl_mode) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* stages = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  GemmCtl* ctl = reinterpret_cast<GemmCtl*>(stages + gm::kStages * gm::kStageBytes);
  // programmatic dependent launch: 1 -- an operand is the previous kernel's
  // output, wait for it first; 2 -- none is, wait only before finishing
  pdl_launch_dependents();
  if (pdl_mode == 1) pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = (int)((M + gm::kM - 1) / gm::kM);
  const int tiles_n = (N + gm::kN - 1) / gm::kN;
  const int n_tiles = tiles_m * tiles_n * nz;
  // split-K: slice z adds k-blocks [z * kb_per_split, ...) into the output
  // slice z (c_split elements apart)
  const int KB_all = (K + gm::kKB - 1) / gm::kKB;
  auto kb_range = [&](int z, int& kb0, int& nkb) {
    kb0 = kb_per_split > 0 ? z * kb_per_split : 0;
    nkb = kb_per_split > 0 ? min(kb_per_split, KB_all - kb0) : KB_all;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < gm::kStages; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int b = 0; b < gm::kAcc; ++b) {
      mbar_init(&ctl->accf[b], 1);
      mbar_init(&ctl->acce[b], 4);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem, gm::kAcc * gm::kN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t issued_mask = 0, issued_par = 0;
      bool ok = true;
      int f = 0;  // stage fills so far
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const TileCoord tc = tile_of(t, tiles_m, tiles_n);
        int kb0, nkb;
        kb_range(tc.z, kb0, nkb);
        for (int kb = 0; kb < nkb; ++kb, ++f) {
          const int stage = f % gm::kStages;
          const uint32_t phase = (uint32_t)(f / gm::kStages) & 1;
          if (!gemm_wait(&ctl->empty[stage], phase ^ 1, ctl, status)) { ok = false; break; }
          unsigned char* sa = stages + stage * gm::kStageBytes;
          unsigned char* sb = sa + gm::kABytes;
          const int kc = (kb0 + kb) * gm::kKB;
          mbar_arrive_expect_tx(&ctl->full[stage], gm::kStageBytes);
          if (AMN) {
#pragma unroll
            for (int j = 0; j < gm::kM / gm::kBox; ++j)
              tma_load_2d(sa + j * gm::kBox * 128, &tmA, &ctl->full[stage],
                          (int32_t)tc.m0 + j * gm::kBox, kc);
          } else {
            tma_load_2d(sa, &tmA, &ctl->full[stage], kc, (int32_t)tc.m0);
          }
          if (BMN) {
#pragma unroll
            for (int j = 0; j < gm::kN / gm::kBox; ++j)
              tma_load_2d(sb + j * gm::kBox * 128, &tmB, &ctl->full[stage],
                          tc.n0 + j * gm::kBox, kc);
          } else {
            tma_load_2d(sb, &tmB, &ctl->full[stage], kc, tc.n0);
          }
          issued_mask |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        }
      }
      if (!ok) {
        for (int s = 0; s < gm::kStages; ++s)
          if (issued_mask & (1u << s))
            for (unsigned long long i = 0; i < kSpinLimit; ++i)
              if (mbar_try_wait(&ctl->full[s], (issued_par >> s) & 1)) break;
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(gm::kM, gm::kN) | (AMN ? (1u << 15) : 0u) |
                             (BMN ? (1u << 16) : 0u);
      bool ok = true;
      int f = 0, li = 0;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++li) {
        const TileCoord tc = tile_of(t, tiles_m, tiles_n);
        int kb0, nkb;
        kb_range(tc.z, kb0, nkb);
        const int buf = li & 1;
        // this accumulator is free once the epilogue has read its last tile
        if (!gemm_wait(&ctl->acce[buf], ((li >> 1) & 1) ^ 1, ctl, status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dt = tmem + (uint32_t)(buf * gm::kN);
        for (int kb = 0; kb < nkb; ++kb, ++f) {
          const int stage = f % gm::kStages;
          const uint32_t phase = (uint32_t)(f / gm::kStages) & 1;
          if (!gemm_wait(&ctl->full[stage], phase, ctl, status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(stages + stage * gm::kStageBytes);
          const uint32_t sb = sa + gm::kABytes;
#pragma unroll
          for (int kk = 0; kk < gm::kKB / 16; ++kk) {
            // K = 16 per MMA: 32 bytes along a K-major line, 16 lines of an MN-major box
            const uint64_t ad = AMN ? smem_desc_mn128(sa + kk * 2048) : smem_desc_k128(sa + kk * 32);
            const uint64_t bd = BMN ? smem_desc_mn128(sb + kk * 2048) : smem_desc_k128(sb + kk * 32);
            tc_mma_f16(dt, ad, bd, idesc, (kb | kk) != 0);
          }
          tc_commit(&ctl->empty[stage]);
        }
        if (ok) tc_commit(&ctl->accf[buf]);
      }
      tc_commit(&ctl->drain);
      for (unsigned long long i = 0; i < kSpinLimit; ++i)
        if (mbar_try_wait(&ctl->drain, 0)) break;
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    int li = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++li) {
      const TileCoord tc = tile_of(t, tiles_m, tiles_n);
      const int buf = li & 1;
      const bool got = gemm_wait(&ctl->accf[buf], (li >> 1) & 1, ctl, status);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int64_t m = tc.m0 + row;
      void* Cz = static_cast<char*>(Cv) + (int64_t)tc.z * c_split * (OUT != 0 ? 4 : 2);
      for (int g = 0; g < gm::kN / 32; ++g) {
        const int col0 = tc.n0 + g * 32;
        if (col0 >= N) break;
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) + buf * gm::kN + g * 32, r);
        tmem_ld_wait();
        if (m < M && OUT != 0) {
          float* dst = static_cast<float*>(Cz) + m * N + col0;
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
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(Cz) + m * N + col0;
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
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->acce[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, gm::kAcc * gm::kN);
  }
  if (pdl_mode == 2) pdl_wait();
}

bool gemm_tc_supported(int64_t M, int N, int K) {
  return M >= 1 && N >= 16 && K >= gm::kKB && N % 8 == 0 && K % 8 == 0;
}

static int num_sms() {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
      sms = v;
    else
      return 148;
  }
  return sms;
}

// out_mode: 0 bf16 (epi applied), 1 fp32, 2 fp32 accumulate; epi only with bf16 output.
// splits > 1: split-K into `splits` slices of C, c_split elements apart.
// a_mn / b_mn: A is [K][M] / B is [K][N] (M / N contiguous) instead of [M][K] / [N][K].
cudaError_t launch_gemm_tc(const void* A, const void* B, int64_t M, int N, int K, int epi,
                           int out_mode, void* C, int32_t* status, cudaStream_t stream,
                           int splits, int64_t c_split, bool a_mn, bool b_mn, int pdl_mode) {
  if (M <= 0) return cudaSuccess;
  // more than one 128-row tile: pairs of SMs share 256 x 256 tiles (k_gemm_tc2.cu)
  if (gemm_tc2_useful(M)) {
    const cudaError_t e2 = launch_gemm_tc2(A, B, M, N, K, epi, out_mode, C, status, stream,
                                           splits, c_split, a_mn, b_mn, pdl_mode);
    if (e2 != cudaErrorNotSupported) return e2;
  }
  CUtensorMap tmA, tmB;
  if (a_mn) {
    if (M % 8) return cudaErrorInvalidValue;  // the row stride of [K][M] is 16-byte aligned
    const uint64_t dims[2] = {(uint64_t)M, (uint64_t)K};
    const uint64_t strides[1] = {(uint64_t)M * 2};
    const uint32_t box[2] = {(uint32_t)gm::kBox, (uint32_t)gm::kKB};
    if (!make_tmap_bf16(&tmA, A, 2, dims, strides, box)) return cudaErrorInvalidValue;
  } else {
    const uint64_t dims[2] = {(uint64_t)K, (uint64_t)M};
    const uint64_t strides[1] = {(uint64_t)K * 2};
    const uint32_t box[2] = {(uint32_t)gm::kKB, (uint32_t)gm::kM};
    if (!make_tmap_bf16(&tmA, A, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  if (b_mn) {
    const uint64_t dims[2] = {(uint64_t)N, (uint64_t)K};
    const uint64_t strides[1] = {(uint64_t)N * 2};
    const uint32_t box[2] = {(uint32_t)gm::kBox, (uint32_t)gm::kKB};
    if (!make_tmap_bf16(&tmB, B, 2, dims, strides, box)) return cudaErrorInvalidValue;
  } else {
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
  const int64_t tiles = (M + gm::kM - 1) / gm::kM * ((N + gm::kN - 1) / gm::kN) * nz;
  const unsigned grid = (unsigned)(tiles < num_sms() ? tiles : num_sms());
  cudaError_t e = cudaSuccess;
  auto go = [&](auto kern) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)gm::kSmemBytes);
    if (e != cudaSuccess) return;
    e = launch_maybe_pdl(pdl_mode != 0, kern, dim3(grid), dim3(gm::kThreads), gm::kSmemBytes,
                         stream, tmA, tmB, M, N, K, C, kbps, nz, c_split, status, pdl_mode);
  };
#define PKM_GEMM_LAYOUTS(E_, O_)                                   \
  if (a_mn && b_mn) go(gemm_tc_kernel<E_, O_, true, true>);        \
  else if (a_mn) go(gemm_tc_kernel<E_, O_, true, false>);          \
  else if (b_mn) go(gemm_tc_kernel<E_, O_, false, true>);          \
  else go(gemm_tc_kernel<E_, O_, false, false>)
  if (out_mode == 1) {
    PKM_GEMM_LAYOUTS(0, 1);
  } else if (out_mode == 2) {
    PKM_GEMM_LAYOUTS(0, 2);
  } else if (epi == 1) {
    PKM_GEMM_LAYOUTS(1, 0);
  } else {
    PKM_GEMM_LAYOUTS(0, 0);
  }
#undef PKM_GEMM_LAYOUTS
  if (e != cudaSuccess) return e;
  note_launch();
  return cudaGetLastError();
}

}  // namespace pkm
