// k_score_small.cu -- sub-key scoring and per-half top-k for batches of at
// most 32 tokens (decode steps), on the tensor cores.
//
// "모델 안의 메모리", "작동 방식": each half of the query is compared with all
// of its ~sqrt(N) half-keys and the best are kept.  With a handful of tokens
// the work is the sub-key tables themselves (every row is read once), so the
// grid is (1, 2H, chunks): one CTA per (head, half, 256-column chunk), whose
// k best per token go to the split lists hv/hi [chunk][T, H, 2, k] that the
// combine kernel merges (k_combine.cu).
//   warp 0     TMA producer: the 64-wide k-blocks of the token tile (rows
//              past T read as zero) and of the chunk's sub-keys, 4 stages.
//   warp 1     TMEM owner and MMA issuer: tcgen05.mma kind::f16, M=128,
//              N=256, fp32 accumulator in 256 TMEM columns.
//   warp 4     reads the accumulator rows of the live tokens (TMEM lanes
//              0..31 belong to it), scales them to scores
//                s = sqrt(d_half) * rq[t] * rk[a] * acc
//              and stores them to shared memory (the stage ring, free once
//              the MMAs are done).
//   all warps  one token at a time per warp: the chunk's 256 scores, 8 per
//              lane, are sorted by a bitonic network across the warp (keys:
//              order-preserving score bits above the complemented position,
//              so equal scores order the smaller position first) and the
//              first k are the token's list.
// With 32 or fewer tokens only one warp could read the accumulator, and a
// per-thread running top-k would leave the other five idle; the shared
// staging spreads the selection over the CTA.
//
// Every spin-wait is bounded: on a timeout the CTA records PKM_ERR_TIMEOUT,
// stops issuing work, waits (bounded) for its copies and MMAs in flight,
// frees its TMEM and exits without writing lists.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tmap.h"

namespace pkm {

namespace ss {
constexpr int kM = 128;          // TMEM lanes (token tile, mostly padding)
constexpr int kN = 256;          // sub-key columns per CTA
constexpr int kKB = 64;
constexpr int kStages = 4;
constexpr int kABytes = kM * kKB * 2;
constexpr int kBBytes = kN * kKB * 2;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 192;
constexpr int kMaxRows = 32;
constexpr size_t kSmemBytes = (size_t)kStages * kStageBytes + 256;
static_assert(kMaxRows * kN * 4 <= kStages * kStageBytes, "scores fit in the stage ring");
}  // namespace ss

namespace {

struct SmallCtl {
  uint64_t full[ss::kStages];
  uint64_t empty[ss::kStages];
  uint64_t accf;
  uint64_t drain;
  uint32_t tmem;
  volatile int abort;
};

__device__ __forceinline__ bool wait_small(uint64_t* bar, uint32_t parity, SmallCtl* ctl,
                                           int32_t* status) {
  return mbar_wait_or_abort(bar, parity, &ctl->abort, status);
}

__device__ __forceinline__ uint32_t ord_bits(float s) {
  const uint32_t u = __float_as_uint(s + 0.0f);  // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float unord_bits(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
  return ((uint64_t)hi << 32) | lo;
}

// Bitonic sort, descending, of the 256 keys held as v[s] on lane l at
// position p = 32 s + l.
__device__ __forceinline__ void warp_sort256_desc(uint64_t (&v)[8]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 256; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride >= 32) {  // partner in another slot of the same lane
        const int ds = stride >> 5;
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          if ((s & ds) == 0) {
            const bool desc = ((s * 32 + lane) & size) == 0;
            const uint64_t a = v[s], b = v[s + ds];
            const bool sw = desc ? (a < b) : (a > b);
            v[s] = sw ? b : a;
            v[s + ds] = sw ? a : b;
          }
        }
      } else {  // partner on lane ^ stride
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const bool desc = ((s * 32 + lane) & size) == 0;
          const bool lower = (lane & stride) == 0;
          const uint64_t o = shfl_xor_u64(v[s], stride);
          const uint64_t mx = v[s] > o ? v[s] : o, mn = v[s] > o ? o : v[s];
          v[s] = (lower == desc) ? mx : mn;
        }
      }
    }
  }
}

__global__ void __launch_bounds__(ss::kThreads, 1) score_topk_small_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int T,
    int H, int dh, int n, int k, const float* __restrict__ rq, const float* __restrict__ rk,
    float* __restrict__ hv, int32_t* __restrict__ hi, int32_t* status) {
  using namespace ss;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* stages = smem_raw;
  SmallCtl* ctl = reinterpret_cast<SmallCtl*>(smem_raw + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hc = blockIdx.y;
  const int chunk = blockIdx.z;
  const int c0 = chunk * kN;
  const int ncols = min(kN, n - c0);
  const int KB = dh / kKB;
  const bool misaligned = (smem_u32(smem_raw) & 1023u) != 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    mbar_init(&ctl->accf, 1);
    mbar_init(&ctl->drain, 1);
    ctl->abort = misaligned ? 1 : 0;
    if (misaligned) set_status(status, PKM_ERR_DEVICE);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1 && !misaligned) {
    tmem_alloc(&ctl->tmem, kN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem;
  const bool run = !misaligned;

  if (warp == 0) {
    if (lane == 0 && run) {
      uint32_t issued_mask = 0, issued_par = 0;
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        const int stage = kb % kStages;
        const uint32_t phase = (uint32_t)(kb / kStages) & 1;
        if (!wait_small(&ctl->empty[stage], phase ^ 1, ctl, status)) { ok = false; break; }
        unsigned char* sa = stages + stage * kStageBytes;
        mbar_arrive_expect_tx(&ctl->full[stage], kStageBytes);
        tma_load_3d(sa, &tmA, &ctl->full[stage], kb * kKB, hc, 0);
        tma_load_3d(sa + kABytes, &tmB, &ctl->full[stage], kb * kKB, c0, hc);
        issued_mask |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
      }
      if (!ok) {
        for (int s = 0; s < kStages; ++s)
          if (issued_mask & (1u << s))
            for (unsigned long long i = 0; i < kSpinLimit; ++i)
              if (mbar_try_wait(&ctl->full[s], (issued_par >> s) & 1)) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && run) {
      const uint32_t idesc = idesc_bf16_f32(kM, kN);
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        const int stage = kb % kStages;
        const uint32_t phase = (uint32_t)(kb / kStages) & 1;
        if (!wait_small(&ctl->full[stage], phase, ctl, status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = smem_u32(stages + stage * kStageBytes);
        const uint32_t sb = sa + kABytes;
#pragma unroll
        for (int kk = 0; kk < kKB / 16; ++kk)
          tc_mma_f16(tmem, smem_desc_k128(sa + kk * 32), smem_desc_k128(sb + kk * 32), idesc,
                     (kb | kk) != 0);
        tc_commit(&ctl->empty[stage]);
      }
      if (ok) tc_commit(&ctl->accf);
      tc_commit(&ctl->drain);
      for (unsigned long long i = 0; i < kSpinLimit; ++i)
        if (mbar_try_wait(&ctl->drain, 0)) break;
    }
  } else if (warp == 4 && run) {
    // TMEM lanes 0..31: the live tokens' rows; scores into the stage ring
    const bool got = wait_small(&ctl->accf, 0, ctl, status);
    if (__all_sync(0xffffffffu, got)) {
      tc_fence_after();
      float* sc = reinterpret_cast<float*>(stages);  // [32][256]
      const bool live = lane < T;
      const float rowf = live ? sqrtf((float)dh) * rq[((int64_t)lane * H * 2) + hc] : 0.f;
      const float* rkc = rk + (int64_t)hc * n + c0;  // padded by a chunk: in bounds
      for (int g = 0; g < kN / 8; ++g) {
        uint32_t r[8];
        tmem_ld_32x32b_x8(tmem + g * 8, r);
        const float4 ka = __ldg(reinterpret_cast<const float4*>(rkc + g * 8));
        const float4 kb4 = __ldg(reinterpret_cast<const float4*>(rkc + g * 8) + 1);
        tmem_ld_wait();
        const float kr[8] = {ka.x, ka.y, ka.z, ka.w, kb4.x, kb4.y, kb4.z, kb4.w};
        if (live) {
          float4 o0, o1;
          o0.x = __uint_as_float(r[0]) * kr[0] * rowf;
          o0.y = __uint_as_float(r[1]) * kr[1] * rowf;
          o0.z = __uint_as_float(r[2]) * kr[2] * rowf;
          o0.w = __uint_as_float(r[3]) * kr[3] * rowf;
          o1.x = __uint_as_float(r[4]) * kr[4] * rowf;
          o1.y = __uint_as_float(r[5]) * kr[5] * rowf;
          o1.z = __uint_as_float(r[6]) * kr[6] * rowf;
          o1.w = __uint_as_float(r[7]) * kr[7] * rowf;
          float4* d = reinterpret_cast<float4*>(sc + lane * kN + g * 8);
          d[0] = o0;
          d[1] = o1;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1 && run) {
    tc_fence_after();
    tmem_dealloc(tmem, kN);
  }
  if (!run || ctl->abort) return;  // uniform: the whole CTA leaves

  // per-token top-k of the chunk, one token per warp at a time
  const float* sc = reinterpret_cast<const float*>(stages);
  for (int t = warp; t < T; t += kThreads / 32) {
    const float4* src = reinterpret_cast<const float4*>(sc + t * kN + lane * 8);
    const float4 a = src[0], b = src[1];
    const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint64_t v[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      // slot s of lane l holds column 8 l + s of the chunk (any placement is
      // fine for a full sort)
      const int col = lane * 8 + s;
      v[s] = col < ncols ? ((uint64_t)ord_bits(f[s]) << 32) |
                               (uint64_t)(0xffffffffu - (uint32_t)(c0 + col))
                         : 0ull;
    }
    warp_sort256_desc(v);
    if (lane < k) {  // slot 0 holds positions 0..31: the k best
      const int64_t o = (((int64_t)chunk * T + t) * H * 2 + hc) * k + lane;
      const uint64_t key = v[0];
      hv[o] = key ? unord_bits((uint32_t)(key >> 32)) : -INFINITY;
      hi[o] = key ? (int32_t)(0xffffffffu - (uint32_t)key) : 0x7fffffff;
    }
  }
}

}  // namespace

bool score_small_supported(pkm_dtype dt, int64_t T, int dh, int n, int k) {
  const int chunks = (n + ss::kN - 1) / ss::kN;
  return dt == PKM_BF16 && T >= 1 && T <= ss::kMaxRows && dh % ss::kKB == 0 && dh <= 2048 &&
         n >= ss::kN && n % 4 == 0 && k <= 32 && chunks <= 32;
}

int score_small_chunks(int n) { return (n + ss::kN - 1) / ss::kN; }

cudaError_t launch_score_topk_small(const void* q, const void* K, int64_t T, int H, int dh,
                                    int n, int k, const float* rq, const float* rk, float* hv,
                                    int32_t* hi, int32_t* status, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  CUtensorMap tmA, tmB;
  {
    const uint64_t dims[3] = {(uint64_t)dh, (uint64_t)H * 2, (uint64_t)T};
    const uint64_t strides[2] = {(uint64_t)dh * 2, (uint64_t)H * 2 * dh * 2};
    const uint32_t box[3] = {(uint32_t)ss::kKB, 1, (uint32_t)ss::kM};
    if (!make_tmap_bf16(&tmA, q, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {(uint64_t)dh, (uint64_t)n, (uint64_t)H * 2};
    const uint64_t strides[2] = {(uint64_t)dh * 2, (uint64_t)n * dh * 2};
    const uint32_t box[3] = {(uint32_t)ss::kKB, (uint32_t)ss::kN, 1};
    if (!make_tmap_bf16(&tmB, K, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(score_topk_small_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)ss::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(1, (unsigned)(H * 2), (unsigned)score_small_chunks(n));
  score_topk_small_kernel<<<grid, ss::kThreads, ss::kSmemBytes, stream>>>(
      tmA, tmB, (int)T, H, dh, n, k, rq, rk, hv, hi, status);
  note_launch();
  return cudaGetLastError();
}

}  // namespace pkm
