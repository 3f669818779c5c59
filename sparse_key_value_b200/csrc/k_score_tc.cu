// k_score_tc.cu -- sub-key scoring on the tensor cores with the per-half
// top-k fused into the epilogue.
//
// "모델 안의 메모리", "작동 방식": each half of the query is compared with all
// of its ~sqrt(N) half-keys and the best are kept; "Memory Layers at Scale"
// digest, "Product-key 검색": 2*sqrt(N) comparisons per lookup.  For one
// (head h, half c) the comparisons of 128 tokens against 256 half-keys form
// the GEMM tile D[128 x 256] = Q_c[128 x d_half] * K_c[256 x d_half]^T.
//
// Per CTA: 128 tokens x one (h, c) x a range of 256-column chunks; two CTAs
// share an SM, so the MMAs of one overlap the epilogue of the other.
//   warp 0     TMA producer: per chunk and 64-wide k-block, the query tile
//              [128 x 64] and the sub-key tile [256 x 64] (bf16, 128-byte
//              swizzle) into a 2-stage ring.
//   warp 1     TMEM owner and MMA issuer: tcgen05.mma kind::f16, M=128,
//              N=256, K=16, fp32 accumulator in 256 TMEM columns.
//   warps 2-5  epilogue, one thread per token row (TMEM lane), reading its
//              row's 256 products with tcgen05.ld and scaling them,
//                p = acc * rk[a],   s = p * (sqrt(d_half) * rq).
//
// The epilogue keeps a running top-k per row in two passes over the chunks:
//   prefix pass  over the first P chunks: the maximum of every group of 8
//                columns goes into a per-row byte histogram of s (bins of
//                1/16 over [-2, 6)).  Group maxima are distinct elements,
//                so the lower edge of the bin where the count from the top
//                reaches k is a lower bound of the row's k-th best score.
//   main pass    over all chunks (starting with the one still in TMEM, so
//                it is computed once): products above the bound (and above
//                the running k-th best) go to a 16-entry per-row buffer in
//                shared memory; when any row of the warp has more than 8,
//                the warp sorts each buffer with a bitonic network in
//                registers and merges it into the row's sorted list of 32
//                64-bit keys (order-preserving score bits, then the
//                complemented column, so ties favour the smaller id).
// The histogram and the buffer share each warp's 4 KiB of shared memory.
// The raw bf16 inputs feed the MMA (products exact in fp32); the
// normalisation is applied in fp32 in the epilogue.
//
// Every spin-wait is bounded: on a timeout the CTA records PKM_ERR_TIMEOUT,
// stops issuing work, waits (bounded) for its copies and MMAs in flight,
// frees its TMEM and exits.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tmap.h"

namespace pkm {

namespace sc {
constexpr int kM = 128;           // tokens per tile (TMEM lanes)
constexpr int kN = 256;           // sub-key columns per chunk
constexpr int kKB = 64;           // k-block width (128 bytes of bf16)
constexpr int kStages = 2;
constexpr int kABytes = kM * kKB * 2;   // 16 KiB
constexpr int kBBytes = kN * kKB * 2;   // 32 KiB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kBuf = 16;          // pending candidates per row
constexpr int kCheck = 8;         // columns between overflow checks
constexpr int kFlushAt = kBuf - kCheck;
constexpr int kThreads = 192;
constexpr int kCtasPerSm = 2;     // two CTAs share an SM: their MMAs and epilogues interleave
constexpr int kMaxK = 32;
constexpr int kGroup = 8;         // columns per group maximum in the prefix pass
constexpr int kBins = 128;        // histogram bins per row, one byte each
constexpr float kBinsPerUnit = 16.0f;
constexpr float kBinOffset = 32.0f;     // bin = floor(16 * s + 32): bin 1 starts at s = -1.9375
constexpr int kMaxPrefix = 4;     // chunks in the prefix pass
constexpr int kWarpBytes = 32 * kBuf * 8;  // one epilogue warp's buffers or histograms
static_assert(kWarpBytes == 32 * kBins, "the histogram and the buffers share a region");
static_assert(kMaxPrefix * (kN / kGroup) <= 255, "bin counts fit in a byte");
constexpr size_t kSmemBytes = (size_t)kStages * kStageBytes + 4 * (size_t)kWarpBytes +
                              128 /*barriers*/;
}  // namespace sc

struct ScoreSmemCtl {
  uint64_t full[sc::kStages];
  uint64_t empty[sc::kStages];
  uint64_t accf;
  uint64_t acce;
  uint64_t drain;
  uint32_t tmem;
  volatile int abort;
};

// bounded wait that also gives up when another role of the CTA aborted
__device__ __forceinline__ bool wait_ctl(uint64_t* bar, uint32_t parity, ScoreSmemCtl* ctl,
                                         int32_t* status) {
  return mbar_wait_or_abort(bar, parity, &ctl->abort, status);
}

__device__ __forceinline__ uint32_t ord_f32(float s) {
  uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float unord_f32(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}
__device__ __forceinline__ uint64_t pack_key(float s, int32_t id) {
  return ((uint64_t)ord_f32(s) << 32) | (uint64_t)(0xffffffffu - (uint32_t)id);
}

// thr_raw <- max(thr_raw, a filter level for the raw products): any column
// whose score s = p * rowf (rounded) is >= thr has p above the returned
// level, since it is thr / rowf lowered by 2^-20 relative.  A level that
// overflows (rowf tiny or zero) leaves thr_raw as it is.
__device__ __forceinline__ void raise_threshold(float& thr_raw, float thr, float rowf) {
  const float r = thr / rowf;
  const float t = r - fabsf(r) * 9.5367431640625e-7f;
  if (fabsf(t) < INFINITY) thr_raw = fmaxf(thr_raw, t);
}

// Chunk (relative to the CTA's first) of step `it` with a prefix pass over
// the first P chunks: steps 0..P-1 are the prefix chunks 0..P-1; step P-1
// also runs the main pass on the chunk still in TMEM, so the main pass goes
// on with chunks 0..P-2 and P.. at steps P..  The MMA issuer computes one
// chunk per step, so chunk P-1 is computed once.
__device__ __forceinline__ int chunk_of(int it, int P) {
  if (it < P || P == 0) return it;
  const int r = it - P;
  return r < P - 1 ? r : r + 1;
}

#define CAS_DESC(a, b)                 \
  {                                    \
    uint64_t x_ = (a), y_ = (b);       \
    (a) = x_ > y_ ? x_ : y_;           \
    (b) = x_ > y_ ? y_ : x_;           \
  }

// sort 32 keys descending (bitonic network, fully unrolled)
__device__ __forceinline__ void sort32_desc(uint64_t* v) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int j = i ^ stride;
        if (j > i) {
          if ((i & size) == 0) {
            CAS_DESC(v[i], v[j]);
          } else {
            CAS_DESC(v[j], v[i]);
          }
        }
      }
    }
  }
}

// sort 16 keys descending
__device__ __forceinline__ void sort16_desc(uint64_t* v) {
#pragma unroll
  for (int size = 2; size <= 16; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int j = i ^ stride;
        if (j > i) {
          if ((i & size) == 0) {
            CAS_DESC(v[i], v[j]);
          } else {
            CAS_DESC(v[j], v[i]);
          }
        }
      }
    }
  }
}

// L (sorted desc, 32) <- top 32 of L u B (B sorted desc, 16)
__device__ __forceinline__ void merge16_desc(uint64_t* L, const uint64_t* B) {
#pragma unroll
  for (int i = 16; i < 32; ++i) L[i] = L[i] > B[31 - i] ? L[i] : B[31 - i];
#pragma unroll
  for (int stride = 16; stride > 0; stride >>= 1) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if ((i & stride) == 0) CAS_DESC(L[i], L[i + stride]);
    }
  }
}

// L (sorted desc) <- top 32 of L u B (B sorted desc)
__device__ __forceinline__ void merge32_desc(uint64_t* L, const uint64_t* B) {
#pragma unroll
  for (int i = 0; i < 32; ++i) L[i] = L[i] > B[31 - i] ? L[i] : B[31 - i];
#pragma unroll
  for (int stride = 16; stride > 0; stride >>= 1) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if ((i & stride) == 0) CAS_DESC(L[i], L[i + stride]);
    }
  }
}

// Merge the thread's pending candidates (pairs (p, column) at a stride of 32
// entries from pend up to wp) into its sorted list L, empty the buffer and
// refresh the filter threshold.
__device__ __forceinline__ void flush_pending(uint64_t (&L)[32], float2* pend, float2*& wp,
                                              float& thr_raw, int k, float rowf) {
  const int cnt = (int)(wp - pend) >> 5;
  uint64_t B[sc::kBuf];
#pragma unroll
  for (int j = 0; j < sc::kBuf; ++j) {
    const float2 e = pend[j * 32];
    B[j] = j < cnt ? pack_key(e.x * rowf, __float_as_int(e.y)) : 0ull;
  }
  sort16_desc(B);
  merge16_desc(L, B);
  wp = pend;
  uint64_t kth = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if (i == k - 1) kth = L[i];
  if (kth != 0) raise_threshold(thr_raw, unord_f32((uint32_t)(kth >> 32)), rowf);
}

// The inverse sub-key norms of one chunk, 8 consecutive columns per lane
// (lane l holds columns 8l..8l+7), loaded before the chunk's accumulator is
// waited for so that the global-memory latency is hidden.  The buffer is
// padded by one chunk, so the reads past column n stay inside it.
struct ChunkNorms {
  float4 lo, hi;
};
__device__ __forceinline__ ChunkNorms load_chunk_norms(const float* rk_chunk, int lane) {
  const float4* p = reinterpret_cast<const float4*>(rk_chunk + lane * 8);
  return ChunkNorms{__ldg(p), __ldg(p + 1)};
}

// The products p = acc * rk[a] of the 8 columns of group g of the chunk in
// TMEM; columns at or past ncols read as -inf.
__device__ __forceinline__ void load_products8(uint32_t taddr, const ChunkNorms& kn, int g,
                                               int ncols, float (&p)[8]) {
  uint32_t r[8];
  tmem_ld_32x32b_x8(taddr, r);
  const float kr[8] = {__shfl_sync(0xffffffffu, kn.lo.x, g), __shfl_sync(0xffffffffu, kn.lo.y, g),
                       __shfl_sync(0xffffffffu, kn.lo.z, g), __shfl_sync(0xffffffffu, kn.lo.w, g),
                       __shfl_sync(0xffffffffu, kn.hi.x, g), __shfl_sync(0xffffffffu, kn.hi.y, g),
                       __shfl_sync(0xffffffffu, kn.hi.z, g), __shfl_sync(0xffffffffu, kn.hi.w, g)};
  tmem_ld_wait();
#pragma unroll
  for (int j = 0; j < 8; ++j) p[j] = __uint_as_float(r[j]) * kr[j];
  if (g * 8 + 8 > ncols) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (g * 8 + j >= ncols) p[j] = -INFINITY;
  }
}

__global__ void __launch_bounds__(sc::kThreads, sc::kCtasPerSm) score_topk_tc_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int64_t T,
    int H, int dh, int n, int k, int chunks_per_split, int prefix, const float* __restrict__ rq,
    const float* __restrict__ rk, float* __restrict__ hv, int32_t* __restrict__ hi,
    int32_t* status) {
  // dynamic shared memory starts 1024-byte aligned (required by the 128-byte
  // swizzle of the TMA tiles); checked below
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* stages = smem_raw;
  unsigned char* regions = smem_raw + sc::kStages * sc::kStageBytes;
  ScoreSmemCtl* ctl = reinterpret_cast<ScoreSmemCtl*>(regions + 4 * sc::kWarpBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hc = blockIdx.y;
  const int64_t m0 = (int64_t)blockIdx.x * sc::kM;
  const int n_chunks = (n + sc::kN - 1) / sc::kN;
  const int c_begin = blockIdx.z * chunks_per_split;
  const int c_end = min(n_chunks, c_begin + chunks_per_split);
  const int nch = c_end - c_begin;
  // prefix chunks 0..P-1, then the main pass P-1 (reused), 0..P-2, P..nch-1
  const int P = min(prefix, nch);
  const int iters = P > 0 ? nch + P - 1 : nch;
  const int KB = dh / sc::kKB;
  if ((smem_u32(smem_raw) & 1023u) != 0) {  // uniform: every thread leaves
    if (threadIdx.x == 0) set_status(status, PKM_ERR_DEVICE);
    return;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < sc::kStages; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    mbar_init(&ctl->accf, 1);
    mbar_init(&ctl->acce, 4);
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem, sc::kN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_par = 0;
      bool ok = true;
      for (int it = 0; it < iters && ok; ++it) {
        const int c = c_begin + chunk_of(it, P);
        for (int kb = 0; kb < KB; ++kb) {
          if (!wait_ctl(&ctl->empty[stage], phase ^ 1, ctl, status)) { ok = false; break; }
          unsigned char* sa = stages + stage * sc::kStageBytes;
          mbar_arrive_expect_tx(&ctl->full[stage], sc::kStageBytes);
          tma_load_3d(sa, &tmA, &ctl->full[stage], kb * sc::kKB, hc, (int32_t)m0);
          tma_load_3d(sa + sc::kABytes, &tmB, &ctl->full[stage], kb * sc::kKB, c * sc::kN, hc);
          issued_mask |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == sc::kStages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {  // let every copy in flight land before the CTA exits
        for (int s = 0; s < sc::kStages; ++s)
          if (issued_mask & (1u << s)) {
            for (unsigned long long i = 0; i < kSpinLimit; ++i)
              if (mbar_try_wait(&ctl->full[s], (issued_par >> s) & 1)) break;
          }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(sc::kM, sc::kN);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      uint32_t use = 0;
      for (int it = 0; it < iters && ok; ++it, use ^= 1) {
        // the accumulator is free once the epilogue has read the last chunk
        if (!wait_ctl(&ctl->acce, use ^ 1, ctl, status)) { ok = false; break; }
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb) {
          if (!wait_ctl(&ctl->full[stage], phase, ctl, status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(stages + stage * sc::kStageBytes);
          const uint32_t sb = sa + sc::kABytes;
#pragma unroll
          for (int kk = 0; kk < sc::kKB / 16; ++kk) {
            tc_mma_f16(tmem, smem_desc_k128(sa + kk * 32), smem_desc_k128(sb + kk * 32), idesc,
                       (kb | kk) != 0);
          }
          tc_commit(&ctl->empty[stage]);  // the stage is free once these MMAs finish
          if (++stage == sc::kStages) { stage = 0; phase ^= 1; }
        }
        if (ok) tc_commit(&ctl->accf);
      }
      // every MMA issued must complete before TMEM is released
      tc_commit(&ctl->drain);
      for (unsigned long long i = 0; i < kSpinLimit; ++i)
        if (mbar_try_wait(&ctl->drain, 0)) break;
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes this warp may read
    const int row = quarter * 32 + lane;
    const int64_t t = m0 + row;
    const bool live = t < T;
    const float rowf = live ? sqrtf((float)dh) * rq[t * H * 2 + hc] : 0.f;
    const float c16 = rowf * sc::kBinsPerUnit;
    const float* rkc = rk + (int64_t)hc * n;
    unsigned char* region = regions + quarter * sc::kWarpBytes;
    float2* pw = reinterpret_cast<float2*>(region) + lane;  // entry j at pw[32 * j]
    float2* wp = pw;                                        // next free entry
    unsigned char* hrow = region + lane * sc::kBins;        // bin b at hrow[b ^ (lane << 2)]
    const int hswz = lane << 2;
    uint64_t L[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) L[i] = 0;
    // rows past the end of the batch (or with a zero query) keep nothing
    float thr_raw = live && rowf > 0.f ? -INFINITY : INFINITY;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    if (P > 0) {
#pragma unroll
      for (int i = 0; i < sc::kBins / 16; ++i)
        reinterpret_cast<uint4*>(hrow)[(i + lane) & 7] = make_uint4(0u, 0u, 0u, 0u);
    }

    uint32_t use = 0;
    bool ok = true;
    for (int it = 0; it < iters; ++it, use ^= 1) {
      const int c = c_begin + chunk_of(it, P);
      const int c0 = c * sc::kN;
      const ChunkNorms kn = load_chunk_norms(rkc + c0, lane);
      const bool got = wait_ctl(&ctl->accf, use, ctl, status);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      const int ncols = min(sc::kN, n - c0);
      if (it < P) {
        // prefix pass: histogram of the group maxima
        for (int g = 0; g < sc::kN / 8; ++g) {
          if (g * 8 >= ncols) break;
          float p[8];
          load_products8(tmem + lane_base + g * 8, kn, g, ncols, p);
          const float gm = fmaxf(fmaxf(fmaxf(p[0], p[1]), fmaxf(p[2], p[3])),
                                 fmaxf(fmaxf(p[4], p[5]), fmaxf(p[6], p[7])));
          const float tb = fminf(fmaxf(fmaf(gm, c16, sc::kBinOffset), 0.f), (float)(sc::kBins - 1));
          hrow[(int)tb ^ hswz] += 1;
        }
        if (it == P - 1) {
          // the bound: lower edge of the bin where the count from the top reaches k
          int cum = 0, bstar = 0;
          const uint32_t* hw = reinterpret_cast<const uint32_t*>(hrow);
          for (int w = sc::kBins / 4 - 1; w >= 0; --w) {
            const uint32_t word = hw[w ^ lane];
            const int s4 = (int)__dp4a(word, 0x01010101u, 0u);
            if (cum + s4 >= k) {
              for (int e = 3; e >= 0; --e) {
                cum += (int)((word >> (8 * e)) & 255u);
                if (cum >= k) { bstar = 4 * w + e; break; }
              }
              break;
            }
            cum += s4;
          }
          // members of bin b >= 1 have s >= (b - 32) / 16 up to rounding; 2^-10 covers it
          if (bstar > 0)
            raise_threshold(thr_raw,
                            ((float)bstar - sc::kBinOffset) / sc::kBinsPerUnit - 9.765625e-4f,
                            rowf);
          __syncwarp();  // the histograms become the candidate buffers
        }
      }
      if (it >= P - 1) {
        // main pass: candidates above the threshold into the buffer
        for (int g = 0; g < sc::kN / 8; ++g) {
          const int col0 = c0 + g * 8;
          if (g * 8 >= ncols) break;
          float p[8];
          load_products8(tmem + lane_base + g * 8, kn, g, ncols, p);
#pragma unroll
          for (int h = 0; h < 8; h += sc::kCheck) {
#pragma unroll
            for (int j = h; j < h + sc::kCheck; ++j) {
              if (p[j] > thr_raw) {
                *wp = make_float2(p[j], __int_as_float(col0 + j));
                wp += 32;
              }
            }
            if (__any_sync(0xffffffffu, wp > pw + 32 * sc::kFlushAt))
              flush_pending(L, pw, wp, thr_raw, k, rowf);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->acce);
    }
    if (ok) {
      if (__any_sync(0xffffffffu, wp != pw)) flush_pending(L, pw, wp, thr_raw, k, rowf);
      if (live) {
        const int64_t orow = ((int64_t)blockIdx.z * T + t) * H * 2 + hc;
        float* ov = hv + orow * k;
        int32_t* oi = hi + orow * k;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if (i < k) {
            const uint64_t key = L[i];
            ov[i] = key ? unord_f32((uint32_t)(key >> 32)) : -INFINITY;
            oi[i] = key ? (int32_t)(0xffffffffu - (uint32_t)key) : 0x7fffffff;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, sc::kN);
  }
}

bool score_tc_supported(pkm_dtype dt, int dh, int n, int k) {
  // n % 4: the epilogue reads the inverse sub-key norms as aligned float4
  return dt == PKM_BF16 && dh % sc::kKB == 0 && dh <= 2048 && n >= sc::kN && n % 4 == 0 &&
         k <= sc::kMaxK;
}

int score_tc_splits(int64_t T, int H, int n) {
  const int64_t tiles = (T + sc::kM - 1) / sc::kM * H * 2;
  const int chunks = (n + sc::kN - 1) / sc::kN;
  int splits = 1;
  // split the sub-key columns when the grid would not fill the 148 SMs
  while (splits < 32 && splits * 2 <= chunks && tiles * splits < 148) splits *= 2;
  // every split gets the same number of chunks
  const int per = (chunks + splits - 1) / splits;
  return (chunks + per - 1) / per;
}

// Prefix chunks per CTA: none for a single chunk (the running k-th best is
// as good there), else up to kMaxPrefix.
static int score_tc_prefix(int chunks_per_cta) {
  return chunks_per_cta <= 1 ? 0 : min(chunks_per_cta, sc::kMaxPrefix);
}

cudaError_t launch_score_topk_tc(const void* q, const void* K, int64_t T, int H, int dh, int n,
                                 int k, int splits, const float* rq, const float* rk, float* hv,
                                 int32_t* hi, int32_t* status, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  CUtensorMap tmA, tmB;
  {
    const uint64_t dims[3] = {(uint64_t)dh, (uint64_t)H * 2, (uint64_t)T};
    const uint64_t strides[2] = {(uint64_t)dh * 2, (uint64_t)H * 2 * dh * 2};
    const uint32_t box[3] = {(uint32_t)sc::kKB, 1, (uint32_t)sc::kM};
    if (!make_tmap_bf16(&tmA, q, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {(uint64_t)dh, (uint64_t)n, (uint64_t)H * 2};
    const uint64_t strides[2] = {(uint64_t)dh * 2, (uint64_t)n * dh * 2};
    const uint32_t box[3] = {(uint32_t)sc::kKB, (uint32_t)sc::kN, 1};
    if (!make_tmap_bf16(&tmB, K, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  const int chunks = (n + sc::kN - 1) / sc::kN;
  const int per = (chunks + splits - 1) / splits;
  cudaError_t e = cudaFuncSetAttribute(score_topk_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sc::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((T + sc::kM - 1) / sc::kM), (unsigned)(H * 2), (unsigned)splits);
  score_topk_tc_kernel<<<grid, sc::kThreads, sc::kSmemBytes, stream>>>(
      tmA, tmB, T, H, dh, n, k, per, score_tc_prefix(per), rq, rk, hv, hi, status);
  note_launch();
  return cudaGetLastError();
}

}  // namespace pkm
