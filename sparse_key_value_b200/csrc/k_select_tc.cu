// k_select_tc.cu -- the whole product-key selection in one kernel: query
// norms, sub-key scores on the tensor cores, per-half top-k, the k x k
// combine, the final top-k and the softmax weights.
//
// "Memory Layers at Scale" digest, "Product-key 검색": the key is split in
// two sub-keys and the top-k of N full keys is found from 2*sqrt(N)
// comparisons; "Memory+ 블록": qk-normalization.  "모델 안의 메모리", "작동
// 방식": each half of the query is compared with its ~sqrt(N) half-keys, the
// best of each half are combined (a 1,000 x 1,000 grid searched with 2,000
// comparisons) and the values read are averaged with weights.
//
// Grid: (token tiles of 128) x (2H), one CTA per (token tile, head, half).
// Each CTA scores its 128 tokens against all n sub-keys of its (head, half),
// 128 columns per chunk:
//   warp 0     TMA producer: per chunk and 64-wide k-block the query tile
//              [128 x 64] and the sub-key tile [128 x 64] (bf16, 128-byte
//              swizzle) into a 3-stage ring.
//   warp 1     TMEM owner and MMA issuer: tcgen05.mma kind::f16, M=128,
//              N=128, K=16, fp32 accumulators in two sets of 128 TMEM
//              columns: chunk c goes to set c % 2, so the MMAs of the next
//              chunk run while the epilogue reads this one.
//   warps 2-5  epilogue, one thread per token row (TMEM lane).
// Two CTAs share an SM (112 KiB of shared memory each).
//
// Per-row top-k over the scores s = sqrt(d_half) * rq * rk[a] * acc:
//   * the epilogue filters raw products p = acc * rk[a] against a threshold
//     thr (a lower bound of the row's final k-th best p) and appends the
//     survivors (p, a) to a 16-entry per-row buffer in shared memory;
//   * whenever some row of the warp holds more than 8, the warp merges each
//     row's buffer into the row's sorted list of the k best (scores and
//     positions in registers, bitonic sort and merge networks) and raises
//     thr to the list's k-th best;
//   * before the first chunk's filter pass a histogram pass over the same
//     chunk (still in TMEM) counts the maxima of groups of 4 columns into
//     score bins of 1/16; the lower edge of the bin where the count from the
//     top reaches k bounds the chunk's (and so the row's) k-th best score
//     from below, since group maxima are distinct elements.  That starts the
//     filter near its final level instead of at -inf.
// Candidates are fp32 scores with their positions carried alongside (see
// "keys" below); exactly equal scores are ties in either order.
//
// Combine: each CTA writes its rows' sorted lists to the workspace (they
// stay in L2), then counts itself in on its (token tile, head) pair with an
// atomic after a fence; the second CTA of the pair to arrive reads both
// halves' lists back and, one warp per token, takes the top k of the cells
// of the k x k grid S[i][j] = s1[i] + s2[j] that can reach it, forms the row
// ids a*n+b and the softmax weights and writes them.  The first CTA of the pair just exits.  (A 2-CTA
// cluster exchanging the lists through distributed shared memory was
// measured first: cluster launch held this kernel to one CTA per SM.)
//
// Every spin-wait is bounded: on a timeout the CTA records PKM_ERR_TIMEOUT,
// stops issuing work, waits (bounded) for its copies and MMAs in flight,
// marks its half's lists invalid (the pair is then not combined), frees its
// TMEM and exits.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tmap.h"
#include "warp_sort32.cuh"

namespace pkm {

namespace sl {
constexpr int kM = 128;           // tokens per tile (TMEM lanes)
constexpr int kN = 128;           // sub-key columns per chunk
constexpr int kKB = 64;           // k-block width (128 bytes of bf16)
constexpr int kStages = 3;
constexpr int kAcc = 2;           // TMEM accumulators: the MMA fills one while the epilogue reads the other
constexpr int kABytes = kM * kKB * 2;   // 16 KiB
constexpr int kBBytes = kN * kKB * 2;   // 16 KiB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 192;
constexpr int kBuf = 16;          // pending candidates per row
constexpr int kFlushAt = 8;       // merge once a row holds more (checked every 8 columns)
constexpr int kMaxK = 32;
constexpr int kGroup = 4;         // columns per group maximum in the histogram pass
constexpr int kBins = 64;         // histogram bins per row, one byte each
constexpr float kBinsPerUnit = 16.0f;
constexpr float kBinOffset = 16.0f;     // bin = floor(16 s + 16) over [-1, 3): bin 1 starts at -15/16
constexpr int kPendBytes = kBuf * kM * 4 + kBuf * kM * 2;   // p (fp32) and column (u16)
// a row's bins are the words [w][row] of the fp32 part of the pending buffers,
// which hold only that row's entries: no row's bins overlap another row's data
static_assert(kBins / 4 <= kBuf, "the histogram aliases the row's own fp32 entries");
static_assert(2 * kN / kGroup <= 255, "bin counts (two chunks) fit in a byte");
constexpr int kRkBytes = 4 * kAcc * kN * 4;  // each epilogue warp's norms of the chunks in TMEM
constexpr size_t kSmemBytes =
    (size_t)kStages * kStageBytes + kPendBytes + kRkBytes + 256 /*barriers*/;
// after the last MMA the stage ring holds the combine's arrays: both halves'
// lists (scores and positions, [2][32][129], one column per row) and the
// table of the k x k cells that can reach the top k
constexpr int kHeapPad = kM + 1;
constexpr int kCellSlots = 128;   // >= the cells (i+1)(j+1) <= 32 (119)
constexpr int kCombOff = (2 * kMaxK * kHeapPad * 6 + 255) / 256 * 256;
static_assert(kCombOff + kCellSlots * 2 <= kStages * kStageBytes,
              "both halves' lists and the cell table fit in the stage ring");
constexpr int kListKeys = kMaxK * kM;  // keys of one (tile, head, half) list block [32][128]
}  // namespace sl

struct SelectCtl {
  uint64_t full[sl::kStages];
  uint64_t empty[sl::kStages];
  uint64_t aread[sl::kStages];  // the epilogue has read the query rows of a first-chunk stage
  uint64_t accf[sl::kAcc];
  uint64_t acce[sl::kAcc];
  uint64_t drain;
  uint32_t tmem;
  volatile int abort;
  int combine;  // this CTA is the second of its pair and both halves are valid
};

// L2-coherent load (skips L1): the other CTA of the pair wrote these
__device__ __forceinline__ uint64_t ld_cg_u64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.global.cg.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// 8 columns of the accumulator; the wait names the registers so that no use
// of them is moved above it
__device__ __forceinline__ void tmem_wait_x8(uint32_t (&r)[8]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7])
               :
               : "memory");
}

// ---------------------------------------------------------------- keys --
// A candidate is its fp32 score (-inf: empty) and its position or row id
// (u32), held as two parallel register arrays: the exchange networks compare
// the scores with fp32 max / min and move the ids with one select each, all
// 32-bit work (a 64-bit key ordering the id too was measured 3.8x slower per
// exchange on B200).  Exactly equal scores may come out in either order; the
// selection rules treat equal scores as ties.

__device__ __forceinline__ float canon(float s) { return s + 0.0f; }  // -0 -> +0

__device__ __forceinline__ void cas_desc(float& a, uint32_t& ai, float& b, uint32_t& bi) {
  const bool sw = b > a;
  const float hi = fmaxf(a, b), lo = fminf(a, b);
  const uint32_t h = sw ? bi : ai, l = sw ? ai : bi;
  a = hi;
  b = lo;
  ai = h;
  bi = l;
}

// sort 16 candidates descending (bitonic network)
__device__ __forceinline__ void sort16_desc(float* v, uint32_t* c) {
#pragma unroll
  for (int size = 2; size <= 16; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int j = i ^ stride;
        if (j > i) {
          if ((i & size) == 0) {
            cas_desc(v[i], c[i], v[j], c[j]);
          } else {
            cas_desc(v[j], c[j], v[i], c[i]);
          }
        }
      }
    }
  }
}

// L (sorted desc, 32) <- top 32 of L u B (B sorted desc, 16): the larger of
// L[i] and B[31-i] for i >= 16 makes L bitonic, five exchange stages sort it
__device__ __forceinline__ void merge16_desc(float* L, uint32_t* Lc, const float* B,
                                             const uint32_t* Bc) {
#pragma unroll
  for (int i = 16; i < 32; ++i) {
    const bool sw = B[31 - i] > L[i];
    L[i] = fmaxf(L[i], B[31 - i]);
    Lc[i] = sw ? Bc[31 - i] : Lc[i];
  }
#pragma unroll
  for (int stride = 16; stride > 0; stride >>= 1) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if ((i & stride) == 0) cas_desc(L[i], Lc[i], L[i + stride], Lc[i + stride]);
    }
  }
}

// list entries in the workspace: the score's bits, then the position / id
__device__ __forceinline__ uint64_t pack_entry(float s, uint32_t c) {
  return ((uint64_t)c << 32) | (uint64_t)__float_as_uint(s);
}
__device__ __forceinline__ float entry_score(uint64_t e) { return __uint_as_float((uint32_t)e); }
__device__ __forceinline__ uint32_t entry_id(uint64_t e) { return (uint32_t)(e >> 32); }

// thr_raw <- max(thr_raw, a filter level for the raw products): any column
// whose score s = p * rowf (rounded) is >= thr has p above the returned
// level, which is thr * (1/rowf) lowered by 2^-20 relative (more than the
// two roundings of the estimate).  A level that overflows is ignored.
__device__ __forceinline__ void raise_threshold(float& thr_raw, float thr, float inv_rowf) {
  const float r = thr * inv_rowf;
  const float t = r - fabsf(r) * 9.5367431640625e-7f;
  if (fabsf(t) < INFINITY) thr_raw = fmaxf(thr_raw, t);
}

// Merge the row's pending candidates (pairs (p, column) at a stride of 128
// entries, cnt of them) into its sorted list (L, Lc), empty the buffer and
// raise the filter level to the list's k-th best.
template <bool K32>
__device__ __forceinline__ void flush_pending(float (&L)[32], uint32_t (&Lc)[32],
                                              const float* pp, const uint16_t* pc, int& cnt,
                                              float& thr_raw, int k, float rowf,
                                              float inv_rowf) {
  float B[sl::kBuf];
  uint32_t Bc[sl::kBuf];
#pragma unroll
  for (int j = 0; j < sl::kBuf; ++j) {  // all kBuf slots are read, those past cnt dropped
    const float pv = pp[j * sl::kM];
    const uint32_t pcv = pc[j * sl::kM];
    B[j] = j < cnt ? canon(pv * rowf) : -INFINITY;
    Bc[j] = j < cnt ? pcv : 0xffffffffu;
  }
  sort16_desc(B, Bc);
  merge16_desc(L, Lc, B, Bc);
  cnt = 0;
  float kth;
  if constexpr (K32) {
    kth = L[31];
  } else {
    kth = L[0];
#pragma unroll
    for (int i = 1; i < 32; ++i)
      if (i == k - 1) kth = L[i];
  }
  if (kth > -INFINITY) raise_threshold(thr_raw, kth, inv_rowf);
}

// bounded wait that also gives up when another role of the CTA aborted
__device__ __forceinline__ bool wait_sel(uint64_t* bar, uint32_t parity, SelectCtl* ctl,
                                         int32_t* status) {
  return mbar_wait_or_abort(bar, parity, &ctl->abort, status);
}

// The products p = acc * rk of 8 columns (norms from the warp's shared copy
// of the chunk's inverse sub-key norms, read as broadcasts); columns at or
// past ncols read as -inf.
__device__ __forceinline__ void products8(const uint32_t (&r)[8], const float* rkw, int g,
                                          int ncols, float (&p)[8]) {
  const float4* kv = reinterpret_cast<const float4*>(rkw + g * 8);
  const float4 a = kv[0], b = kv[1];
  p[0] = __uint_as_float(r[0]) * a.x;
  p[1] = __uint_as_float(r[1]) * a.y;
  p[2] = __uint_as_float(r[2]) * a.z;
  p[3] = __uint_as_float(r[3]) * a.w;
  p[4] = __uint_as_float(r[4]) * b.x;
  p[5] = __uint_as_float(r[5]) * b.y;
  p[6] = __uint_as_float(r[6]) * b.z;
  p[7] = __uint_as_float(r[7]) * b.w;
  if (g * 8 + 8 > ncols) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (g * 8 + j >= ncols) p[j] = -INFINITY;
  }
}

template <bool K32>
__global__ void __launch_bounds__(sl::kThreads, 2) select_tc_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int64_t T,
    int H, int dh, int n, int k, const float* __restrict__ rk, int32_t* __restrict__ idx,
    float* __restrict__ wout, uint64_t* __restrict__ lists, int32_t* __restrict__ pair_count,
    int32_t* __restrict__ half_ok, int32_t* status) {
  using namespace sl;
  // dynamic shared memory starts 1024-byte aligned (the 128-byte swizzle of
  // the TMA tiles needs it); checked below
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* stages = smem_raw;
  float* pend_p = reinterpret_cast<float*>(smem_raw + kStages * kStageBytes);  // [kBuf][128]
  uint16_t* pend_c = reinterpret_cast<uint16_t*>(pend_p + kBuf * kM);          // [kBuf][128]
  unsigned char* hist = reinterpret_cast<unsigned char*>(pend_p);  // words [kBins/4][128]
  float* rkbuf = reinterpret_cast<float*>(smem_raw + kStages * kStageBytes + kPendBytes);
  SelectCtl* ctl =
      reinterpret_cast<SelectCtl*>(smem_raw + kStages * kStageBytes + kPendBytes + kRkBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hc = blockIdx.y;  // 2h + half
  const int h = hc >> 1;
  const int64_t m0 = (int64_t)blockIdx.x * kM;
  const int nch = (n + kN - 1) / kN;
  const int KB = dh / kKB;
  const bool misaligned = (smem_u32(smem_raw) & 1023u) != 0;  // the same in every CTA
  // the next kernel (the Memory+ gate GEMM, which reads neither idx nor w)
  // may start on SMs this grid's last wave leaves free
  pdl_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
      mbar_init(&ctl->aread[s], 4);
    }
    for (int b = 0; b < kAcc; ++b) {
      mbar_init(&ctl->accf[b], 1);
      mbar_init(&ctl->acce[b], 4);
    }
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
    tmem_alloc(&ctl->tmem, kAcc * kN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem;
  const bool run = !misaligned;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0 && run) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_par = 0;
      bool ok = true;
      int f = 0;  // stage fills so far
      for (int c = 0; c < nch && ok; ++c) {
        for (int kb = 0; kb < KB; ++kb, ++f) {
          if (!wait_sel(&ctl->empty[stage], phase ^ 1, ctl, status)) { ok = false; break; }
          // a first-chunk stage is refilled only after the epilogue read its query rows
          if (f >= kStages && f - kStages < KB &&
              !wait_sel(&ctl->aread[stage], ((f - kStages) / kStages) & 1, ctl, status)) {
            ok = false;
            break;
          }
          unsigned char* sa = stages + stage * kStageBytes;
          mbar_arrive_expect_tx(&ctl->full[stage], kStageBytes);
          tma_load_3d(sa, &tmA, &ctl->full[stage], kb * kKB, hc, (int32_t)m0);
          tma_load_3d(sa + kABytes, &tmB, &ctl->full[stage], kb * kKB, c * kN, hc);
          issued_mask |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {  // let every copy in flight land before the CTA moves on
        for (int s = 0; s < kStages; ++s)
          if (issued_mask & (1u << s)) {
            for (unsigned long long i = 0; i < kSpinLimit; ++i)
              if (mbar_try_wait(&ctl->full[s], (issued_par >> s) & 1)) break;
          }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0 && run) {
      const uint32_t idesc = idesc_bf16_f32(kM, kN);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int c = 0; c < nch && ok; ++c) {
        // accumulator c % 2 is free once the epilogue has read chunk c - 2
        const int b = c & 1;
        if (!wait_sel(&ctl->acce[b], ((c >> 1) & 1) ^ 1, ctl, status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dt = tmem + (uint32_t)(b * kN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!wait_sel(&ctl->full[stage], phase, ctl, status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(stages + stage * kStageBytes);
          const uint32_t sb = sa + kABytes;
#pragma unroll
          for (int kk = 0; kk < kKB / 16; ++kk)
            tc_mma_f16(dt, smem_desc_k128(sa + kk * 32), smem_desc_k128(sb + kk * 32), idesc,
                       (kb | kk) != 0);
          tc_commit(&ctl->empty[stage]);  // the stage is free once these MMAs finish
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        if (ok) tc_commit(&ctl->accf[b]);
      }
      // every MMA issued must complete before TMEM is released
      tc_commit(&ctl->drain);
      for (unsigned long long i = 0; i < kSpinLimit; ++i)
        if (mbar_try_wait(&ctl->drain, 0)) break;
    }
  } else if (run) {
    // ----------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes this warp may read
    const int row = quarter * 32 + lane;
    const int64_t t = m0 + row;
    const bool live = t < T;
    float* pp = pend_p + row;   // entry j at pp[128 j]
    uint16_t* pc = pend_c + row;
    float* rkw = rkbuf + (warp - 2) * kAcc * kN;  // this warp's norms of chunk c at rkw[128 (c & 1)]
    const float* rkc = rk + (int64_t)hc * n;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    bool ok = true;

    // 1. the row's query norm from the first chunk's stages
    float ss[4] = {0.f, 0.f, 0.f, 0.f};  // four partial sums: short FMA chains
    for (int kb = 0; kb < KB; ++kb) {
      const int stage = kb % kStages;
      const bool got = wait_sel(&ctl->full[stage], (kb / kStages) & 1, ctl, status);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      // piece u ^ (row & 7) at step u: neighbouring rows on different banks
      const uint4* arow = reinterpret_cast<const uint4*>(stages + stage * kStageBytes + row * 128);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint4 v = arow[u ^ (row & 7)];
        float f[8];
        unpack16<PKM_BF16>(v, f);
#pragma unroll
        for (int e = 0; e < 8; ++e) ss[e & 3] = fmaf(f[e], f[e], ss[e & 3]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->aread[stage]);
    }
    const float rq = 1.0f / fmaxf(sqrtf((ss[0] + ss[1]) + (ss[2] + ss[3])), kNormEps);
    const float rowf = sqrtf((float)dh) * rq;
    const float inv_rowf = 1.0f / rowf;

    float L[32];
    uint32_t Lc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      L[i] = -INFINITY;
      Lc[i] = 0xffffffffu;
    }
    int cnt = 0;
    // rows past the end of the batch keep nothing
    float thr_raw = live ? -INFINITY : INFINITY;

    // 2. the chunks; chunk c sits in accumulator c & 1
    auto stage_norms = [&](int c, float4 v) {
      reinterpret_cast<float4*>(rkw + (c & 1) * kN)[lane] = v;
    };
    auto load_norms = [&](int c) {  // the norm buffer is padded by 256 columns: in bounds
      return __ldg(reinterpret_cast<const float4*>(rkc + c * kN) + lane);
    };
    float4 kn = make_float4(0.f, 0.f, 0.f, 0.f);
    if (ok) {
      stage_norms(0, load_norms(0));
      if (nch > 1) stage_norms(1, load_norms(1));
      if (nch > 2) kn = load_norms(2);
      __syncwarp();
    }
    for (int it = 0; it < nch && ok; ++it) {
      const int b = it & 1;
      const int c0 = it * kN;
      const int ncols = min(kN, n - c0);
      if (it >= 2) {
        __syncwarp();  // every lane is done with chunk it - 2's norms
        stage_norms(it, kn);
        __syncwarp();
        if (it + 1 < nch) kn = load_norms(it + 1);
      }
      const bool got = wait_sel(&ctl->accf[b], (it >> 1) & 1, ctl, status);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      uint32_t nxt[8], cur[8];

      if (it == 0) {
        // histogram pass over the first two chunks (both in TMEM): maxima of
        // groups of 4 columns into score bins
        const int nh = min(nch, 2);
        if (nh == 2) {
          const bool got1 = wait_sel(&ctl->accf[1], 0, ctl, status);
          if (!__all_sync(0xffffffffu, got1)) { ok = false; break; }
          tc_fence_after();
        }
        uint32_t* hw = reinterpret_cast<uint32_t*>(hist) + row;  // word w at hw[128 w]
#pragma unroll
        for (int w = 0; w < kBins / 4; ++w) hw[w * kM] = 0u;
        unsigned char* hb = hist + row * 4;  // bin b at hb[512 (b >> 2) + (b & 3)]
        const float c16 = rowf * kBinsPerUnit;
        for (int hcn = 0; hcn < nh; ++hcn) {
          const uint32_t ta = tmem + lane_base + hcn * kN;
          const float* rkv = rkw + hcn * kN;
          const int nc = min(kN, n - hcn * kN);
          tmem_ld_32x32b_x8(ta, nxt);
#pragma unroll 1
          for (int g = 0; g < kN / 8; ++g) {
            tmem_wait_x8(nxt);
#pragma unroll
            for (int j = 0; j < 8; ++j) cur[j] = nxt[j];
            if (g + 1 < kN / 8) tmem_ld_32x32b_x8(ta + (g + 1) * 8, nxt);
            float p[8];
            products8(cur, rkv, g, nc, p);
#pragma unroll
            for (int q = 0; q < 8 / kGroup; ++q) {
              const float gm = fmaxf(fmaxf(p[4 * q], p[4 * q + 1]), fmaxf(p[4 * q + 2], p[4 * q + 3]));
              const float tb = fminf(fmaxf(fmaf(gm, c16, kBinOffset), 0.f), (float)(kBins - 1));
              const int bin = (int)tb;
              hb[512 * (bin >> 2) + (bin & 3)] += 1;
            }
          }
        }
        // the bound: lower edge of the bin where the count from the top reaches k
        int cum = 0, bstar = 0;
        for (int w = kBins / 4 - 1; w >= 0; --w) {
          const uint32_t word = hw[w * kM];
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
        // members of bin b >= 1 have s >= (b - 16) / 16 up to rounding; 2^-10 covers it
        if (bstar > 0)
          raise_threshold(thr_raw, ((float)bstar - kBinOffset) / kBinsPerUnit - 9.765625e-4f,
                          inv_rowf);
        __syncwarp();  // the bins become the pending buffers
      }

      // filter pass: products above the level into the row's buffer; one
      // merge site for the whole loop keeps the code (and its misses) small
      const uint32_t taddr = tmem + lane_base + b * kN;
      const float* rkv = rkw + b * kN;
      tmem_ld_32x32b_x8(taddr, nxt);
#pragma unroll 1
      for (int g = 0; g < kN / 8; ++g) {
        tmem_wait_x8(nxt);
#pragma unroll
        for (int j = 0; j < 8; ++j) cur[j] = nxt[j];
        if (g + 1 < kN / 8) tmem_ld_32x32b_x8(taddr + (g + 1) * 8, nxt);
        float p[8];
        products8(cur, rkv, g, ncols, p);
        const int col0 = c0 + g * 8;
        // predicated appends (unconditional stores at the next free slot
        // measured slower: the extra shared-memory writes compete with the
        // MMAs' operand reads)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (p[j] > thr_raw) {
            pp[cnt * kM] = p[j];
            pc[cnt * kM] = (uint16_t)(col0 + j);
            ++cnt;
          }
        }
        if (__any_sync(0xffffffffu, cnt > kFlushAt))
          flush_pending<K32>(L, Lc, pp, pc, cnt, thr_raw, k, rowf, inv_rowf);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->acce[b]);
    }
    if (ok) {
      if (__any_sync(0xffffffffu, cnt > 0))
        flush_pending<K32>(L, Lc, pp, pc, cnt, thr_raw, k, rowf, inv_rowf);
      // the sorted list into this (tile, head, half)'s block [32][128] of the workspace
      uint64_t* list = lists + ((int64_t)blockIdx.x * gridDim.y + hc) * kListKeys;
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i < k) list[i * kM + row] = pack_entry(L[i], Lc[i]);
      __threadfence();  // the list is visible device-wide before the pair count below
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1 && run) {
    tc_fence_after();
    tmem_dealloc(tmem, kAcc * kN);
  }

  // -------------------------------------------------------- k x k combine
  // count this half in on its (tile, head) pair; the second to arrive combines
  const int64_t pair = (int64_t)blockIdx.x * H + h;
  if (threadIdx.x == 0) {
    half_ok[pair * 2 + (hc & 1)] = ctl->abort == 0 ? 1 : 0;
    __threadfence();  // this CTA's lists and flag before the count
    const int prev = atomicAdd(pair_count + pair, 1);
    int go = 0;
    if (prev == 1) {
      __threadfence();  // the other half's lists and flag after the count
      const volatile int32_t* other = half_ok + pair * 2 + ((hc & 1) ^ 1);
      go = ctl->abort == 0 && *other != 0;
    }
    ctl->combine = go;
  }
  __syncthreads();
  if (ctl->combine) {
    constexpr int P = kHeapPad;
    float* sv = reinterpret_cast<float*>(stages);                    // [2][32][P] scores
    uint16_t* cv = reinterpret_cast<uint16_t*>(sv + 2 * kMaxK * P);  // [2][32][P] positions
    uint16_t* cells = reinterpret_cast<uint16_t*>(stages + kCombOff);  // [128]
    const uint64_t* pl = lists + ((int64_t)blockIdx.x * gridDim.y + 2 * h) * kListKeys;
    // the cells (i, j) with (i+1)(j+1) <= k, row-major
    if (threadIdx.x < kCellSlots) cells[threadIdx.x] = topk_cell(threadIdx.x, k);
    // both halves' lists of the tile's rows (L2): half c's entry j of row r at sv[c][j][r]
    for (int e = threadIdx.x; e < 2 * k * kM; e += kThreads) {
      const int half = e / (k * kM);
      const int j = (e / kM) % k;
      const int r = e % kM;
      const uint64_t ent = ld_cg_u64(pl + (int64_t)half * kListKeys + j * kM + r);
      sv[(half * kMaxK + j) * P + r] = entry_score(ent);
      cv[(half * kMaxK + j) * P + r] = (uint16_t)entry_id(ent);
    }
    __syncthreads();
    const int rows = T - m0 < kM ? (int)(T - m0) : kM;
    for (int r = warp; r < rows; r += kThreads / 32) {
      const int64_t o = ((m0 + r) * H + h) * k;
      const bool in = lane < k;
      const int e = lane * P + r;
      combine_lists_warp<K32>(in ? sv[e] : -INFINITY, in ? cv[e] : 0u,
                              in ? sv[kMaxK * P + e] : -INFINITY, in ? cv[kMaxK * P + e] : 0u,
                              cells, n, k, idx + o, wout + o);
    }
  }
}

bool select_tc_supported(pkm_dtype dt, int dh, int n, int k) {
  // n % 4: the epilogue reads the inverse sub-key norms as aligned float4;
  // n < 65536: positions are held as 16 bits
  return dt == PKM_BF16 && dh % sl::kKB == 0 && dh <= 2048 && n >= sl::kN && n % 4 == 0 &&
         n < 65536 && k <= sl::kMaxK;
}

size_t select_tc_workspace(int64_t T, int H) {
  const size_t tiles = (size_t)((T + sl::kM - 1) / sl::kM);
  const size_t lists = tiles * H * 2 * sl::kListKeys * sizeof(uint64_t);
  const size_t counts = (tiles * H * 3 * sizeof(int32_t) + 255) / 256 * 256;
  return lists + counts;
}

cudaError_t launch_select_tc(const void* q, const void* K, int64_t T, int H, int dh, int n,
                             int k, const float* rk, int32_t* idx, float* w, void* workspace,
                             int32_t* status, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const int64_t tiles = (T + sl::kM - 1) / sl::kM;
  uint64_t* lists = static_cast<uint64_t*>(workspace);
  int32_t* pair_count = reinterpret_cast<int32_t*>(lists + tiles * H * 2 * sl::kListKeys);
  int32_t* half_ok = pair_count + tiles * H;
  cudaError_t e = cudaMemsetAsync(pair_count, 0, sizeof(int32_t) * tiles * H, stream);
  if (e != cudaSuccess) return e;
  CUtensorMap tmA, tmB;
  {
    const uint64_t dims[3] = {(uint64_t)dh, (uint64_t)H * 2, (uint64_t)T};
    const uint64_t strides[2] = {(uint64_t)dh * 2, (uint64_t)H * 2 * dh * 2};
    const uint32_t box[3] = {(uint32_t)sl::kKB, 1, (uint32_t)sl::kM};
    if (!make_tmap_bf16(&tmA, q, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {(uint64_t)dh, (uint64_t)n, (uint64_t)H * 2};
    const uint64_t strides[2] = {(uint64_t)dh * 2, (uint64_t)n * dh * 2};
    const uint32_t box[3] = {(uint32_t)sl::kKB, (uint32_t)sl::kN, 1};
    if (!make_tmap_bf16(&tmB, K, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  auto kern = k == 32 ? select_tc_kernel<true> : select_tc_kernel<false>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)sl::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)tiles, (unsigned)(H * 2), 1);
  kern<<<grid, sl::kThreads, sl::kSmemBytes, stream>>>(tmA, tmB, T, H, dh, n, k, rk, idx, w,
                                                       lists, pair_count, half_ok, status);
  note_launch();
  return cudaGetLastError();
}

}  // namespace pkm
