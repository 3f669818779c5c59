// k_select_small.cu -- the whole product-key selection in one kernel for
// batches of at most 32 tokens (decode steps): sub-key norms, query norms,
// scores on the tensor cores, per-half top-k, the k x k combine, the final
// top-k and the softmax weights.
//
// "Memory Layers at Scale" digest, "Product-key 검색" (top-k of N full keys
// from 2*sqrt(N) sub-key comparisons) and "Memory+ 블록" (qk-normalization);
// "모델 안의 메모리", "작동 방식" (each query half against its ~sqrt(N)
// half-keys, the best of the two halves combined, a weighted average).
//
// With a handful of tokens the work is reading the sub-key tables, so the
// grid spreads the columns: one CTA per (256-column chunk, head, half).
//   warp 0     TMA producer: per 64-wide k-block the token tile [128 x 64]
//              (rows past T read as zero) and the chunk's sub-keys [256 x 64]
//              (bf16, 128-byte swizzle) into a 4-stage ring.
//   warp 1     TMEM owner and MMA issuer: tcgen05.mma kind::f16, M=128,
//              N=256, fp32 accumulator in 256 TMEM columns.
//   warps 6-7  the table of the k x k cells the combine reads.
//   warps 2-5  norms: while each k-block sits in shared memory they add the
//              squares of the chunk's 256 sub-key rows and of the token rows
//              (the swizzle only permutes 16-byte pieces within a row); the
//              producer refills a stage only after they have read it.  So
//              the sub-keys are read once, by the TMA, and no separate norm
//              pass runs.  Warp 4 (TMEM lanes 0..31: the tokens) then scales
//              the accumulator to scores
//                s = sqrt(d_half) * rq[t] * rk[a] * acc
//              into shared memory.
//   all warps  one token per warp: the chunk's 256 scores, 8 per lane, as
//              eight warp-sorted groups of 32 merged down to the top 32,
//              written to the workspace.
// The last CTA of a (head, half) to finish (an atomic count after a fence)
// merges the chunks' lists of every token into the half's list; the second
// of the two halves of a head to get there runs the k x k combine and the
// softmax (warp_sort32.cuh) and writes idx and w.  No CTA waits for another.
//
// Every spin-wait is bounded: on a timeout the CTA records PKM_ERR_TIMEOUT,
// stops issuing work, waits (bounded) for its copies and MMAs in flight,
// frees its TMEM and exits without counting itself in, so the merges and
// the combine of its head do not run.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tmap.h"
#include "warp_sort32.cuh"

namespace pkm {

namespace ssm {
constexpr int kM = 128;          // TMEM lanes (token tile, mostly padding)
constexpr int kN = 256;          // sub-key columns per CTA
constexpr int kKB = 64;
constexpr int kStages = 4;
constexpr int kABytes = kM * kKB * 2;
constexpr int kBBytes = kN * kKB * 2;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 256;      // 8 warps: up to 8 tokens per round of the list phases
constexpr int kWarps = kThreads / 32;
constexpr int kNormThreads = 128;  // warps 2..5
constexpr int kMaxRows = 32;
constexpr int kMaxChunks = 32;
constexpr int kList = 32;          // entries per list (>= k)
constexpr int kCellSlots = 128;
constexpr int kScoreStride = kN + 4;  // floats per score row: 16 bytes of padding spread the banks
constexpr size_t kRksOff = (size_t)kStages * kStageBytes;
constexpr size_t kRqsOff = kRksOff + kN * 4;
constexpr size_t kCellsOff = kRqsOff + kMaxRows * 4;
constexpr size_t kCtlOff = kCellsOff + kCellSlots * 2;
constexpr size_t kSmemBytes = kCtlOff + 256;
static_assert(kMaxRows * kScoreStride * 4 <= kStages * kStageBytes, "scores fit in the stage ring");
static_assert(kN == 2 * kNormThreads, "two sub-key rows per norm thread");
}  // namespace ssm

namespace {

struct SmallCtl {
  uint64_t full[ssm::kStages];
  uint64_t empty[ssm::kStages];
  uint64_t nread[ssm::kStages];  // the norm warps have read the stage
  uint64_t accf;
  uint64_t drain;
  uint32_t tmem;
  volatile int abort;
  int merge;    // this CTA merges its (head, half)'s chunk lists
  int combine;  // ... and then combines its head's two halves
};

__device__ __forceinline__ bool wait_small(uint64_t* bar, uint32_t parity, SmallCtl* ctl,
                                           int32_t* status) {
  return mbar_wait_or_abort(bar, parity, &ctl->abort, status);
}

__device__ __forceinline__ uint64_t pack_entry(float s, uint32_t id) {
  return ((uint64_t)id << 32) | (uint64_t)__float_as_uint(s);
}
__device__ __forceinline__ float entry_score(uint64_t e) { return __uint_as_float((uint32_t)e); }
__device__ __forceinline__ uint32_t entry_id(uint64_t e) { return (uint32_t)(e >> 32); }

// L2-coherent load (skips L1): other CTAs wrote these.  A plain load with the
// .cg hint, so that a warp's loads of all chunks can be in flight together
// (the __syncthreads after the count keeps them below it)
__device__ __forceinline__ uint64_t ld_cg_u64(const uint64_t* p) {
  return __ldcg(reinterpret_cast<const unsigned long long*>(p));
}

// wait for the TMEM loads in flight; names the registers of the load being
// consumed so that no use of them moves above the wait
__device__ __forceinline__ void tmem_wait_x32(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                 "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

__device__ __forceinline__ void norm_barrier() {
  asm volatile("bar.sync 1, %0;" ::"n"(ssm::kNormThreads) : "memory");
}

// sum of squares of the 64 bf16 of row `r` of a stage tile (128-byte rows).
// The lanes of a warp hold consecutive rows, so step u reads 16-byte piece
// u ^ (r & 7) of the row: eight neighbouring rows then cover all 32 banks
// (the same piece of every row would put the whole warp on four banks).
// The sum runs over the pieces in that order.
// Four partial sums (element e of each piece into ss[e & 3]) keep the FMA
// chains short.
__device__ __forceinline__ void row_sq(const unsigned char* tile, int r, float (&ss)[4]) {
  const uint4* row = reinterpret_cast<const uint4*>(tile + r * 128);
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    float f[8];
    unpack16<PKM_BF16>(row[u ^ (r & 7)], f);
#pragma unroll
    for (int e = 0; e < 8; ++e) ss[e & 3] = fmaf(f[e], f[e], ss[e & 3]);
  }
}
__device__ __forceinline__ float sum4(const float (&ss)[4]) {
  return (ss[0] + ss[1]) + (ss[2] + ss[3]);
}

__global__ void __launch_bounds__(ssm::kThreads, 1) select_small_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int T,
    int H, int dh, int n, int k, int32_t* __restrict__ idx, float* __restrict__ wout,
    uint64_t* __restrict__ chunk_lists, uint64_t* __restrict__ half_lists,
    int32_t* __restrict__ counts, int32_t* status) {
  using namespace ssm;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* stages = smem_raw;
  float* rks = reinterpret_cast<float*>(smem_raw + kRksOff);
  float* rqs = reinterpret_cast<float*>(smem_raw + kRqsOff);  // sqrt(d_half) / ||q_t||
  uint16_t* cells = reinterpret_cast<uint16_t*>(smem_raw + kCellsOff);
  SmallCtl* ctl = reinterpret_cast<SmallCtl*>(smem_raw + kCtlOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x;
  const int chunks = gridDim.x;
  const int hc = blockIdx.y;  // 2h + half
  const int h = hc >> 1;
  const int c0 = chunk * kN;
  const int ncols = min(kN, n - c0);
  const int KB = dh / kKB;
  const bool misaligned = (smem_u32(smem_raw) & 1023u) != 0;
  // the next kernel (a Memory+ gate GEMM that does not read the selection)
  // may start on the SMs this grid leaves free
  pdl_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
      mbar_init(&ctl->nread[s], kNormThreads / 32);
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
    // ------------------------------------------------------ TMA producer
    if (lane == 0 && run) {
      uint32_t issued_mask = 0, issued_par = 0;
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        const int stage = kb % kStages;
        const uint32_t phase = (uint32_t)(kb / kStages) & 1;
        if (!wait_small(&ctl->empty[stage], phase ^ 1, ctl, status)) { ok = false; break; }
        // the norm warps must be done with k-block kb - kStages of this stage
        if (kb >= kStages &&
            !wait_small(&ctl->nread[stage], (uint32_t)((kb - kStages) / kStages) & 1, ctl,
                        status)) {
          ok = false;
          break;
        }
        unsigned char* sa = stages + stage * kStageBytes;
        mbar_arrive_expect_tx(&ctl->full[stage], kStageBytes);
        tma_load_3d(sa, &tmA, &ctl->full[stage], kb * kKB, hc, 0);
        tma_load_3d(sa + kABytes, &tmB, &ctl->full[stage], kb * kKB, c0, hc);
        issued_mask |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
      }
      if (!ok) {  // let every copy in flight land before the CTA moves on
        for (int s = 0; s < kStages; ++s)
          if (issued_mask & (1u << s))
            for (unsigned long long i = 0; i < kSpinLimit; ++i)
              if (mbar_try_wait(&ctl->full[s], (issued_par >> s) & 1)) break;
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
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
      // every MMA issued must complete before TMEM is released
      tc_commit(&ctl->drain);
      for (unsigned long long i = 0; i < kSpinLimit; ++i)
        if (mbar_try_wait(&ctl->drain, 0)) break;
    }
  } else if (warp >= 6) {
    // ------------------------------------- the k x k cells (for the combine)
    if (run)
      for (int e = threadIdx.x - 192; e < kCellSlots; e += 64) cells[e] = topk_cell(e, k);
  } else if (run) {
    // ------------------------------------------------ norms, then scores
    const int tid = threadIdx.x - 64;  // 0..127
    const int ta = (tid + 96) & 127;   // token row of this thread (warp 5 first: warp 4 has the TMEM pass)
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb0[4] = {0.f, 0.f, 0.f, 0.f}, sb1[4] = {0.f, 0.f, 0.f, 0.f};
    bool ok = true;
    for (int kb = 0; kb < KB; ++kb) {
      const int stage = kb % kStages;
      const bool got = wait_small(&ctl->full[stage], (uint32_t)(kb / kStages) & 1, ctl, status);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      const unsigned char* st = stages + stage * kStageBytes;
      row_sq(st + kABytes, tid, sb0);
      row_sq(st + kABytes, tid + kNormThreads, sb1);
      if (ta < T) row_sq(st, ta, sa);
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->nread[stage]);
    }
    // every norm warp reaches the barrier, also after an abort
    if (ok) {
      rks[tid] = 1.0f / fmaxf(sqrtf(sum4(sb0)), kNormEps);
      rks[tid + kNormThreads] = 1.0f / fmaxf(sqrtf(sum4(sb1)), kNormEps);
      if (ta < T) rqs[ta] = sqrtf((float)dh) / fmaxf(sqrtf(sum4(sa)), kNormEps);
    }
    norm_barrier();
    if (warp == 4 && ok) {
      // TMEM lanes 0..31: the tokens' raw products into the stage ring (the
      // scaling is applied when the warps read them back)
      const bool got = wait_small(&ctl->accf, 0, ctl, status);
      if (__all_sync(0xffffffffu, got)) {
        tc_fence_after();
        float* sc = reinterpret_cast<float*>(stages);  // [32][kScoreStride]
        // 32 columns per TMEM load, the next load in flight while this one is stored
        uint32_t r[2][32];
        tmem_ld_32x32b_x32(tmem, r[0]);
#pragma unroll
        for (int g = 0; g < kN / 32; ++g) {
          tmem_wait_x32(r[g & 1]);
          if (g + 1 < kN / 32) tmem_ld_32x32b_x32(tmem + (g + 1) * 32, r[(g + 1) & 1]);
          if (lane < T) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<uint4*>(sc + lane * kScoreStride + g * 32 + q * 4) =
                  make_uint4(r[g & 1][q * 4], r[g & 1][q * 4 + 1], r[g & 1][q * 4 + 2],
                             r[g & 1][q * 4 + 3]);
          }
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
  if (!run || ctl->abort) return;  // uniform: the whole CTA leaves, uncounted

  // ---------------------------------------- the chunk's top 32 per token
  // s = acc * rk[a] * (sqrt(d_half) * rq[t]); columns past n are -inf
  const float* sc = reinterpret_cast<const float*>(stages);
  for (int t = warp; t < T; t += kWarps) {
    const float rowf = rqs[t];
    float v[8];
    uint32_t id[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const int col = 32 * s + lane;
      v[s] = col < ncols ? sc[t * kScoreStride + col] * rks[col] * rowf : -INFINITY;
      id[s] = col < ncols ? (uint32_t)(c0 + col) : 0xffffffffu;
      warp_sort32_desc(v[s], id[s]);
    }
#pragma unroll
    for (int w = 1; w < 8; w <<= 1)
#pragma unroll
      for (int s = 0; s < 8; s += 2 * w) warp_merge32_desc(v[s], id[s], v[s + w], id[s + w]);
    chunk_lists[(((int64_t)hc * chunks + chunk) * T + t) * kList + lane] = pack_entry(v[0], id[0]);
  }
  __threadfence();  // this CTA's lists are visible device-wide before its count
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(counts + hc, 1);
    ctl->merge = prev == chunks - 1;
    if (ctl->merge) __threadfence();  // the other chunks' lists after the count
  }
  __syncthreads();
  if (!ctl->merge) return;

  // ------------------------- the last CTA of (head, half): merge the chunks
  for (int t = warp; t < T; t += kWarps) {
    const uint64_t* src = chunk_lists + ((int64_t)hc * chunks * T + t) * kList + lane;
    // all chunks' entries in flight at once, then a tree of merges
    uint64_t e[kMaxChunks];
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c)
      e[c] = c < chunks ? ld_cg_u64(src + (int64_t)c * T * kList) : pack_entry(-INFINITY, ~0u);
    float v[kMaxChunks];
    uint32_t id[kMaxChunks];
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      v[c] = entry_score(e[c]);
      id[c] = entry_id(e[c]);
    }
#pragma unroll
    for (int w = 1; w < kMaxChunks; w <<= 1)
#pragma unroll
      for (int c = 0; c < kMaxChunks; c += 2 * w)
        if (c + w < chunks) warp_merge32_desc(v[c], id[c], v[c + w], id[c + w]);
    half_lists[((int64_t)hc * T + t) * kList + lane] = pack_entry(v[0], id[0]);
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(counts + gridDim.y + h, 1);
    ctl->combine = prev == 1;
    if (ctl->combine) __threadfence();  // the other half's lists after the count
  }
  __syncthreads();
  if (!ctl->combine) return;

  // ------------------ the second half of the head to arrive: k x k combine
  for (int t = warp; t < T; t += kWarps) {
    const bool in = lane < k;
    const uint64_t e1 = ld_cg_u64(half_lists + ((int64_t)(2 * h) * T + t) * kList + lane);
    const uint64_t e2 = ld_cg_u64(half_lists + ((int64_t)(2 * h + 1) * T + t) * kList + lane);
    const int64_t o = ((int64_t)t * H + h) * k;
    const float v1 = in ? entry_score(e1) : -INFINITY, v2 = in ? entry_score(e2) : -INFINITY;
    if (k == 32)  // the grid's first row is already in order
      combine_lists_warp<true>(v1, entry_id(e1), v2, entry_id(e2), cells, n, k, idx + o, wout + o);
    else
      combine_lists_warp<false>(v1, entry_id(e1), v2, entry_id(e2), cells, n, k, idx + o, wout + o);
  }
}

}  // namespace

bool select_small_supported(pkm_dtype dt, int64_t T, int dh, int n, int k) {
  const int chunks = (n + ssm::kN - 1) / ssm::kN;
  return dt == PKM_BF16 && T >= 1 && T <= ssm::kMaxRows && dh % ssm::kKB == 0 && dh <= 2048 &&
         n >= ssm::kN && n % 4 == 0 && k <= ssm::kList && chunks <= ssm::kMaxChunks;
}

size_t select_small_workspace(int64_t T, int H, int n) {
  const size_t chunks = (size_t)((n + ssm::kN - 1) / ssm::kN);
  const size_t lists = (size_t)H * 2 * (chunks + 1) * (size_t)T * ssm::kList * sizeof(uint64_t);
  return lists + ((size_t)H * 3 * sizeof(int32_t) + 255) / 256 * 256;
}

cudaError_t launch_select_small(const void* q, const void* K, int64_t T, int H, int dh, int n,
                                int k, int32_t* idx, float* w, void* workspace, int32_t* status,
                                cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const int chunks = (n + ssm::kN - 1) / ssm::kN;
  uint64_t* chunk_lists = static_cast<uint64_t*>(workspace);
  uint64_t* half_lists = chunk_lists + (size_t)H * 2 * chunks * T * ssm::kList;
  int32_t* counts = reinterpret_cast<int32_t*>(half_lists + (size_t)H * 2 * T * ssm::kList);
  cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * H * 3, stream);
  if (e != cudaSuccess) return e;
  CUtensorMap tmA, tmB;
  {
    const uint64_t dims[3] = {(uint64_t)dh, (uint64_t)H * 2, (uint64_t)T};
    const uint64_t strides[2] = {(uint64_t)dh * 2, (uint64_t)H * 2 * dh * 2};
    const uint32_t box[3] = {(uint32_t)ssm::kKB, 1, (uint32_t)ssm::kM};
    if (!make_tmap_bf16(&tmA, q, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {(uint64_t)dh, (uint64_t)n, (uint64_t)H * 2};
    const uint64_t strides[2] = {(uint64_t)dh * 2, (uint64_t)n * dh * 2};
    const uint32_t box[3] = {(uint32_t)ssm::kKB, (uint32_t)ssm::kN, 1};
    if (!make_tmap_bf16(&tmB, K, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  e = cudaFuncSetAttribute(select_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)ssm::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)chunks, (unsigned)(H * 2), 1);
  select_small_kernel<<<grid, ssm::kThreads, ssm::kSmemBytes, stream>>>(
      tmA, tmB, (int)T, H, dh, n, k, idx, w, chunk_lists, half_lists, counts, status);
  note_launch();
  return cudaGetLastError();
}

}  // namespace pkm
