// k_gemm_tc2.cu -- the dense GEMMs of the Memory+ block on pairs of SMs
// ("Memory Layers at Scale" digest, "Memory+ 블록": out = (y ⊙ silu(x W1)) W2,
// and the weight and input gradients of the same products).
//
//   C[M, N] = epi(A[M, K] * B[N, K]^T), bf16 operands, fp32 accumulation,
//   the same operand layouts, epilogues and split-K slices as
//   k_gemm_tc.cu's single-SM kernel.
//
// Why pairs: with 128 x 256 tiles on one SM the tensor cores wait for their
// operands -- every k-block brings 48 KiB from L2 for 128 x 256 x 64 MMAs,
// and the L2-to-SM stream, not the MMA, sets the pace.  Here two CTAs of a
// cluster share one 256 x 256 tile through tcgen05.mma.cta_group::2: each
// loads its own 128 rows of A and its own half (128 columns) of B, and one
// MMA instruction reads both CTAs' shared memory.  Per SM the operand stream
// drops to 32 KiB per k-block for the same MMA work.
//
// Per CTA pair (cluster of 2; rank 0 leads):
//   warp 0     TMA producer of this CTA's halves into a 6-stage ring; the
//              copies report their bytes to the leader's stage barrier,
//              where the leader's producer registers both CTAs' bytes.
//   warp 1     TMEM (both CTAs allocate the same 512 columns together); in
//              the leader, the MMA issuer: M = 256, N = 256 into one of two
//              256-column accumulators; its commits arrive on the stage and
//              accumulator barriers of both CTAs.
//   warps 2-5  epilogue of this CTA's 128 rows; they report a drained
//              accumulator to the leader's barrier (8 warps in all).
// Persistent: each pair walks the 256 x 256 tiles (N fastest, then split-K
// slices).  No load uses cluster multicast: each CTA loads only its own data.
// Spin-waits are bounded; on a timeout the CTA records PKM_ERR_TIMEOUT and
// stops issuing work; the pair meets at a cluster barrier before TMEM is
// freed and the CTAs exit, after the leader has waited (bounded) for every
// copy it was told about.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tmap.h"

namespace pkm {

namespace g2 {
constexpr int kM = 128;            // rows per CTA (the pair covers 256)
constexpr int kN = 256;            // columns per tile (each CTA loads 128)
constexpr int kNh = kN / 2;
constexpr int kKB = 64, kStages = 6, kAcc = 2;
constexpr int kABytes = kM * kKB * 2, kBBytes = kNh * kKB * 2;
constexpr int kStageBytes = kABytes + kBBytes;  // 32 KiB per CTA
constexpr int kThreads = 192;
constexpr int kBox = 64;
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + 256;
}  // namespace g2

namespace {

struct Gemm2Ctl {
  uint64_t full[g2::kStages];   // leader: both CTAs' copies of a stage landed
  uint64_t empty[g2::kStages];  // each CTA: the MMAs are done with a stage
  uint64_t accf[g2::kAcc];      // each CTA: an accumulator is ready
  uint64_t acce[g2::kAcc];      // leader: both epilogues drained an accumulator
  uint64_t drain;
  uint32_t tmem;
  volatile int abort;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
// shared::cluster address of `p` (this CTA's shared memory) in CTA `rank`
__device__ __forceinline__ uint32_t map_to(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void remote_arrive(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];"
               ::"r"(cluster_addr) : "memory");
}
// 2-D tile copy into this CTA's shared memory whose completion is counted on
// a barrier of either CTA of the pair (cluster address)
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const void* tmap,
                                                 uint32_t bar_cluster, int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(smem_dst)), "l"(tmap), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(smem_dst)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;"
               ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_mma_f16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive on the barrier at this shared-memory offset in both CTAs of the
// pair once this thread's MMAs so far have completed
__device__ __forceinline__ void tc_commit_pair_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;"
      ::"r"(smem_u32(bar)), "h"((uint16_t)3) : "memory");
}
// ... and on this CTA's barrier only
__device__ __forceinline__ void tc_commit_pair_local(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool gemm2_wait(uint64_t* bar, uint32_t parity, Gemm2Ctl* ctl,
                                           int32_t* status) {
  return mbar_wait_or_abort(bar, parity, &ctl->abort, status);
}

// Shared-memory descriptor of an MN-major operand tile with the 128-byte
// swizzle (as in k_gemm_tc.cu): consecutive 64-element groups along M/N one
// box (8 KiB) apart, 8 k-lines 1024 B apart.
__device__ __forceinline__ uint64_t smem_desc_mn128_g2(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((g2::kBox * 128) >> 4) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

struct Tile2 {
  int64_t m0;  // first row of the pair's tile
  int n0, z;
};

__device__ __forceinline__ Tile2 tile2_of(int t, int tiles_m, int tiles_n) {
  const int nt = t % tiles_n;
  const int r = t / tiles_n;
  return Tile2{(int64_t)(r % tiles_m) * (2 * g2::kM), nt * g2::kN, r / tiles_m};
}

// OUT: 0 bf16 store, 1 fp32 store, 2 fp32 accumulate (C += result).
template <int EPI, int OUT, bool AMN, bool BMN>
__global__ void __launch_bounds__(g2::kThreads, 1) gemm_tc2_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int64_t M,
    int N, int K, void* __restrict__ Cv, int kb_per_split, int nz, int64_t c_split,
    int32_t* status, int pdl_mode) {
  using namespace g2;
  // programmatic dependent launch: 1 -- an operand is the previous kernel's
  // output, wait for it first; 2 -- none is, wait only before finishing
  pdl_launch_dependents();
  if (pdl_mode == 1) pdl_wait();
  extern __shared__ unsigned char smem_raw[];
  unsigned char* stages = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Gemm2Ctl* ctl = reinterpret_cast<Gemm2Ctl*>(stages + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, pairs = gridDim.x >> 1;
  const int tiles_m = (int)((M + 2 * kM - 1) / (2 * kM));
  const int tiles_n = (N + kN - 1) / kN;
  const int n_tiles = tiles_m * tiles_n * nz;
  const int KB_all = (K + kKB - 1) / kKB;
  auto kb_range = [&](int z, int& kb0, int& nkb) {
    kb0 = kb_per_split > 0 ? z * kb_per_split : 0;
    nkb = kb_per_split > 0 ? min(kb_per_split, KB_all - kb0) : KB_all;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->full[s], 1);   // the leader's producer registers both CTAs' bytes
      mbar_init(&ctl->empty[s], 1);  // the leader's commit
    }
    for (int b = 0; b < kAcc; ++b) {
      mbar_init(&ctl->accf[b], 1);
      mbar_init(&ctl->acce[b], 8);   // four epilogue warps in each CTA
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
    tmem_alloc_pair(&ctl->tmem, kAcc * kN);
    tmem_relinquish_pair();
  }
  __syncwarp();  // the cluster barrier is warp-aligned: reconverge first
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers and TMEM exist before any remote use
  tc_fence_after();
  const uint32_t tmem = ctl->tmem;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t issued_mask = 0, issued_par = 0;
      bool ok = true;
      int f = 0;  // stage fills so far
      for (int t = pair; t < n_tiles && ok; t += pairs) {
        const Tile2 tc = tile2_of(t, tiles_m, tiles_n);
        const int64_t am = tc.m0 + (int64_t)rank * kM;  // this CTA's rows
        const int bn = tc.n0 + (int)rank * kNh;         // this CTA's half of the columns
        int kb0, nkb;
        kb_range(tc.z, kb0, nkb);
        for (int kb = 0; kb < nkb; ++kb, ++f) {
          const int stage = f % kStages;
          const uint32_t phase = (uint32_t)(f / kStages) & 1;
          if (!gemm2_wait(&ctl->empty[stage], phase ^ 1, ctl, status)) { ok = false; break; }
          unsigned char* sa = stages + stage * kStageBytes;
          unsigned char* sb = sa + kABytes;
          const int kc = (kb0 + kb) * kKB;
          const uint32_t bar = map_to(&ctl->full[stage], 0);
          // the leader registers the bytes of both CTAs' copies (a local
          // arrive: a remote one per stage measured slower, each is a
          // cluster-scope release); a copy of the partner's that lands first
          // only takes the count below zero until then
          if (leader) mbar_arrive_expect_tx(&ctl->full[stage], 2 * kStageBytes);
          if (AMN) {
#pragma unroll
            for (int j = 0; j < kM / kBox; ++j)
              tma_load_2d_pair(sa + j * kBox * 128, &tmA, bar, (int32_t)am + j * kBox, kc);
          } else {
            tma_load_2d_pair(sa, &tmA, bar, kc, (int32_t)am);
          }
          if (BMN) {
#pragma unroll
            for (int j = 0; j < kNh / kBox; ++j)
              tma_load_2d_pair(sb + j * kBox * 128, &tmB, bar, bn + j * kBox, kc);
          } else {
            tma_load_2d_pair(sb, &tmB, bar, kc, bn);
          }
          issued_mask |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        }
      }
      // on an abort the leader lets every copy it was told about land (the
      // partner's copies count on the leader's barriers)
      if (!ok && leader) {
        for (int s = 0; s < kStages; ++s)
          if (issued_mask & (1u << s))
            for (unsigned long long i = 0; i < kSpinLimit; ++i)
              if (mbar_try_wait(&ctl->full[s], (issued_par >> s) & 1)) break;
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------- MMA issuer (leader)
    if (lane == 0 && leader) {
      const uint32_t idesc = idesc_bf16_f32(2 * kM, kN) | (AMN ? (1u << 15) : 0u) |
                             (BMN ? (1u << 16) : 0u);
      bool ok = true;
      int f = 0, li = 0;
      for (int t = pair; t < n_tiles && ok; t += pairs, ++li) {
        const Tile2 tc = tile2_of(t, tiles_m, tiles_n);
        int kb0, nkb;
        kb_range(tc.z, kb0, nkb);
        const int buf = li & 1;
        // both epilogues have drained this accumulator's previous tile
        if (!gemm2_wait(&ctl->acce[buf], ((li >> 1) & 1) ^ 1, ctl, status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dt = tmem + (uint32_t)(buf * kN);
        for (int kb = 0; kb < nkb; ++kb, ++f) {
          const int stage = f % kStages;
          const uint32_t phase = (uint32_t)(f / kStages) & 1;
          if (!gemm2_wait(&ctl->full[stage], phase, ctl, status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(stages + stage * kStageBytes);
          const uint32_t sb = sa + kABytes;
#pragma unroll
          for (int kk = 0; kk < kKB / 16; ++kk) {
            const uint64_t ad = AMN ? smem_desc_mn128_g2(sa + kk * 2048) : smem_desc_k128(sa + kk * 32);
            const uint64_t bd = BMN ? smem_desc_mn128_g2(sb + kk * 2048) : smem_desc_k128(sb + kk * 32);
            tc_mma_f16_pair(dt, ad, bd, idesc, (kb | kk) != 0);
          }
          tc_commit_pair_both(&ctl->empty[stage]);  // both CTAs may refill the stage
        }
        if (ok) tc_commit_pair_both(&ctl->accf[buf]);
      }
      // every MMA issued must complete before either CTA frees TMEM or exits
      tc_commit_pair_local(&ctl->drain);
      for (unsigned long long i = 0; i < kSpinLimit; ++i)
        if (mbar_try_wait(&ctl->drain, 0)) break;
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    int li = 0;
    for (int t = pair; t < n_tiles; t += pairs, ++li) {
      const Tile2 tc = tile2_of(t, tiles_m, tiles_n);
      const int buf = li & 1;
      const bool got = gemm2_wait(&ctl->accf[buf], (li >> 1) & 1, ctl, status);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int64_t m = tc.m0 + (int64_t)rank * kM + row;
      void* Cz = static_cast<char*>(Cv) + (int64_t)tc.z * c_split * (OUT != 0 ? 4 : 2);
      for (int g = 0; g < kN / 32; ++g) {
        const int col0 = tc.n0 + g * 32;
        if (col0 >= N) break;
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) + buf * kN + g * 32, r);
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
              // ulp in fp32, far below the bf16 rounding that follows)
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
      if (lane == 0) remote_arrive(map_to(&ctl->acce[buf], 0));
    }
  }

  // both CTAs finished: the leader's MMAs no longer read either CTA's shared
  // memory or write either CTA's TMEM
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, kAcc * kN);
  if (pdl_mode == 2) pdl_wait();
}

}  // namespace

// CTA pairs that can be resident at once (0 if none or the query fails)
static int pair_slots(const void* kern) {
  static int cached[16] = {0};
  static const void* keys[16] = {nullptr};
  for (int i = 0; i < 16; ++i)
    if (keys[i] == kern) return cached[i];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(g2::kThreads, 1, 1);
  cfg.dynamicSmemBytes = g2::kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  for (int i = 0; i < 16; ++i)
    if (!keys[i]) {
      keys[i] = kern;
      cached[i] = n;
      break;
    }
  return n;
}

bool gemm_tc2_useful(int64_t M) { return M > g2::kM; }

// Same contract as launch_gemm_tc; returns cudaErrorNotSupported (nothing
// launched) when no CTA pair can be resident.
cudaError_t launch_gemm_tc2(const void* A, const void* B, int64_t M, int N, int K, int epi,
                            int out_mode, void* C, int32_t* status, cudaStream_t stream,
                            int splits, int64_t c_split, bool a_mn, bool b_mn, int pdl_mode) {
  if (M <= 0) return cudaSuccess;
  CUtensorMap tmA, tmB;
  if (a_mn) {
    if (M % 8) return cudaErrorInvalidValue;
    const uint64_t dims[2] = {(uint64_t)M, (uint64_t)K};
    const uint64_t strides[1] = {(uint64_t)M * 2};
    const uint32_t box[2] = {(uint32_t)g2::kBox, (uint32_t)g2::kKB};
    if (!make_tmap_bf16(&tmA, A, 2, dims, strides, box)) return cudaErrorInvalidValue;
  } else {
    const uint64_t dims[2] = {(uint64_t)K, (uint64_t)M};
    const uint64_t strides[1] = {(uint64_t)K * 2};
    const uint32_t box[2] = {(uint32_t)g2::kKB, (uint32_t)g2::kM};
    if (!make_tmap_bf16(&tmA, A, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  if (b_mn) {
    const uint64_t dims[2] = {(uint64_t)N, (uint64_t)K};
    const uint64_t strides[1] = {(uint64_t)N * 2};
    const uint32_t box[2] = {(uint32_t)g2::kBox, (uint32_t)g2::kKB};
    if (!make_tmap_bf16(&tmB, B, 2, dims, strides, box)) return cudaErrorInvalidValue;
  } else {
    const uint64_t dims[2] = {(uint64_t)K, (uint64_t)N};
    const uint64_t strides[1] = {(uint64_t)K * 2};
    const uint32_t box[2] = {(uint32_t)g2::kKB, (uint32_t)g2::kNh};
    if (!make_tmap_bf16(&tmB, B, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  const int KB = (K + g2::kKB - 1) / g2::kKB;
  int kbps = 0, nz = 1;
  if (splits > 1) {  // every slice gets at least one k-block
    kbps = (KB + splits - 1) / splits;
    nz = (KB + kbps - 1) / kbps;
  }
  const int64_t tiles = (M + 2 * g2::kM - 1) / (2 * g2::kM) * ((N + g2::kN - 1) / g2::kN) * nz;
  cudaError_t e = cudaSuccess;
  auto go = [&](auto kern) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)g2::kSmemBytes);
    if (e != cudaSuccess) return;
    const int slots = pair_slots(reinterpret_cast<const void*>(kern));
    if (slots < 1) {
      e = cudaErrorNotSupported;
      return;
    }
    const int64_t pairs = tiles < slots ? tiles : slots;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
    cfg.blockDim = dim3(g2::kThreads, 1, 1);
    cfg.dynamicSmemBytes = g2::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_mode != 0 ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, kern, tmA, tmB, M, N, K, C, kbps, nz, c_split, status,
                           pdl_mode);
  };
#define PKM_GEMM2_LAYOUTS(E_, O_)                                   \
  if (a_mn && b_mn) go(gemm_tc2_kernel<E_, O_, true, true>);        \
  else if (a_mn) go(gemm_tc2_kernel<E_, O_, true, false>);          \
  else if (b_mn) go(gemm_tc2_kernel<E_, O_, false, true>);          \
  else go(gemm_tc2_kernel<E_, O_, false, false>)
  if (out_mode == 1) {
    PKM_GEMM2_LAYOUTS(0, 1);
  } else if (out_mode == 2) {
    PKM_GEMM2_LAYOUTS(0, 2);
  } else if (epi == 1) {
    PKM_GEMM2_LAYOUTS(1, 0);
  } else {
    PKM_GEMM2_LAYOUTS(0, 0);
  }
#undef PKM_GEMM2_LAYOUTS
  if (e != cudaSuccess) return e;
  note_launch();
  return cudaGetLastError();
}

}  // namespace pkm
