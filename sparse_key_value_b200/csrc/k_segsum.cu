// k_segsum.cu -- deterministic segmented sums over sorted (key, entry)
// pairs: out[key] = sum over entries e with that key, in sorted (= stable,
// input) order, of coef[e] * src[row(e)], row(e) = e / div.
//
// This is the sort-by-index scatter-add of the training step: value-row
// gradients (key = value row, src = dy) and sub-key gradients (key =
// (head, half, sub-key), src = the query half).  No atomics: the sorted
// entries are cut into fixed chunks of kChunk; one CTA walks a chunk in order
// and finishes every segment that starts and ends inside it; the pieces of a
// segment that crosses chunk boundaries go to per-chunk carry rows and a
// fix-up kernel adds them in chunk order.  The work per CTA is fixed, so a
// hot key with many entries (Zipf popularity) spreads over many CTAs.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace pkm {

namespace {
constexpr int kChunk = 256;
constexpr int kThreads = 256;
constexpr int kUnroll = 8;
}  // namespace

size_t segsum_workspace(int64_t n, int d) {
  const int64_t chunks = (n + kChunk - 1) / kChunk;
  size_t b = 0;
  b += (size_t)(chunks + 64) * 4;          // chunk head counts -> segment base
  b += (size_t)chunks * 4 * 2 + 256;       // first-ends flag, last segment id
  b += (size_t)chunks * d * 4 * 2 + 512;   // carry rows
  return b + 1024;
}

namespace {

struct SegWs {
  uint32_t* seg_base;   // [chunks + 1]
  uint32_t* first_end;  // [chunks]
  uint32_t* last_seg;   // [chunks]: segment id of the carried last part, or ~0
  float* carry_first;   // [chunks, d]
  float* carry_last;    // [chunks, d]
};

SegWs carve(void* ws, int64_t n, int d) {
  const int64_t chunks = (n + kChunk - 1) / kChunk;
  char* p = static_cast<char*>(ws);
  SegWs w;
  auto take = [&](size_t bytes) {
    char* r = p;
    p += (bytes + 255) / 256 * 256;
    return r;
  };
  w.seg_base = reinterpret_cast<uint32_t*>(take((size_t)(chunks + 64) * 4));
  w.first_end = reinterpret_cast<uint32_t*>(take((size_t)chunks * 4));
  w.last_seg = reinterpret_cast<uint32_t*>(take((size_t)chunks * 4));
  w.carry_first = reinterpret_cast<float*>(take((size_t)chunks * d * 4));
  w.carry_last = reinterpret_cast<float*>(take((size_t)chunks * d * 4));
  return w;
}

__device__ __forceinline__ bool is_head(const uint32_t* skey, int64_t i, uint32_t mark) {
  const uint32_t k = skey[i];
  return k != mark && (i == 0 || skey[i - 1] != k);
}

// heads per chunk (one warp per chunk)
__global__ void chunk_heads_kernel(const uint32_t* __restrict__ skey, int64_t n, uint32_t mark,
                                   uint32_t* __restrict__ heads) {
  const int64_t c = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  const int64_t chunks = (n + kChunk - 1) / kChunk;
  if (c >= chunks) return;
  uint32_t cnt = 0;
  for (int j = lane; j < kChunk; j += 32) {
    const int64_t i = c * kChunk + j;
    if (i < n && is_head(skey, i, mark)) ++cnt;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) heads[c] = cnt;
}

struct SegOutDev {
  int32_t* uniq_rows;
  float* grad_rows;
  int64_t cap;
  float* dense_add;
  float* dense_set;
};

template <int V>
__device__ __forceinline__ void emit_final(const SegOutDev& o, uint32_t seg, uint32_t key, int d,
                                           int ch, const float* acc, int32_t* status) {
  const int64_t col = (int64_t)ch * V;
  if (o.grad_rows) {
    if ((int64_t)seg < o.cap) {
      if (ch == 0 && o.uniq_rows) o.uniq_rows[seg] = (int32_t)key;
      // streaming stores: the gradient rows are written once and must not
      // push the source rows out of L2
      float* g = o.grad_rows + (int64_t)seg * d + col;
#pragma unroll
      for (int e = 0; e < V; e += 4)
        __stcs(reinterpret_cast<float4*>(g + e), make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]));
    } else if (ch == 0) {
      set_status(status, PKM_ERR_DEVICE);
    }
  }
  if (o.dense_add) {
    float* g = o.dense_add + (int64_t)key * d + col;
#pragma unroll
    for (int e = 0; e < V; e += 4) {
      float4 v = *reinterpret_cast<float4*>(g + e);
      v.x += acc[e];
      v.y += acc[e + 1];
      v.z += acc[e + 2];
      v.w += acc[e + 3];
      *reinterpret_cast<float4*>(g + e) = v;
    }
  }
  if (o.dense_set) {
    float* g = o.dense_set + (int64_t)key * d + col;
#pragma unroll
    for (int e = 0; e < V; e += 4)
      __stcs(reinterpret_cast<float4*>(g + e), make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]));
  }
}

template <int V>
__device__ __forceinline__ void store_row(float* dst, const float* acc) {
#pragma unroll
  for (int e = 0; e < V; e += 4)
    *reinterpret_cast<float4*>(dst + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
}

// One CTA per chunk; each thread owns NV consecutive 16-byte column vectors
// (W elements) of the rows and walks the chunk's entries in order.
template <pkm_dtype DT, int NV>
__global__ void __launch_bounds__(kThreads) segsum_chunk_kernel(
    const uint32_t* __restrict__ skey, const uint32_t* __restrict__ sval, int64_t n,
    uint32_t mark, const float* __restrict__ coef, const typename Elem<DT>::T* __restrict__ src,
    int64_t div, int d, SegWs ws, SegOutDev out, int32_t* status) {
  constexpr int V = Elem<DT>::kVec;
  constexpr int W = V * NV;
  __shared__ uint32_t keys[kChunk + 1];
  __shared__ uint32_t rows[kChunk];  // source row of each entry, entry / div
  __shared__ float cf[kChunk];
  const int64_t c = blockIdx.x;
  const int64_t i0 = c * kChunk;
  const int len = (int)min((int64_t)kChunk, n - i0);
  const uint32_t div32 = (uint32_t)div;
  for (int j = threadIdx.x; j <= len; j += blockDim.x) {
    const int64_t i = i0 + j;
    keys[j] = i < n ? skey[i] : mark;
    if (j < len) {
      const uint32_t e = sval[i];
      rows[j] = e / div32;
      cf[j] = keys[j] != mark ? coef[e] : 0.f;
    }
  }
  const uint32_t prev_key = i0 > 0 ? skey[i0 - 1] : mark;
  __syncthreads();
  const uint32_t base = ws.seg_base[c];
  const int groups = d / W;
  if (threadIdx.x == 0) {
    ws.first_end[c] = 1;
    ws.last_seg[c] = 0xffffffffu;
  }
  // the chunk's first part continues a segment from the previous chunk?
  const bool cont0 = keys[0] != mark && prev_key == keys[0];

  // valid entries come first (the mark sorts last)
  __shared__ int n_valid;
  if (threadIdx.x == 0) n_valid = 0;
  __syncthreads();
  {
    int cnt = 0;
    for (int j = threadIdx.x; j < len; j += blockDim.x) cnt += keys[j] != mark;
    if (cnt) atomicAdd(&n_valid, cnt);
  }
  __syncthreads();
  const int lv = n_valid;
  constexpr int kU = kUnroll / NV;  // source rows in flight per thread
  // the source rows (dy or the queries) are re-read by many chunks: keep
  // them in L2 while the gradient rows stream out
  const uint64_t keep = l2_policy_keep();

  for (int ch = threadIdx.x; ch < groups; ch += blockDim.x) {
    float acc[W];
#pragma unroll
    for (int e = 0; e < W; ++e) acc[e] = 0.f;
    uint32_t heads = 0;
    bool part_starts = !cont0;
    // kU source rows in flight regardless of where segments end; the sums
    // still run entry by entry in sorted order
    for (int j0 = 0; j0 < lv; j0 += kU) {
      uint4 v[kU][NV];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int j = j0 + u;
        if (j < lv) {
          const typename Elem<DT>::T* row = src + (int64_t)rows[j] * d + (int64_t)ch * W;
#pragma unroll
          for (int q = 0; q < NV; ++q) v[u][q] = ldg_nc_16_hint(row + q * V, keep);
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int j = j0 + u;
        if (j >= lv) break;
        float f[W];
#pragma unroll
        for (int q = 0; q < NV; ++q) unpack16<DT>(v[u][q], f + q * V);
        const float2 w2 = make_float2(cf[j], cf[j]);
        // acc += w * f, two lanes per instruction (each rounded as fmaf)
#pragma unroll
        for (int e = 0; e < W; e += 2) {
          const float2 r = __ffma2_rn(w2, make_float2(f[e], f[e + 1]),
                                      make_float2(acc[e], acc[e + 1]));
          acc[e] = r.x;
          acc[e + 1] = r.y;
        }
        const uint32_t key = keys[j];
        if (j + 1 < len && keys[j + 1] == key) continue;  // the part goes on in this chunk
        // the part ending at entry j is complete within the chunk
        const bool seg_ends = keys[j + 1] != key;  // keys[len] is the next chunk's first
        if (part_starts) ++heads;
        const uint32_t seg = base + heads - 1;
        if (part_starts && seg_ends) {
          emit_final<W>(out, seg, key, d, ch, acc, status);
        } else if (!part_starts) {
          store_row<W>(ws.carry_first + c * d + (int64_t)ch * W, acc);
          if (ch == threadIdx.x && threadIdx.x == 0) ws.first_end[c] = seg_ends ? 1u : 0u;
        } else {
          store_row<W>(ws.carry_last + c * d + (int64_t)ch * W, acc);
          if (ch == threadIdx.x && threadIdx.x == 0) ws.last_seg[c] = seg;
        }
#pragma unroll
        for (int e = 0; e < W; ++e) acc[e] = 0.f;
        part_starts = true;
      }
    }
  }
}

// ------------------------------------------------ value rows with dw ----
// The value gradient of the bf16 backward with the softmax's upstream
// gradient in the same walk: for each sorted (value row r, slot e) entry,
// grad[r] += w[e] * dy[t(e)] and dw[e] = <dy[t(e)], V[r]> ("Memory Layers at
// Scale" digest, "병렬 EmbeddingBag 구현": the backward of the weighted bag).
// One warp per chunk of kChunk entries (same chunks, segment ids and carry
// rows as segsum_chunk_kernel), holding whole rows: lane l owns the 16-byte
// column chunks l, l + 32, ...  The rows come through shared memory by bulk
// copies (cp.async.bulk, one per 16-bit row) into per-warp rings: dy rows
// kDwRing entries ahead of the warp, the table row of each segment as soon as
// a ring slot is free (each distinct value row is read once per chunk, not
// once per slot).  The dot products reduce within the warp, in a fixed order.
constexpr int kDwRing = 4;   // dy rows in flight per warp
constexpr int kDwVRing = 4;  // table rows in flight per warp (segments may be one entry long)

__device__ __forceinline__ void bulk_row(void* smem_dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(smem_dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__host__ __device__ inline size_t segsum_dw_warp_smem(int d) {
  return (size_t)(kDwRing + kDwVRing) * d * 2 + (size_t)kChunk * 16 +
         (size_t)(kDwRing + kDwVRing) * 8;
}

// Rows wider than 512 are cut into `slices` column slices, each walked by
// its own warp; slice s writes its partial dot products to dw_out[s][entry]
// (summed in slice order by the softmax backward).
template <int Q>  // 16-byte (8 x bf16) column chunks per lane: d / slices = 256 Q
__global__ void __launch_bounds__(256) segsum_dw_kernel(
    const uint32_t* __restrict__ skey, const uint32_t* __restrict__ sval, int64_t n,
    uint32_t mark, const float* __restrict__ coef, const __nv_bfloat16* __restrict__ src,
    int64_t div, int d, int slices, SegWs ws, SegOutDev out,
    const __nv_bfloat16* __restrict__ table, float* __restrict__ dw_out, int32_t* status) {
  constexpr int E = 8 * Q;
  extern __shared__ __align__(16) unsigned char smem_dw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int64_t gw = (int64_t)blockIdx.x * nwarps + warp;
  const int64_t c = gw / slices;   // chunk
  const int sl = (int)(gw % slices);
  const int ds = d / slices;       // this slice's columns
  const int64_t chunks = (n + kChunk - 1) / kChunk;
  const size_t per_warp = segsum_dw_warp_smem(ds);
  unsigned char* base = smem_dw + (size_t)warp * per_warp;
  __nv_bfloat16* dring = reinterpret_cast<__nv_bfloat16*>(base);
  __nv_bfloat16* vring = dring + (size_t)kDwRing * ds;
  uint32_t* key_s = reinterpret_cast<uint32_t*>(vring + (size_t)kDwVRing * ds);
  uint32_t* row_s = key_s + kChunk;
  uint32_t* e_s = row_s + kChunk;
  float* cf_s = reinterpret_cast<float*>(e_s + kChunk);
  uint64_t* dbar = reinterpret_cast<uint64_t*>(cf_s + kChunk);
  uint64_t* vbar = dbar + kDwRing;
  if (c >= chunks) return;  // whole warp
  const int64_t i0 = c * kChunk;
  const int len = (int)min((int64_t)kChunk, n - i0);
  const uint32_t div32 = (uint32_t)div;
  const uint32_t row_bytes = (uint32_t)ds * 2;
  const int64_t col0 = (int64_t)sl * ds;  // first column of the slice

  if (lane == 0) {
    for (int s2 = 0; s2 < kDwRing; ++s2) mbar_init(&dbar[s2], 1);
    for (int s2 = 0; s2 < kDwVRing; ++s2) mbar_init(&vbar[s2], 1);
    fence_barrier_init();
  }
  int nvalid = 0;
  for (int j = lane; j < kChunk; j += 32) {
    const int64_t i = i0 + j;
    const uint32_t key = j < len ? skey[i] : mark;
    const uint32_t e = j < len ? sval[i] : 0u;
    key_s[j] = key;
    e_s[j] = e;
    row_s[j] = e / div32;
    cf_s[j] = key != mark ? coef[e] : 0.f;
    nvalid += key != mark && j < len;
  }
  const int lv = (int)warp_sum((float)nvalid);  // valid entries come first (the mark sorts last)
  const uint32_t nextk = i0 + len < n ? skey[i0 + len] : mark;
  const uint32_t prev_key = i0 > 0 ? skey[i0 - 1] : mark;
  __syncwarp();
  const uint32_t seg_base = ws.seg_base[c];
  if (lane == 0 && sl == 0) {
    ws.first_end[c] = 1;
    ws.last_seg[c] = 0xffffffffu;
  }
  const bool cont0 = key_s[0] != mark && prev_key == key_s[0];
  volatile int abort_flag = 0;

  // producer state (lane 0 issues): next entry to fetch, table rows fetched
  int pj = 0, ps = 0;
  int cs = 0;  // table rows consumed (segments started) so far
  auto produce = [&](int j) {
    if (lane == 0) {
      fence_proxy_async_smem();  // the warp's reads of the freed slots come first
      while (pj < lv && pj < j + kDwRing) {
        const bool starts = pj == 0 || key_s[pj] != key_s[pj - 1];
        if (starts && ps - cs >= kDwVRing) break;  // its table-row slot is still in use
        const int slot = pj % kDwRing;
        mbar_arrive_expect_tx(&dbar[slot], row_bytes);
        bulk_row(dring + (size_t)slot * ds, src + (int64_t)row_s[pj] * d + col0, row_bytes,
                 &dbar[slot]);
        if (starts) {
          const int vs = ps % kDwVRing;
          mbar_arrive_expect_tx(&vbar[vs], row_bytes);
          bulk_row(vring + (size_t)vs * ds, table + (int64_t)key_s[pj] * d + col0, row_bytes,
                   &vbar[vs]);
          ++ps;
        }
        ++pj;
      }
    }
    __syncwarp();
  };

  float acc[E];
#pragma unroll
  for (int q = 0; q < E; ++q) acc[q] = 0.f;
  uint32_t vr[E / 2];  // the segment's table row, packed bf16 pairs
  uint32_t heads = 0;
  bool part_starts = !cont0;
  int j = 0;
  for (; j < lv; ++j) {
    produce(j);
    const uint32_t key = key_s[j];
    if (j == 0 || key != key_s[j - 1]) {
      const int vs = cs % kDwVRing;
      const bool got = mbar_wait_or_abort(&vbar[vs], (uint32_t)(cs / kDwVRing) & 1,
                                          &abort_flag, status);
      if (!__all_sync(0xffffffffu, got)) break;
      const uint4* vrow = reinterpret_cast<const uint4*>(vring + (size_t)vs * ds);
#pragma unroll
      for (int q = 0; q < Q; ++q) {
        const uint4 t = vrow[lane + 32 * q];
        vr[4 * q] = t.x;
        vr[4 * q + 1] = t.y;
        vr[4 * q + 2] = t.z;
        vr[4 * q + 3] = t.w;
      }
      ++cs;
    }
    const int slot = j % kDwRing;
    const bool got = mbar_wait_or_abort(&dbar[slot], (uint32_t)(j / kDwRing) & 1, &abort_flag,
                                        status);
    if (!__all_sync(0xffffffffu, got)) break;
    const uint4* drow = reinterpret_cast<const uint4*>(dring + (size_t)slot * ds);
    const float cf = cf_s[j];
    const float2 w2 = make_float2(cf, cf);
    float pd[4] = {0.f, 0.f, 0.f, 0.f};  // four partial dot products: short FMA chains
#pragma unroll
    for (int q = 0; q < Q; ++q) {
      const uint4 t = drow[lane + 32 * q];
      float f[8];
      unpack16<PKM_BF16>(t, f);
#pragma unroll
      for (int e2 = 0; e2 < 8; e2 += 2) {
        const float2 r = __ffma2_rn(w2, make_float2(f[e2], f[e2 + 1]),
                                    make_float2(acc[8 * q + e2], acc[8 * q + e2 + 1]));
        acc[8 * q + e2] = r.x;
        acc[8 * q + e2 + 1] = r.y;
        const uint32_t vp = vr[4 * q + e2 / 2];
        pd[e2 >> 1] = fmaf(f[e2], bf16_lo(vp), pd[e2 >> 1]);
        pd[e2 >> 1] = fmaf(f[e2 + 1], bf16_hi(vp), pd[e2 >> 1]);
      }
    }
    const float pdot = warp_sum((pd[0] + pd[1]) + (pd[2] + pd[3]));
    if (lane == 0) dw_out[(int64_t)sl * n + e_s[j]] = pdot;
    // segment bookkeeping, as in segsum_chunk_kernel
    const uint32_t nk = j + 1 < len ? key_s[j + 1] : nextk;
    if (j + 1 < len && nk == key) {
      __syncwarp();  // every lane is done with slot j before it is refilled
      continue;
    }
    const bool seg_ends = nk != key;
    if (part_starts) ++heads;
    const uint32_t seg = seg_base + heads - 1;
#pragma unroll
    for (int q = 0; q < Q; ++q) {
      const int ch = (int)(col0 / 8) + lane + 32 * q;  // 16-byte column chunk of the row
      if (part_starts && seg_ends) {
        emit_final<8>(out, seg, key, d, ch, acc + 8 * q, status);
      } else if (!part_starts) {
        store_row<8>(ws.carry_first + c * d + (int64_t)ch * 8, acc + 8 * q);
      } else {
        store_row<8>(ws.carry_last + c * d + (int64_t)ch * 8, acc + 8 * q);
      }
    }
    if (lane == 0 && sl == 0) {
      if (!part_starts) ws.first_end[c] = seg_ends ? 1u : 0u;
      else if (!seg_ends) ws.last_seg[c] = seg;
    }
#pragma unroll
    for (int q = 0; q < E; ++q) acc[q] = 0.f;
    part_starts = true;
    __syncwarp();
  }
  if (j < lv && lane == 0) {
    // a wait ran out: let every copy issued land before the warp leaves
    for (int jj = j; jj < pj; ++jj)
      for (unsigned long long it = 0; it < kSpinLimit; ++it)
        if (mbar_try_wait(&dbar[jj % kDwRing], (uint32_t)(jj / kDwRing) & 1)) break;
    for (int ss = cs; ss < ps; ++ss)
      for (unsigned long long it = 0; it < kSpinLimit; ++it)
        if (mbar_try_wait(&vbar[ss % kDwVRing], (uint32_t)(ss / kDwVRing) & 1)) break;
  }
  // entries with an invalid row id get dw = 0
  for (int jj = lv + lane; jj < len; jj += 32) dw_out[(int64_t)sl * n + e_s[jj]] = 0.f;
}

// ------------------------------------------- wide rows through a ring ----
// The same segmented sum for bf16 source rows of d % 512 == 0 columns (the
// value gradient: src = dy): one CTA per chunk, the chunk's source rows
// brought into a deep ring of shared-memory slots by bulk copies
// (cp.async.bulk, one per row) that a producer lane issues up to R rows ahead,
// so the L2 sees many whole-row reads in flight per SM instead of a few
// 16-byte loads per thread.  Consumer warp w, lane l owns the 16-byte column
// chunks (w Q + q) 32 + l, q < Q; each warp releases a slot once its lanes
// have read it.  Sums run entry by entry in sorted order (bitwise the same as
// segsum_chunk_kernel).
constexpr int kRingQ = 2;                  // 16-byte column chunks per consumer lane
constexpr size_t kRingBytes = 32u << 10;   // ring slots per CTA: six CTAs per SM
constexpr int kRingMaxSlots = 32;

__device__ __forceinline__ void bulk_row_hint(void* smem_dst, const void* src, uint32_t bytes,
                                              uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;"
      ::"r"(smem_u32(smem_dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

__host__ __device__ inline int segsum_ring_slots(int d) {
  const int r = (int)(kRingBytes / ((size_t)d * 2));
  return r < kRingMaxSlots ? r : kRingMaxSlots;
}
__host__ __device__ inline size_t segsum_ring_smem(int d) {
  return (size_t)segsum_ring_slots(d) * d * 2 + (size_t)(kChunk + 4) * 4 * 3 +
         (size_t)kRingMaxSlots * 16;
}

__global__ void __launch_bounds__(32 * 9) segsum_ring_kernel(
    const uint32_t* __restrict__ skey, const uint32_t* __restrict__ sval, int64_t n,
    uint32_t mark, const float* __restrict__ coef, const __nv_bfloat16* __restrict__ src,
    int64_t div, int d, SegWs ws, SegOutDev out, int32_t* status) {
  constexpr int Q = kRingQ;
  constexpr int E = 8 * Q;
  extern __shared__ __align__(16) unsigned char smem_ring[];
  const int R = segsum_ring_slots(d);
  const int nw = (int)(blockDim.x >> 5) - 1;  // consumer warps; warp nw produces
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __nv_bfloat16* ring = reinterpret_cast<__nv_bfloat16*>(smem_ring);  // [R][d]
  uint32_t* key_s = reinterpret_cast<uint32_t*>(smem_ring + (size_t)R * d * 2);  // [kChunk + 1]
  uint32_t* row_s = key_s + kChunk + 4;
  float* cf_s = reinterpret_cast<float*>(row_s + kChunk + 4);
  uint64_t* full = reinterpret_cast<uint64_t*>(cf_s + kChunk + 4);
  uint64_t* empty = full + kRingMaxSlots;
  __shared__ int n_valid;
  __shared__ volatile int abort_flag;

  const int64_t c = blockIdx.x;
  const int64_t i0 = c * kChunk;
  const int len = (int)min((int64_t)kChunk, n - i0);
  const uint32_t div32 = (uint32_t)div;
  if (threadIdx.x == 0) {
    n_valid = 0;
    abort_flag = 0;
    for (int s = 0; s < R; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], (uint32_t)nw);
    }
    fence_barrier_init();
  }
  for (int j = threadIdx.x; j <= len; j += blockDim.x) {
    const int64_t i = i0 + j;
    key_s[j] = i < n ? skey[i] : mark;
    if (j < len) {
      const uint32_t e = sval[i];
      row_s[j] = e / div32;
      cf_s[j] = key_s[j] != mark ? coef[e] : 0.f;
    }
  }
  const uint32_t prev_key = i0 > 0 ? skey[i0 - 1] : mark;
  __syncthreads();
  {
    int cnt = 0;
    for (int j = threadIdx.x; j < len; j += blockDim.x) cnt += key_s[j] != mark;
    if (cnt) atomicAdd(&n_valid, cnt);
  }
  const uint32_t base = ws.seg_base[c];
  if (threadIdx.x == 0) {
    ws.first_end[c] = 1;
    ws.last_seg[c] = 0xffffffffu;
  }
  __syncthreads();
  const int lv = n_valid;  // valid entries come first (the mark sorts last)
  const uint32_t row_bytes = (uint32_t)d * 2;

  if (warp == nw) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t keep = l2_policy_keep();  // dy rows are re-read by many chunks
      int j = 0;
      for (int slot = 0, round = 0; j < lv; ++j) {
        if (round > 0 &&
            !mbar_wait_or_abort(&empty[slot], (uint32_t)(round - 1) & 1, &abort_flag, status))
          break;
        fence_proxy_async_smem();  // the consumers' reads of the slot come first
        mbar_arrive_expect_tx(&full[slot], row_bytes);
        bulk_row_hint(ring + (size_t)slot * d, src + (int64_t)row_s[j] * d, row_bytes,
                      &full[slot], keep);
        if (++slot == R) { slot = 0; ++round; }
      }
      if (j < lv) {
        // a wait gave up: every copy issued lands before the CTA leaves
        for (int jj = j > R ? j - R : 0; jj < j; ++jj)
          for (unsigned long long it = 0; it < kSpinLimit; ++it)
            if (mbar_try_wait(&full[jj % R], (uint32_t)(jj / R) & 1)) break;
      }
    }
    return;
  }

  // ---------------------------------------------------------------- consumers
  float acc[E];
#pragma unroll
  for (int q = 0; q < E; ++q) acc[q] = 0.f;
  uint32_t heads = 0;
  bool part_starts = !(key_s[0] != mark && prev_key == key_s[0]);
  for (int j = 0, slot = 0, round = 0; j < lv; ++j) {
    const bool got = mbar_wait_or_abort(&full[slot], (uint32_t)round & 1, &abort_flag, status);
    if (!__all_sync(0xffffffffu, got)) break;
    const uint4* rowp = reinterpret_cast<const uint4*>(ring + (size_t)slot * d);
    uint4 v[Q];
#pragma unroll
    for (int q = 0; q < Q; ++q) v[q] = rowp[(warp * Q + q) * 32 + lane];
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
    if (++slot == R) { slot = 0; ++round; }
    const float cf = cf_s[j];
    const float2 w2 = make_float2(cf, cf);
#pragma unroll
    for (int q = 0; q < Q; ++q) {
      float f[8];
      unpack16<PKM_BF16>(v[q], f);
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const float2 r = __ffma2_rn(w2, make_float2(f[e], f[e + 1]),
                                    make_float2(acc[8 * q + e], acc[8 * q + e + 1]));
        acc[8 * q + e] = r.x;
        acc[8 * q + e + 1] = r.y;
      }
    }
    const uint32_t key = key_s[j];
    if (j + 1 < len && key_s[j + 1] == key) continue;  // the part goes on in this chunk
    const bool seg_ends = key_s[j + 1] != key;  // key_s[len] is the next chunk's first
    if (part_starts) ++heads;
    const uint32_t seg = base + heads - 1;
#pragma unroll
    for (int q = 0; q < Q; ++q) {
      const int ch = (warp * Q + q) * 32 + lane;  // 16-byte column chunk of the row
      if (part_starts && seg_ends) {
        emit_final<8>(out, seg, key, d, ch, acc + 8 * q, status);
      } else if (!part_starts) {
        store_row<8>(ws.carry_first + c * d + (int64_t)ch * 8, acc + 8 * q);
      } else {
        store_row<8>(ws.carry_last + c * d + (int64_t)ch * 8, acc + 8 * q);
      }
    }
    if (warp == 0 && lane == 0) {
      if (!part_starts) ws.first_end[c] = seg_ends ? 1u : 0u;
      else if (!seg_ends) ws.last_seg[c] = seg;
    }
#pragma unroll
    for (int q = 0; q < E; ++q) acc[q] = 0.f;
    part_starts = true;
  }
}

// Adds the carried pieces of every segment that crosses chunk boundaries.
template <int V>
__global__ void __launch_bounds__(kThreads) segsum_fixup_kernel(const uint32_t* __restrict__ skey,
                                                                int64_t n, int d, SegWs ws,
                                                                SegOutDev out, int32_t* status) {
  const int64_t c = blockIdx.x;
  const uint32_t seg = ws.last_seg[c];
  if (seg == 0xffffffffu) return;
  const int64_t chunks = (n + kChunk - 1) / kChunk;
  const uint32_t key = skey[min(n, (c + 1) * kChunk) - 1];
  for (int ch = threadIdx.x; ch < d / V; ch += blockDim.x) {
    float acc[V];
    const float* p = ws.carry_last + c * d + (int64_t)ch * V;
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = p[e];
    for (int64_t c2 = c + 1; c2 < chunks; ++c2) {
      const float* q = ws.carry_first + c2 * d + (int64_t)ch * V;
#pragma unroll
      for (int e = 0; e < V; ++e) acc[e] += q[e];
      if (ws.first_end[c2]) break;
    }
    emit_final<V>(out, seg, key, d, ch, acc, status);
  }
}

}  // namespace

cudaError_t launch_scan_exclusive(uint32_t* data, int64_t len, uint32_t* total, int64_t* total64,
                                  cudaStream_t stream);

bool segsum_has_dw(pkm_dtype dt, int d) {
  return dt == PKM_BF16 && d % 256 == 0 && d <= 2048 && (d / segsum_dw_slices(d)) % 256 == 0;
}
// the ring kernel: bf16 rows of 1024..4096 columns in steps of 512, whose
// bulk copies start 16-byte aligned
static bool segsum_ring_ok(pkm_dtype dt, int d, const void* src) {
  return dt == PKM_BF16 && d % (256 * kRingQ) == 0 && d >= 1024 && d <= 4096 &&
         (reinterpret_cast<uintptr_t>(src) & 15u) == 0;
}
// column slices of the dw walk: 512 columns per warp (narrower slices put more
// warps on a chunk: each warp's walk over its entries is a chain of dependent
// steps)
int segsum_dw_slices(int d) { return d > 512 ? d / 512 : 1; }

// Segmented sums of coef[e] * src[e / div] over the sorted pairs; entries
// with key == mark (sorted last) are ignored.  Outputs: sparse rows
// (uniq_rows/grad_rows, capacity cap; n_uniq receives the number of keys),
// dense_add[key] += sum, dense_set[key] = sum (any may be null).
cudaError_t launch_segsum(const uint32_t* skey, const uint32_t* sval, int64_t n, uint32_t mark,
                          const float* coef, const void* src, pkm_dtype dt, int64_t div, int d,
                          int32_t* uniq_rows, float* grad_rows, int64_t cap, int64_t* n_uniq,
                          float* dense_add, float* dense_set, void* workspace, int32_t* status,
                          cudaStream_t stream, const void* table, float* dw) {
  if (n <= 0) {
    if (n_uniq) return cudaMemsetAsync(n_uniq, 0, sizeof(int64_t), stream);
    return cudaSuccess;
  }
  const int64_t chunks = (n + kChunk - 1) / kChunk;
  SegWs ws = carve(workspace, n, d);
  chunk_heads_kernel<<<(unsigned)((chunks + 7) / 8), 256, 0, stream>>>(skey, n, mark,
                                                                       ws.seg_base);
  note_launch();
  cudaError_t e = launch_scan_exclusive(ws.seg_base, chunks, nullptr, n_uniq, stream);
  if (e != cudaSuccess) return e;
  SegOutDev out{uniq_rows, grad_rows, cap, dense_add, dense_set};
  if (table && dw && segsum_has_dw(dt, d)) {
    // value rows with dw: one warp per chunk, rows through bulk-copy rings
    const int slices = segsum_dw_slices(d);
    const int ds = d / slices;
    const size_t per_warp = segsum_dw_warp_smem(ds);
    const int nw = (int)std::min<size_t>(8, (200u << 10) / per_warp);
    const size_t smem = per_warp * nw;
    const unsigned grid = (unsigned)((chunks * slices + nw - 1) / nw);
    auto go = [&](auto kern) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return;
      kern<<<grid, 32 * nw, smem, stream>>>(skey, sval, n, mark, coef,
                                              (const __nv_bfloat16*)src, div, d, slices, ws, out,
                                              (const __nv_bfloat16*)table, dw, status);
    };
    switch (ds / 256) {
      case 1: go(segsum_dw_kernel<1>); break;
      case 2: go(segsum_dw_kernel<2>); break;
      case 3: go(segsum_dw_kernel<3>); break;
      case 4: go(segsum_dw_kernel<4>); break;
      case 5: go(segsum_dw_kernel<5>); break;
      case 6: go(segsum_dw_kernel<6>); break;
      case 7: go(segsum_dw_kernel<7>); break;
      default: go(segsum_dw_kernel<8>); break;
    }
    if (e != cudaSuccess) return e;
    segsum_fixup_kernel<8><<<(unsigned)chunks, min(kThreads, ((d / 8) + 31) / 32 * 32), 0,
                             stream>>>(skey, n, d, ws, out, status);
    note_launch(2);
    return cudaGetLastError();
  }
  if (segsum_ring_ok(dt, d, src)) {
    // wide bf16 rows: the ring kernel, 2 consumer lanes' worth of 16-byte
    // chunks per 512 columns
    const int nw = d / (256 * kRingQ);
    const size_t smem = segsum_ring_smem(d);
    e = cudaFuncSetAttribute(segsum_ring_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    segsum_ring_kernel<<<(unsigned)chunks, 32 * (nw + 1), smem, stream>>>(
        skey, sval, n, mark, coef, (const __nv_bfloat16*)src, div, d, ws, out, status);
    segsum_fixup_kernel<8><<<(unsigned)chunks, min(kThreads, ((d / 8) + 31) / 32 * 32), 0,
                             stream>>>(skey, n, d, ws, out, status);
    note_launch(2);
    return cudaGetLastError();
  }
  const int V = dt == PKM_BF16 ? 8 : 4;
  // two 16-byte column vectors per thread when they divide the row
  const int NV = (d / V) % 2 == 0 ? 2 : 1;
  // one thread per column group (whole warps, at most kThreads)
  const int threads = min(kThreads, ((d / V / NV) + 31) / 32 * 32);
  const int fix_threads = min(kThreads, ((d / V) + 31) / 32 * 32);
  if (dt == PKM_BF16) {
    if (NV == 2)
      segsum_chunk_kernel<PKM_BF16, 2><<<(unsigned)chunks, threads, 0, stream>>>(
          skey, sval, n, mark, coef, (const __nv_bfloat16*)src, div, d, ws, out, status);
    else
      segsum_chunk_kernel<PKM_BF16, 1><<<(unsigned)chunks, threads, 0, stream>>>(
          skey, sval, n, mark, coef, (const __nv_bfloat16*)src, div, d, ws, out, status);
    segsum_fixup_kernel<8><<<(unsigned)chunks, fix_threads, 0, stream>>>(skey, n, d, ws, out,
                                                                         status);
  } else {
    if (NV == 2)
      segsum_chunk_kernel<PKM_F32, 2><<<(unsigned)chunks, threads, 0, stream>>>(
          skey, sval, n, mark, coef, (const float*)src, div, d, ws, out, status);
    else
      segsum_chunk_kernel<PKM_F32, 1><<<(unsigned)chunks, threads, 0, stream>>>(
          skey, sval, n, mark, coef, (const float*)src, div, d, ws, out, status);
    segsum_fixup_kernel<4><<<(unsigned)chunks, fix_threads, 0, stream>>>(skey, n, d, ws, out,
                                                                         status);
  }
  note_launch(2);
  return cudaGetLastError();
}

}  // namespace pkm
