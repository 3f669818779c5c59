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

// Segmented sums of coef[e] * src[e / div] over the sorted pairs; entries
// with key == mark (sorted last) are ignored.  Outputs: sparse rows
// (uniq_rows/grad_rows, capacity cap; n_uniq receives the number of keys),
// dense_add[key] += sum, dense_set[key] = sum (any may be null).
cudaError_t launch_segsum(const uint32_t* skey, const uint32_t* sval, int64_t n, uint32_t mark,
                          const float* coef, const void* src, pkm_dtype dt, int64_t div, int d,
                          int32_t* uniq_rows, float* grad_rows, int64_t cap, int64_t* n_uniq,
                          float* dense_add, float* dense_set, void* workspace, int32_t* status,
                          cudaStream_t stream) {
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
