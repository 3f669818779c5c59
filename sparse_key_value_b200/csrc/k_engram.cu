// k_engram.cu -- the Engram lookup: hashed n-gram rows, their sum and the
// context gate, in one kernel.
//
// "Conditional Memory via Scalable Lookup" review, "희소 검색" (multi-head
// hashing of the n-grams ending at each token into large embedding tables)
// and "핵심 수식": e = E_{n,k}[phi_{n,k}(g_{t,n})] and
// alpha = sigmoid(RMSNorm(h)^T RMSNorm(e) / sqrt(d)).  The page leaves the
// hash functions open; the library's definition is stated with
// pkm_engram_forward in include/pkm.h.  The heads' rows are summed (a bag of
// weight-one rows) into e, and v = alpha * e is the gated value.
//
// One CTA of 128 threads per token: the first `heads` threads hash the
// token's n-grams into shared memory, then every thread gathers its NCH
// 16-byte columns of each head's row (eight independent loads in flight per
// thread), the three sums <h,h>, <e,e>, <h,e> are reduced across the CTA in
// a fixed order, and each thread writes its columns of v.  The work is
// HBM-bound on the rows read; the token ids are re-read from L2 by the
// neighbouring tokens' CTAs.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace pkm {

namespace {

constexpr int kEngramThreads = 128;
constexpr float kEngramEps = 1e-6f;
constexpr uint32_t kEngramPad = 0xFFFFFFFFu;
constexpr uint64_t kEngramMul = 0x9E3779B97F4A7C15ull;

struct EngramCfg {
  int n_orders, K, heads;
  int order[PKM_ENGRAM_MAX_ORDERS];
  uint64_t seed[PKM_ENGRAM_MAX_HEADS];
  uint64_t M[PKM_ENGRAM_MAX_HEADS];
  uint64_t R[PKM_ENGRAM_MAX_HEADS];  // floor((2^64 - 1) / M): h mod M by multiply-high
  int64_t offset[PKM_ENGRAM_MAX_HEADS];
};

// Resident CTAs per SM: a CTA's loads are in flight only between its hash
// and its reduction, so as many CTAs as the SM's 2048 threads allow for one
// column per thread (16 measured faster than 10 and 12 despite a 16-byte
// spill); wider rows keep their loads in registers.
template <pkm_dtype DT, int NCH>
__global__ void __launch_bounds__(kEngramThreads, NCH == 1 ? 16 : (NCH == 2 ? 6 : 2)) engram_kernel(
    const __grid_constant__ EngramCfg cfg, int L, const int32_t* __restrict__ tokens,
    const typename Elem<DT>::T* __restrict__ table, int d,
    const typename Elem<DT>::T* __restrict__ h, typename Elem<DT>::T* __restrict__ v,
    float* __restrict__ alpha, int32_t* __restrict__ rows_out,
    typename Elem<DT>::T* __restrict__ e_out) {
  using T = typename Elem<DT>::T;
  constexpr int V = Elem<DT>::kVec;
  __shared__ int32_t s_rows[PKM_ENGRAM_MAX_HEADS];
  __shared__ float s_red[3][kEngramThreads / 32];
  const int64_t t = blockIdx.x;
  const int64_t seq = t / L;
  const int p = (int)(t - seq * L);
  const int tid = threadIdx.x;
  const int C16 = d / V;  // 16-byte columns of a row

  // the hidden-state columns, loaded first so that their latency overlaps
  // the hashing and the gather
  uint4 hraw[NCH];
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int col = tid + c * kEngramThreads;
    hraw[c] = col < C16 ? ldg_nc_16(h + t * d + (int64_t)col * V) : make_uint4(0, 0, 0, 0);
  }

  // hashed rows of this token's n-grams, one head per thread
  if (tid < cfg.heads) {
    const int n = cfg.order[tid / cfg.K];
    const int32_t* s = tokens + seq * L;
    uint64_t x = cfg.seed[tid];
    for (int i = n - 1; i >= 0; --i) {
      const int q = p - i;
      x ^= (uint64_t)(q >= 0 ? (uint32_t)s[q] : kEngramPad);
      x *= kEngramMul;
      x ^= x >> 32;
    }
    // x mod M without a 64-bit division: q = floor(x R / 2^64) undershoots
    // floor(x / M) by at most 2, so at most two subtractions remain
    const uint64_t M = cfg.M[tid];
    uint64_t rem = x - __umul64hi(x, cfg.R[tid]) * M;
    if (rem >= M) rem -= M;
    if (rem >= M) rem -= M;
    const int64_t r = cfg.offset[tid] + (int64_t)rem;
    s_rows[tid] = (int32_t)r;
    if (rows_out) rows_out[t * cfg.heads + tid] = (int32_t)r;
  }
  __syncthreads();

  // e = sum of the heads' rows (fp32, head order) for this thread's columns,
  // HB heads at a time: eight 16-byte loads in flight per thread
  constexpr int HB = NCH >= 8 ? 1 : 8 / NCH;
  float acc[NCH][V];
#pragma unroll
  for (int c = 0; c < NCH; ++c)
#pragma unroll
    for (int k = 0; k < V; ++k) acc[c][k] = 0.f;
  for (int j0 = 0; j0 < cfg.heads; j0 += HB) {
    uint4 raw[HB][NCH];
#pragma unroll
    for (int u = 0; u < HB; ++u)
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        const int col = tid + c * kEngramThreads;
        raw[u][c] = make_uint4(0, 0, 0, 0);
        if (j0 + u < cfg.heads && col < C16) {
          const int64_t r = s_rows[j0 + u];
          raw[u][c] = ldg_nc_16(table + r * d + (int64_t)col * V);
        }
      }
#pragma unroll
    for (int u = 0; u < HB; ++u)
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        float f[V];
        unpack16<DT>(raw[u][c], f);
#pragma unroll
        for (int k = 0; k < V; ++k) acc[c][k] += f[k];
      }
  }

  // <h,h>, <e,e>, <h,e> over the row, then the gate
  float hh = 0.f, ee = 0.f, he = 0.f;
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int col = tid + c * kEngramThreads;
    if (col >= C16) continue;
    float hv[V];
    unpack16<DT>(hraw[c], hv);
#pragma unroll
    for (int k = 0; k < V; ++k) {
      hh = fmaf(hv[k], hv[k], hh);
      ee = fmaf(acc[c][k], acc[c][k], ee);
      he = fmaf(hv[k], acc[c][k], he);
    }
  }
  hh = warp_sum(hh);
  ee = warp_sum(ee);
  he = warp_sum(he);
  if ((tid & 31) == 0) {
    s_red[0][tid / 32] = hh;
    s_red[1][tid / 32] = ee;
    s_red[2][tid / 32] = he;
  }
  __syncthreads();
  hh = ee = he = 0.f;
#pragma unroll
  for (int w = 0; w < kEngramThreads / 32; ++w) {  // same order in every thread
    hh += s_red[0][w];
    ee += s_red[1][w];
    he += s_red[2][w];
  }
  const float inv_d = 1.0f / (float)d;
  const float logit = he / (sqrtf(hh * inv_d + kEngramEps) * sqrtf(ee * inv_d + kEngramEps)) /
                      sqrtf((float)d);
  const float a = 1.0f / (1.0f + expf(-logit));
  if (tid == 0 && alpha) alpha[t] = a;

#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int col = tid + c * kEngramThreads;
    if (col >= C16) continue;
    const int64_t o = t * d + (int64_t)col * V;
    if (e_out) *reinterpret_cast<uint4*>(e_out + o) = pack16<DT>(acc[c]);
    float g[V];
#pragma unroll
    for (int k = 0; k < V; ++k) g[k] = a * acc[c][k];
    __stcs(reinterpret_cast<uint4*>(v + o), pack16<DT>(g));
  }
}

template <pkm_dtype DT>
cudaError_t launch_engram_t(const EngramCfg& cfg, int64_t n_seq, int L, const int32_t* tokens,
                            const void* table, int d, const void* h, void* v, float* alpha,
                            int32_t* rows, void* e, cudaStream_t stream) {
  using T = typename Elem<DT>::T;
  const int64_t T_ = n_seq * L;
  const int C16 = d / Elem<DT>::kVec;
  const int nch = (C16 + kEngramThreads - 1) / kEngramThreads;
  dim3 grid((unsigned)T_);
#define PKM_ENGRAM_LAUNCH(N)                                                                  \
  engram_kernel<DT, N><<<grid, kEngramThreads, 0, stream>>>(                                  \
      cfg, L, tokens, (const T*)table, d, (const T*)h, (T*)v, alpha, rows, (T*)e)
  if (nch <= 1)
    PKM_ENGRAM_LAUNCH(1);
  else if (nch <= 2)
    PKM_ENGRAM_LAUNCH(2);
  else if (nch <= 4)
    PKM_ENGRAM_LAUNCH(4);
  else
    PKM_ENGRAM_LAUNCH(8);
#undef PKM_ENGRAM_LAUNCH
  note_launch();
  return cudaGetLastError();
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

}  // namespace pkm

using namespace pkm;

extern "C" {

PKM_API pkm_status pkm_engram_forward(const pkm_engram_args* a, pkm_stream_t stream) {
  if (!a || a->n_seq < 0 || a->L < 1 || a->n_orders < 1 ||
      a->n_orders > PKM_ENGRAM_MAX_ORDERS || a->K < 1 || a->K > PKM_ENGRAM_MAX_HEADS)
    return PKM_ERR_INVALID_ARG;
  if (a->dtype != PKM_F32 && a->dtype != PKM_BF16) return PKM_ERR_INVALID_ARG;
  const int heads = a->n_orders * a->K;
  if (heads > PKM_ENGRAM_MAX_HEADS) return PKM_ERR_INVALID_ARG;
  const int max_d = a->dtype == PKM_BF16 ? 8192 : 4096;
  if (a->d < 8 || a->d % 8 || a->d > max_d) return PKM_ERR_INVALID_ARG;
  if (!a->orders || !a->seeds || !a->rows_per_head) return PKM_ERR_INVALID_ARG;
  EngramCfg cfg{};
  cfg.n_orders = a->n_orders;
  cfg.K = a->K;
  cfg.heads = heads;
  for (int o = 0; o < a->n_orders; ++o) {
    if (a->orders[o] < 1 || a->orders[o] > 8) return PKM_ERR_INVALID_ARG;
    cfg.order[o] = a->orders[o];
  }
  int64_t total = 0;
  for (int j = 0; j < heads; ++j) {
    if (a->rows_per_head[j] < 1) return PKM_ERR_INVALID_ARG;
    cfg.seed[j] = a->seeds[j];
    cfg.M[j] = (uint64_t)a->rows_per_head[j];
    cfg.R[j] = ~0ull / cfg.M[j];
    cfg.offset[j] = total;
    total += a->rows_per_head[j];
    if (total >= (int64_t(1) << 31)) return PKM_ERR_INVALID_ARG;
  }
  if (a->n_seq == 0) return PKM_OK;
  if (!a->tokens || (reinterpret_cast<uintptr_t>(a->tokens) & 3u)) return PKM_ERR_INVALID_ARG;
  const void* need[] = {a->table, a->h, a->v};
  for (const void* p : need)
    if (!p || !al16(p)) return PKM_ERR_INVALID_ARG;
  if ((a->e && !al16(a->e)) || (a->alpha && (reinterpret_cast<uintptr_t>(a->alpha) & 3u)) ||
      (a->rows && (reinterpret_cast<uintptr_t>(a->rows) & 3u)))
    return PKM_ERR_INVALID_ARG;
  if (a->n_seq * (int64_t)a->L >= (int64_t(1) << 31)) return PKM_ERR_INVALID_ARG;
  // every row id is in range by construction (offset_j + h mod M_j)
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const cudaError_t e =
      a->dtype == PKM_BF16
          ? launch_engram_t<PKM_BF16>(cfg, a->n_seq, a->L, a->tokens, a->table, a->d, a->h, a->v,
                                      a->alpha, a->rows, a->e, st)
          : launch_engram_t<PKM_F32>(cfg, a->n_seq, a->L, a->tokens, a->table, a->d, a->h, a->v,
                                     a->alpha, a->rows, a->e, st);
  return e == cudaSuccess ? PKM_OK : PKM_ERR_CUDA;
}

}  // extern "C"
