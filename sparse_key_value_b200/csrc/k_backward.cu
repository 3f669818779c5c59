// k_backward.cu -- training backward of the product-key lookup, selection
// held fixed (top-k is piecewise constant in its inputs).
//
// With w = softmax(S) over the k kept full scores S_j = s1[a_j] + s2[b_j]
// ("모델 안의 메모리", "작동 방식": a weighted average of the values read) and
// s_c[a] = sqrt(d_half) <u_c, kappa_c[a]>, u = q / max(|q|, eps),
// kappa = K / max(|K|, eps) (qk-normalization, "Memory Layers at Scale"
// digest, "Memory+ 블록"):
//   dw_j      = <dy_t, V[idx_j]>                 (bag_dw: re-gathers V)
//   dS_j      = w_j (dw_j - sum_l w_l dw_l)      (same kernel)
//   du_c      = sqrt(d_half) sum_j dS_j kappa_c[a_j]
//   dq_c      = (du_c - u_c <u_c, du_c>) / max(|q_c|, eps)   (dq_kernel)
//   dkappa_c[a] = sqrt(d_half) sum over (t,h,j) with a_j = a of dS_j u_c
//               (its entries written by dq_kernel too)
//   dK        = (dkappa - kappa <kappa, dkappa>) / max(|K|, eps)
// The value gradient and dkappa are sums over sorted keys (k_sort.cu,
// k_segsum.cu); this file holds the per-token kernels.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace pkm {

__global__ void iota_kernel(uint32_t* __restrict__ v, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) v[i] = (uint32_t)i;
}

cudaError_t launch_iota(uint32_t* v, int64_t n, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  iota_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(v, n);
  note_launch();
  return cudaGetLastError();
}

// keys[i] = idx[i] when 0 <= idx[i] < limit, else `limit` (sorted last and
// skipped by the segmented sums); an out-of-range id sets the status word.
__global__ void sanitize_keys_kernel(const int32_t* __restrict__ idx, int64_t n, int64_t limit,
                                     uint32_t* __restrict__ keys, int32_t* status) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int32_t r = idx[i];
  const bool ok = r >= 0 && (int64_t)r < limit;
  if (!ok) set_status(status, PKM_ERR_DEVICE);
  keys[i] = ok ? (uint32_t)r : (uint32_t)limit;
}

cudaError_t launch_sanitize_keys(const int32_t* idx, int64_t n, int64_t limit, uint32_t* keys,
                                 int32_t* status, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  sanitize_keys_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(idx, n, limit, keys,
                                                                        status);
  note_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ dw, dS
// One CTA per bag; the bag's dy row is staged in shared memory, each warp
// takes rows j = warp, warp + 8, ... and reduces <dy, table[idx_j]> across
// its lanes (16-byte loads, consecutive lanes on consecutive bytes).
template <pkm_dtype DT>
__global__ void __launch_bounds__(256) bag_dw_kernel(
    const typename Elem<DT>::T* __restrict__ dy, const typename Elem<DT>::T* __restrict__ table,
    int64_t n_rows, int d, const int32_t* __restrict__ idx, const float* __restrict__ w,
    int B, int group, float* __restrict__ dw_out, float* __restrict__ dS_out, int32_t* status) {
  constexpr int V = Elem<DT>::kVec;
  extern __shared__ uint4 sdy[];  // [d / V] raw chunks, then dw [B]
  const int chunks = d / V;
  float* sdw = reinterpret_cast<float*>(sdy + chunks);
  const int64_t t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int c = threadIdx.x; c < chunks; c += blockDim.x)
    sdy[c] = ldg_nc_16(dy + t * d + (int64_t)c * V);
  __syncthreads();
  for (int j = warp; j < B; j += blockDim.x / 32) {
    const int32_t r = idx[t * B + j];
    float part = 0.f;
    if (r >= 0 && r < n_rows) {
      const typename Elem<DT>::T* row = table + (int64_t)r * d;
      for (int c0 = lane; c0 < chunks; c0 += 32 * 8) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int c = c0 + u * 32;
          if (c < chunks) v[u] = ldg_nc_16(row + (int64_t)c * V);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int c = c0 + u * 32;
          if (c < chunks) {
            float a[V], b[V];
            unpack16<DT>(v[u], a);
            unpack16<DT>(sdy[c], b);
#pragma unroll
            for (int e = 0; e < V; ++e) part = fmaf(a[e], b[e], part);
          }
        }
      }
    } else if (lane == 0) {
      set_status(status, PKM_ERR_DEVICE);
    }
    part = warp_sum(part);
    if (lane == 0) sdw[j] = part;
  }
  __syncthreads();
  if (dw_out)
    for (int j = threadIdx.x; j < B; j += blockDim.x) dw_out[t * B + j] = sdw[j];
  if (group > 0 && dS_out) {
    // softmax backward per group (one head's k selected rows)
    for (int g = warp; g < B / group; g += blockDim.x / 32) {
      const int j0 = g * group + lane, j1 = j0 + 32;
      const bool v0 = lane < group, v1 = lane + 32 < group;
      const float w0 = v0 ? w[t * B + j0] : 0.f, w1 = v1 ? w[t * B + j1] : 0.f;
      const float d0 = v0 ? sdw[j0] : 0.f, d1 = v1 ? sdw[j1] : 0.f;
      const float sum = warp_sum(w0 * d0 + w1 * d1);
      if (v0) dS_out[t * B + j0] = w0 * (d0 - sum);
      if (v1) dS_out[t * B + j1] = w1 * (d1 - sum);
    }
  }
}

cudaError_t launch_bag_dw(const void* dy, const void* table, int64_t n_rows, int d,
                          pkm_dtype dt, const int32_t* idx, const float* w, int64_t n_bags,
                          int B, int group, float* dw, float* dS, int32_t* status,
                          cudaStream_t stream) {
  if (n_bags <= 0) return cudaSuccess;
  const int V = dt == PKM_BF16 ? 8 : 4;
  const size_t smem = (size_t)(d / V) * 16 + (size_t)B * 4;
  if (dt == PKM_BF16) {
    auto fn = bag_dw_kernel<PKM_BF16>;
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    fn<<<(unsigned)n_bags, 256, smem, stream>>>((const __nv_bfloat16*)dy,
                                                (const __nv_bfloat16*)table, n_rows, d, idx, w,
                                                B, group, dw, dS, status);
  } else {
    auto fn = bag_dw_kernel<PKM_F32>;
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    fn<<<(unsigned)n_bags, 256, smem, stream>>>((const float*)dy, (const float*)table, n_rows, d,
                                                idx, w, B, group, dw, dS, status);
  }
  note_launch();
  return cudaGetLastError();
}

// ----------------------------------------------------------- softmax bwd
// One warp per group of k <= 64 entries (a token's head): dS = w (dw - <w, dw>).
__global__ void __launch_bounds__(256) softmax_bwd_kernel(const float* __restrict__ w,
                                                          const float* __restrict__ dw,
                                                          int slices, int64_t groups, int k,
                                                          float* __restrict__ dS) {
  const int lane = threadIdx.x & 31;
  const int64_t g = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (g >= groups) return;
  const int64_t o = g * k, R = groups * k;
  const bool v0 = lane < k, v1 = lane + 32 < k;
  const float w0 = v0 ? w[o + lane] : 0.f, w1 = v1 ? w[o + lane + 32] : 0.f;
  float d0 = 0.f, d1 = 0.f;
  for (int s = 0; s < slices; ++s) {
    if (v0) d0 += dw[s * R + o + lane];
    if (v1) d1 += dw[s * R + o + lane + 32];
  }
  const float sum = warp_sum(w0 * d0 + w1 * d1);
  if (v0) dS[o + lane] = w0 * (d0 - sum);
  if (v1) dS[o + lane + 32] = w1 * (d1 - sum);
}

cudaError_t launch_softmax_bwd(const float* w, const float* dw, int slices, int64_t groups, int k,
                               float* dS, cudaStream_t stream) {
  if (groups <= 0) return cudaSuccess;
  softmax_bwd_kernel<<<(unsigned)((groups + 7) / 8), 256, 0, stream>>>(w, dw, slices, groups, k,
                                                                       dS);
  note_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------- dq
// One warp per (token, head); lane l holds elements [l*E, (l+1)*E) of the
// d_half-long vectors for E = d_half / 32 (a multiple of 8 up to 64).
// With `keys` the same pass also writes the sub-key gradient's entries: for
// each half c, every distinct sub-key position a among the k selected rows
// becomes one entry
//   key  = (h*2 + c) * n + a,
//   coef = sqrt(d_half) * (sum of dS_j with a_j = a) / max(|q_c|, eps)
// (the sum in j order, the same one du uses); the other slots get key =
// mark.  Entry e = ((t*H + h)*2 + c)*k + j, whose source row is query row e / k.
template <pkm_dtype DT, int E>
__global__ void __launch_bounds__(256) dq_kernel(
    const typename Elem<DT>::T* __restrict__ q, const typename Elem<DT>::T* __restrict__ K,
    const float* __restrict__ rk, const int32_t* __restrict__ idx,
    const float* __restrict__ dS, int64_t T, int H, int dh, int n, int k,
    float* __restrict__ dq, uint32_t mark, uint32_t* __restrict__ keys,
    float* __restrict__ coef) {
  constexpr int V = Elem<DT>::kVec;
  constexpr int NC = E / V;  // 16-byte chunks per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t th = (int64_t)blockIdx.x * (blockDim.x / 32) + warp;
  if (th >= T * H) return;
  const int h = (int)(th % H);
  const float scale = sqrtf((float)dh);
  const int32_t i0 = lane < k ? idx[th * k + lane] : 0;
  const int32_t i1 = lane + 32 < k ? idx[th * k + lane + 32] : 0;
  const float g0 = lane < k ? dS[th * k + lane] : 0.f;
  const float g1 = lane + 32 < k ? dS[th * k + lane + 32] : 0.f;
  __shared__ int32_t s_a[8][64];
  __shared__ float s_g[8][64];
  const int64_t N = (int64_t)n * n;
  for (int c = 0; c < 2; ++c) {
    const int hc = h * 2 + c;
    const typename Elem<DT>::T* Kc = K + (int64_t)hc * n * dh;
    // the query row's elements (held packed until the end) and its norm
    const int64_t qrow = th * 2 + c;
    const typename Elem<DT>::T* qp = q + qrow * dh + (int64_t)lane * E;
    uint4 qv[NC > 0 ? NC : 1];  // (NC = 0: an instance the launcher never runs)
    float ss = 0.f;
#pragma unroll
    for (int cc = 0; cc < NC; ++cc) {
      qv[cc] = ldg_nc_16(qp + cc * V);
      float f[V];
      unpack16<DT>(qv[cc], f);
#pragma unroll
      for (int e = 0; e < V; ++e) ss = fmaf(f[e], f[e], ss);
    }
    const float r = 1.0f / fmaxf(sqrtf(warp_sum(ss)), kNormEps);
    // sub-key positions of this half, each distinct one once with the sum of
    // its dS (in slot order), compacted into the warp's list
    const bool ok0 = lane < k && i0 >= 0 && (int64_t)i0 < N;
    const bool ok1 = lane + 32 < k && i1 >= 0 && (int64_t)i1 < N;
    const int32_t a0 = ok0 ? (c == 0 ? i0 / n : i0 % n) : -1;
    const int32_t a1 = ok1 ? (c == 0 ? i1 / n : i1 % n) : -1;
    bool lead0 = ok0, lead1 = ok1;
    float s0 = 0.f, s1 = 0.f;
    for (int j = 0; j < k; ++j) {
      const int32_t aj = __shfl_sync(0xffffffffu, j < 32 ? a0 : a1, j & 31);
      const float gj = __shfl_sync(0xffffffffu, j < 32 ? g0 : g1, j & 31);
      if (aj == a0) {
        if (j < lane) lead0 = false;
        if (j >= lane) s0 += gj;
      }
      if (aj == a1) {
        if (j < lane + 32) lead1 = false;
        if (j >= lane + 32) s1 += gj;
      }
    }
    if (keys) {
      // the sub-key gradient's entries of this (token, head, half): the same
      // distinct positions with their dS sums, scaled by the query's factor
      if (lane < k) {
        keys[qrow * k + lane] = lead0 ? (uint32_t)(hc * n + a0) : mark;
        coef[qrow * k + lane] = lead0 ? scale * s0 * r : 0.f;
      }
      if (lane + 32 < k) {
        keys[qrow * k + lane + 32] = lead1 ? (uint32_t)(hc * n + a1) : mark;
        coef[qrow * k + lane + 32] = lead1 ? scale * s1 * r : 0.f;
      }
    }
    const unsigned m0 = __ballot_sync(0xffffffffu, lead0);
    const unsigned m1 = __ballot_sync(0xffffffffu, lead1);
    const unsigned lt = (1u << lane) - 1u;
    if (lead0) {
      const int p = __popc(m0 & lt);
      s_a[warp][p] = a0;
      s_g[warp][p] = scale * s0 * rk[(int64_t)hc * n + a0];
    }
    if (lead1) {
      const int p = __popc(m0) + __popc(m1 & lt);
      s_a[warp][p] = a1;
      s_g[warp][p] = scale * s1 * rk[(int64_t)hc * n + a1];
    }
    __syncwarp();
    const int m = __popc(m0) + __popc(m1);
    // the sub-key rows stay in L2 while the query rows and dq stream past
    const uint64_t keep = l2_policy_keep();
    float du[E];
#pragma unroll
    for (int e = 0; e < E; ++e) du[e] = 0.f;
#pragma unroll 4
    for (int i = 0; i < m; ++i) {
      const int32_t a = s_a[warp][i];
      const float coef = s_g[warp][i];
      const typename Elem<DT>::T* row = Kc + (int64_t)a * dh + (int64_t)lane * E;
#pragma unroll
      for (int cc = 0; cc < NC; ++cc) {
        float f[V];
        unpack16<DT>(ldg_nc_16_hint(row + cc * V, keep), f);
#pragma unroll
        for (int e = 0; e < V; ++e) du[cc * V + e] = fmaf(coef, f[e], du[cc * V + e]);
      }
    }
    __syncwarp();
    float u[E];
#pragma unroll
    for (int cc = 0; cc < NC; ++cc) {
      float f[V];
      unpack16<DT>(qv[cc], f);
#pragma unroll
      for (int e = 0; e < V; ++e) u[cc * V + e] = f[e] * r;
    }
    float ud = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) ud = fmaf(u[e], du[e], ud);
    ud = warp_sum(ud);
    const bool clamped = !(r < 1.0f / kNormEps);  // |q| <= eps
    float* out = dq + qrow * dh + (int64_t)lane * E;
#pragma unroll
    for (int e = 0; e < E; e += 4) {
      float4 o;
      o.x = (clamped ? du[e] : du[e] - u[e] * ud) * r;
      o.y = (clamped ? du[e + 1] : du[e + 1] - u[e + 1] * ud) * r;
      o.z = (clamped ? du[e + 2] : du[e + 2] - u[e + 2] * ud) * r;
      o.w = (clamped ? du[e + 3] : du[e + 3] - u[e + 3] * ud) * r;
      *reinterpret_cast<float4*>(out + e) = o;
    }
  }
}

template <pkm_dtype DT>
static cudaError_t launch_dq_t(const void* q, const void* K, const float* rk,
                               const int32_t* idx, const float* dS, int64_t T, int H, int dh,
                               int n, int k, float* dq, uint32_t mark, uint32_t* keys,
                               float* coef, cudaStream_t stream) {
  using Tp = typename Elem<DT>::T;
  const unsigned grid = (unsigned)((T * H + 7) / 8);
  const int E = dh / 32;
#define PKM_DQ(EE)                                                                              \
  dq_kernel<DT, EE><<<grid, 256, 0, stream>>>((const Tp*)q, (const Tp*)K, rk, idx, dS, T, H,     \
                                              dh, n, k, dq, mark, keys, coef)
  if (E % Elem<DT>::kVec != 0) return cudaErrorInvalidValue;
  switch (E) {
    case 4: PKM_DQ(4); break;
    case 8: PKM_DQ(8); break;
    case 16: PKM_DQ(16); break;
    case 24: PKM_DQ(24); break;
    case 32: PKM_DQ(32); break;
    case 40: PKM_DQ(40); break;
    case 48: PKM_DQ(48); break;
    case 56: PKM_DQ(56); break;
    case 64: PKM_DQ(64); break;
    default: return cudaErrorInvalidValue;
  }
#undef PKM_DQ
  note_launch();
  return cudaGetLastError();
}

bool backward_dh_supported(pkm_dtype dt, int dh) {
  const int V = dt == PKM_BF16 ? 8 : 4;
  return dh % (32 * V) == 0 && dh / 32 <= 64;
}

cudaError_t launch_dq(const void* q, const void* K, pkm_dtype dt, const float* rk, const int32_t* idx, const float* dS, int64_t T, int H,
                      int dh, int n, int k, float* dq, uint32_t mark, uint32_t* keys,
                      float* coef, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  return dt == PKM_BF16
             ? launch_dq_t<PKM_BF16>(q, K, rk, idx, dS, T, H, dh, n, k, dq, mark, keys, coef,
                                     stream)
             : launch_dq_t<PKM_F32>(q, K, rk, idx, dS, T, H, dh, n, k, dq, mark, keys, coef,
                                    stream);
}

// ---------------------------------------------------- sub-key Jacobian
// In place: g <- (g - kappa <kappa, g>) * rk, kappa = K * rk; one warp per
// sub-key row (rows with no contribution hold g = 0 and stay 0).
template <pkm_dtype DT>
__global__ void __launch_bounds__(256) dk_jacobian_kernel(const typename Elem<DT>::T* __restrict__ K,
                                                          const float* __restrict__ rk,
                                                          int64_t rows, int dh,
                                                          float* __restrict__ g) {
  constexpr int V = Elem<DT>::kVec;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + warp;
  if (r >= rows) return;
  const float rr = rk[r];
  float kd = 0.f;
  for (int c = lane * V; c < dh; c += 32 * V) {
    float f[V];
    unpack16<DT>(ldg_nc_16(K + r * dh + c), f);
#pragma unroll
    for (int e = 0; e < V; ++e) kd = fmaf(f[e] * rr, g[r * dh + c + e], kd);
  }
  kd = warp_sum(kd);
  const bool clamped = !(rr < 1.0f / kNormEps);
  for (int c = lane * V; c < dh; c += 32 * V) {
    float f[V];
    unpack16<DT>(ldg_nc_16(K + r * dh + c), f);
#pragma unroll
    for (int e = 0; e < V; ++e) {
      const float gv = g[r * dh + c + e];
      g[r * dh + c + e] = (clamped ? gv : gv - f[e] * rr * kd) * rr;
    }
  }
}

cudaError_t launch_dk_jacobian(const void* K, pkm_dtype dt, const float* rk, int64_t rows, int dh,
                               float* g, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (dt == PKM_BF16)
    dk_jacobian_kernel<PKM_BF16><<<grid, 256, 0, stream>>>((const __nv_bfloat16*)K, rk, rows, dh, g);
  else
    dk_jacobian_kernel<PKM_F32><<<grid, 256, 0, stream>>>((const float*)K, rk, rows, dh, g);
  note_launch();
  return cudaGetLastError();
}

}  // namespace pkm
