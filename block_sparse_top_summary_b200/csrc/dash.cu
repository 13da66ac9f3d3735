// DashAttention's adaptive stages on the CUDA cores (DashAttention page,
// "Metodologia", stages 0-2):
//   learned_summary_kernel  S_j = sum_t softmax_t(scale qbar . k_t) k_t per complete block;
//   entmax_route_wh_kernel  per (b, KV head, query block): per head, pooled query,
//   (entmax_route_kernel    logits against the summaries of blocks 0 .. i-1, alpha-entmax
//   when its shared memory  of gamma * logits by bisection on tau, mean over the group;
//   does not fit)           writes the support (ascending) plus the diagonal block as an
//                           index list, with the prior bias sigma * log w per entry (0 on
//                           the diagonal), and optionally the dense probabilities w;
//   attention with the prior: the tensor-core prefill kernel (attn_tc.cu, PRIOR) or the
//                           SIMT one (attn_simt.cu, bias != NULL) with the entry's bias
//                           added to the logits of every key of that block.
#include "common.cuh"
#include "kernels.h"

namespace ssa {

namespace {
__device__ __forceinline__ float to_float(float v) { return v; }
__device__ __forceinline__ float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }

constexpr int kSumRows = 16;      // key rows in flight per warp (learned summary)
constexpr int kRouteThreads = 256;
constexpr int kBisect = 40;       // bisection steps on tau (interval 1 -> 2^-40)
}  // namespace

// E consecutive elements of one row, loaded as one vector of E * sizeof(T)
// bytes (4, 8 or 16), widened to fp32 exactly.
template <int E>
__device__ __forceinline__ void load_row(const float* p, float (&v)[E]) {
  if constexpr (E == 4) {
    const float4 x = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  } else {
    const float2 x = __ldg(reinterpret_cast<const float2*>(p));
    v[0] = x.x; v[1] = x.y;
  }
}
template <int E>
__device__ __forceinline__ void load_row(const __nv_bfloat16* p, float (&v)[E]) {
  if constexpr (E == 4) {
    const uint2 x = __ldg(reinterpret_cast<const uint2*>(p));
    bf16x2_to_f(x.x, v[0], v[1]);
    bf16x2_to_f(x.y, v[2], v[3]);
  } else {
    const uint32_t x = __ldg(reinterpret_cast<const unsigned int*>(p));
    bf16x2_to_f(x, v[0], v[1]);
  }
}

// One warp per (b, KV head, complete block); lane owns D / 32 consecutive
// columns.  kSumRows rows are loaded per step (one vector load each), their
// logits are reduced together, and the step is folded into the online softmax
// with one rescale to the step's new maximum.
template <typename T, int D>
__global__ void __launch_bounds__(256) learned_summary_kernel(
    const T* __restrict__ K, const float* __restrict__ qbar, float* __restrict__ S, int Hkv,
    int N, int B, int nfull, long long units, float scale_log2) {
  constexpr int E = D / 32;  // columns per lane
  const long long u = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (u >= units) return;
  const long long bg = u / nfull;
  const int j = (int)(u - bg * nfull);
  const int g = (int)(bg % Hkv);
  float q[E], acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    q[e] = qbar[(size_t)g * D + lane * E + e] * scale_log2;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const T* base = K + ((size_t)bg * N + (size_t)j * B) * D + lane * E;
  for (int r0 = 0; r0 < B; r0 += kSumRows) {
    float k[kSumRows][E], z[kSumRows];
#pragma unroll
    for (int rr = 0; rr < kSumRows; ++rr) load_row<E>(base + (size_t)min(r0 + rr, B - 1) * D, k[rr]);
#pragma unroll
    for (int rr = 0; rr < kSumRows; ++rr) {
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) a = fmaf(q[e], k[rr][e], a);
      z[rr] = a;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int rr = 0; rr < kSumRows; ++rr) z[rr] += __shfl_xor_sync(0xffffffffu, z[rr], o);
    // one rescale per step: the step's rows against the running max
    float mn = m;
#pragma unroll
    for (int rr = 0; rr < kSumRows; ++rr)
      if (r0 + rr < B) mn = fmaxf(mn, z[rr]);
    const float al = exp2f(m - mn);
    l *= al;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] *= al;
#pragma unroll
    for (int rr = 0; rr < kSumRows; ++rr) {
      const float p = r0 + rr < B ? exp2f(z[rr] - mn) : 0.f;
      l += p;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = fmaf(p, k[rr][e], acc[e]);
    }
    m = mn;
  }
  float* out = S + (size_t)u * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; ++e) out[e] = acc[e] / l;
}

namespace {

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < kRouteThreads / 32; ++i) t += red[i];
  return t;
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float t = -INFINITY;
#pragma unroll
  for (int i = 0; i < kRouteThreads / 32; ++i) t = fmaxf(t, red[i]);
  return t;
}

// [x]_+^inv for x >= 0 (inv = 1 / (alpha - 1))
__device__ __forceinline__ float pos_pow(float x, float inv) {
  if (x <= 0.f) return 0.f;
  if (inv == 1.f) return x;
  if (inv == 2.f) return x * x;
  return exp2f(inv * log2f(x));
}

}  // namespace

// One CTA per (b, KV head, query block); dynamic shared memory: qbar [D] + z [nq] + w [nq].
template <typename T, int D>
__global__ void __launch_bounds__(kRouteThreads) entmax_route_kernel(
    const T* __restrict__ Q, const float* __restrict__ S, int32_t* __restrict__ idx,
    int32_t* __restrict__ cnt, float* __restrict__ bias, float* __restrict__ wout, int Hq,
    int Hkv, int N, int B, int nq, int nfull, int max_sel, float alpha, float zscale,
    float sigma) {
  extern __shared__ float sm_route[];
  float* qb = sm_route;      // [D]
  float* z = qb + D;         // [nq]
  float* w = z + nq;         // [nq]
  __shared__ float red[kRouteThreads / 32];
  __shared__ int wc[kRouteThreads / 32];
  const int i = blockIdx.x % nq;
  const int bg = blockIdx.x / nq;
  const int b = bg / Hkv, g = bg - b * Hkv;
  const int G = Hq / Hkv;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int nc = min(i, nfull);
  const float am1 = alpha - 1.f, inv = 1.f / am1;
  const int r0 = i * B, rows = min(B, N - r0);

  for (int j = t; j < nc; j += kRouteThreads) w[j] = 0.f;
  for (int h = 0; h < G && nc > 0; ++h) {
    // ---- pooled query of head h over the block's rows
    const T* qh = Q + (((size_t)b * Hq + g * G + h) * N + r0) * D;
    __syncthreads();  // qb and z of the previous head are consumed
    for (int c = t; c < D; c += kRouteThreads) {
      float a = 0.f;
      for (int r = 0; r < rows; ++r) a += to_float(qh[(size_t)r * D + c]);
      qb[c] = a / rows;
    }
    __syncthreads();
    // ---- logits of the candidates: one warp per candidate
    for (int j = warp; j < nc; j += kRouteThreads / 32) {
      const float* sj = S + (((size_t)b * Hkv + g) * nfull + j) * D;
      float a = 0.f;
      for (int c = lane; c < D; c += 32) a = fmaf(qb[c], sj[c], a);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0) z[j] = am1 * zscale * a;  // (alpha - 1) * gamma * logit
    }
    __syncthreads();
    // ---- tau by bisection in [max - 1, max]
    float mx = -INFINITY;
    for (int j = t; j < nc; j += kRouteThreads) mx = fmaxf(mx, z[j]);
    mx = block_max(mx, red);
    float lo = mx - 1.f, hi = mx;
    for (int it = 0; it < kBisect; ++it) {
      const float mid = 0.5f * (lo + hi);
      float s = 0.f;
      for (int j = t; j < nc; j += kRouteThreads) s += pos_pow(z[j] - mid, inv);
      s = block_sum(s, red);
      if (s >= 1.f) lo = mid;
      else hi = mid;
    }
    float s = 0.f;
    for (int j = t; j < nc; j += kRouteThreads) s += pos_pow(z[j] - lo, inv);
    s = block_sum(s, red);
    const float norm = 1.f / (s * G);
    for (int j = t; j < nc; j += kRouteThreads) w[j] += pos_pow(z[j] - lo, inv) * norm;
  }
  __syncthreads();

  // ---- support (ascending) + the diagonal block, in order
  const size_t urow = (size_t)bg * nq + i;
  int32_t* irow = idx + urow * max_sel;
  float* brow = bias + urow * max_sel;
  int total = 0;
  for (int base = 0; base < nc; base += kRouteThreads) {
    const int j = base + t;
    const bool on = j < nc && w[j] > 0.f;
    const unsigned bal = __ballot_sync(0xffffffffu, on);
    if (lane == 0) wc[warp] = __popc(bal);
    __syncthreads();
    int off = 0, n = 0;
#pragma unroll
    for (int ww = 0; ww < kRouteThreads / 32; ++ww) {
      if (ww < warp) off += wc[ww];
      n += wc[ww];
    }
    const int pos = total + off + __popc(bal & ((1u << lane) - 1u));
    if (on && pos < max_sel - 1) {
      irow[pos] = j;
      brow[pos] = sigma * logf(w[j]);
    }
    total += n;
    __syncthreads();
  }
  if (t == 0) {
    const int k = min(total, max_sel - 1);
    irow[k] = i;
    brow[k] = 0.f;
    for (int e = k + 1; e < max_sel; ++e) {
      irow[e] = -1;
      brow[e] = 0.f;
    }
    cnt[urow] = k + 1;
  }
  if (wout != nullptr) {
    float* wr = wout + urow * nfull;
    for (int j = t; j < nfull; j += kRouteThreads) wr[j] = j < nc ? w[j] : 0.f;
  }
}

// The same routing with the group's heads spread over the warps: warp h
// pools head h and solves its tau by bisection with warp-level sums, so the
// 40 bisection steps need no block barrier; the logits are formed for all
// heads from one load of each summary.  The pooled queries, the logits and
// the head-ordered sum into w are computed in the order of
// entmax_route_kernel (bitwise the same); only the bisection's sums run in
// another order.  Dynamic shared memory: qbar [G][D], z [G][nq] (the logits,
// then each head's probabilities), w [nq].
template <typename T, int D>
__global__ void __launch_bounds__(kRouteThreads) entmax_route_wh_kernel(
    const T* __restrict__ Q, const float* __restrict__ S, int32_t* __restrict__ idx,
    int32_t* __restrict__ cnt, float* __restrict__ bias, float* __restrict__ wout, int Hq,
    int Hkv, int N, int B, int nq, int nfull, int max_sel, float alpha, float zscale,
    float sigma) {
  constexpr int E = D / 32;       // columns per lane
  constexpr int RB = 8;           // rows in flight per lane while pooling
  constexpr int NW = kRouteThreads / 32;
  extern __shared__ float sm_route[];
  const int G = Hq / Hkv;
  float* qb = sm_route;                  // [G][D]
  float* z = qb + (size_t)G * D;         // [G][nq]
  float* w = z + (size_t)G * nq;         // [nq]
  __shared__ int wc[NW];
  const int i = blockIdx.x % nq;
  const int bg = blockIdx.x / nq;
  const int b = bg / Hkv, g = bg - b * Hkv;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int nc = min(i, nfull);
  const float am1 = alpha - 1.f, inv = 1.f / am1;
  const int r0 = i * B, rows = min(B, N - r0);

  // ---- pooled query of each head: lane owns columns lane + 32 e, rows summed in order
  for (int h = warp; h < G && nc > 0; h += NW) {
    const T* qh = Q + (((size_t)b * Hq + g * G + h) * N + r0) * D + lane;
    float a[E];
#pragma unroll
    for (int e = 0; e < E; ++e) a[e] = 0.f;
    for (int rb = 0; rb < rows; rb += RB) {
      float v[RB][E];
#pragma unroll
      for (int u = 0; u < RB; ++u)
#pragma unroll
        for (int e = 0; e < E; ++e)
          v[u][e] = rb + u < rows ? to_float(qh[(size_t)(rb + u) * D + 32 * e]) : 0.f;
#pragma unroll
      for (int u = 0; u < RB; ++u)
        if (rb + u < rows) {
#pragma unroll
          for (int e = 0; e < E; ++e) a[e] += v[u][e];
        }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) qb[h * D + lane + 32 * e] = a[e] / rows;
  }
  __syncthreads();
  // ---- logits of the candidates: one warp per candidate, every head
  for (int j = warp; j < nc; j += NW) {
    const float* sj = S + ((size_t)bg * nfull + j) * D + lane;
    float sv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) sv[e] = sj[32 * e];
    for (int h = 0; h < G; ++h) {
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) a = fmaf(qb[h * D + lane + 32 * e], sv[e], a);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0) z[(size_t)h * nq + j] = am1 * zscale * a;  // (alpha - 1) * gamma * logit
    }
  }
  __syncthreads();
  // ---- tau of each head by bisection in [max - 1, max], then its probabilities / G
  for (int h = warp; h < G && nc > 0; h += NW) {
    float* zh = z + (size_t)h * nq;
    float mx = -INFINITY;
    for (int j = lane; j < nc; j += 32) mx = fmaxf(mx, zh[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float lo = mx - 1.f, hi = mx;
    for (int it = 0; it < kBisect; ++it) {
      const float mid = 0.5f * (lo + hi);
      float sum = 0.f;
      for (int j = lane; j < nc; j += 32) sum += pos_pow(zh[j] - mid, inv);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (sum >= 1.f) lo = mid;
      else hi = mid;
    }
    float sum = 0.f;
    for (int j = lane; j < nc; j += 32) sum += pos_pow(zh[j] - lo, inv);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float norm = 1.f / (sum * G);
    __syncwarp();
    for (int j = lane; j < nc; j += 32) zh[j] = pos_pow(zh[j] - lo, inv) * norm;
  }
  __syncthreads();
  // ---- w = the heads' probabilities summed in head order
  for (int j = t; j < nc; j += kRouteThreads) {
    float a = 0.f;
    for (int h = 0; h < G; ++h) a += z[(size_t)h * nq + j];
    w[j] = a;
  }
  __syncthreads();

  // ---- support (ascending) + the diagonal block, in order
  const size_t urow = (size_t)bg * nq + i;
  int32_t* irow = idx + urow * max_sel;
  float* brow = bias + urow * max_sel;
  int total = 0;
  for (int base = 0; base < nc; base += kRouteThreads) {
    const int j = base + t;
    const bool on = j < nc && w[j] > 0.f;
    const unsigned bal = __ballot_sync(0xffffffffu, on);
    if (lane == 0) wc[warp] = __popc(bal);
    __syncthreads();
    int off = 0, n = 0;
#pragma unroll
    for (int ww = 0; ww < NW; ++ww) {
      if (ww < warp) off += wc[ww];
      n += wc[ww];
    }
    const int pos = total + off + __popc(bal & ((1u << lane) - 1u));
    if (on && pos < max_sel - 1) {
      irow[pos] = j;
      brow[pos] = sigma * logf(w[j]);
    }
    total += n;
    __syncthreads();
  }
  if (t == 0) {
    const int k = min(total, max_sel - 1);
    irow[k] = i;
    brow[k] = 0.f;
    for (int e = k + 1; e < max_sel; ++e) {
      irow[e] = -1;
      brow[e] = 0.f;
    }
    cnt[urow] = k + 1;
  }
  if (wout != nullptr) {
    float* wr = wout + urow * nfull;
    for (int j = t; j < nfull; j += kRouteThreads) wr[j] = j < nc ? w[j] : 0.f;
  }
}

cudaError_t launch_learned_summary(const void* K, ssa_dtype dt, const float* qbar, int batch,
                                   int Hkv, int N, int d, int B, float* S, cudaStream_t st) {
  const int nfull = N / B;
  const long long units = (long long)batch * Hkv * nfull;
  if (units == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((units + 7) / 8);
  const float sl = 1.4426950408889634f / sqrtf((float)d);
  if (dt == SSA_BF16) {
    if (d == 128)
      learned_summary_kernel<__nv_bfloat16, 128><<<grid, 256, 0, st>>>(
          (const __nv_bfloat16*)K, qbar, S, Hkv, N, B, nfull, units, sl);
    else
      learned_summary_kernel<__nv_bfloat16, 64><<<grid, 256, 0, st>>>(
          (const __nv_bfloat16*)K, qbar, S, Hkv, N, B, nfull, units, sl);
  } else {
    if (d == 128)
      learned_summary_kernel<float, 128><<<grid, 256, 0, st>>>((const float*)K, qbar, S, Hkv, N,
                                                               B, nfull, units, sl);
    else
      learned_summary_kernel<float, 64><<<grid, 256, 0, st>>>((const float*)K, qbar, S, Hkv, N,
                                                              B, nfull, units, sl);
  }
  return cudaGetLastError();
}

cudaError_t launch_entmax_route(const void* Q, ssa_dtype dt, const float* S, int batch, int Hq,
                                int Hkv, int N, int d, int B, float alpha, float gamma,
                                float sigma, int max_sel, int32_t* idx, int32_t* cnt,
                                float* bias, float* w, cudaStream_t st) {
  const int nq = (N + B - 1) / B;
  const int nfull = N / B;
  const int G = Hq / Hkv;
  // heads over the warps while qbar, the G logit rows and w fit in shared memory
  const size_t smem_wh = sizeof(float) * ((size_t)G * d + (size_t)(G + 1) * nq);
  const bool wh = smem_wh <= (size_t)200 * 1024;
  const size_t smem = wh ? smem_wh : sizeof(float) * ((size_t)d + 2 * (size_t)nq);
  const unsigned grid = (unsigned)((long long)batch * Hkv * nq);
  const float zs = gamma / sqrtf((float)d);
  cudaError_t e = cudaSuccess;
#define SSA_LAUNCH_ROUTE(TT, DD)                                                               \
  if (wh) {                                                                                  \
    e = cudaFuncSetAttribute(entmax_route_wh_kernel<TT, DD>,                                 \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);         \
    if (e != cudaSuccess) return e;                                                          \
    entmax_route_wh_kernel<TT, DD><<<grid, kRouteThreads, smem, st>>>(                       \
        (const TT*)Q, S, idx, cnt, bias, w, Hq, Hkv, N, B, nq, nfull, max_sel, alpha, zs,    \
        sigma);                                                                              \
  } else {                                                                                   \
    e = cudaFuncSetAttribute(entmax_route_kernel<TT, DD>,                                    \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);         \
    if (e != cudaSuccess) return e;                                                          \
    entmax_route_kernel<TT, DD><<<grid, kRouteThreads, smem, st>>>(                          \
        (const TT*)Q, S, idx, cnt, bias, w, Hq, Hkv, N, B, nq, nfull, max_sel, alpha, zs,    \
        sigma);                                                                              \
  }
  if (dt == SSA_BF16) {
    if (d == 128) {
      SSA_LAUNCH_ROUTE(__nv_bfloat16, 128);
    } else {
      SSA_LAUNCH_ROUTE(__nv_bfloat16, 64);
    }
  } else {
    if (d == 128) {
      SSA_LAUNCH_ROUTE(float, 128);
    } else {
      SSA_LAUNCH_ROUTE(float, 64);
    }
  }
#undef SSA_LAUNCH_ROUTE
  return cudaGetLastError();
}

}  // namespace ssa
