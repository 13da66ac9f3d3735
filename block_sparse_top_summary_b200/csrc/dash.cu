// DashAttention's adaptive stages on the CUDA cores (DashAttention page,
// "Metodologia", stages 0-2):
//   learned_summary_kernel  S_j = sum_t softmax_t(scale qbar . k_t) k_t per complete block;
//   entmax_route_kernel     per (b, KV head, query block): per head, pooled query,
//                           logits against the summaries of blocks 0 .. i-1, alpha-entmax
//                           of gamma * logits by bisection on tau, mean over the group;
//                           writes the support (ascending) plus the diagonal block as an
//                           index list, with the prior bias sigma * log w per entry (0 on
//                           the diagonal), and optionally the dense probabilities w;
//   attention with the prior: the SIMT prefill kernel with the entry's bias added to the
//                           logits of every key of that block (attn_simt.cu, bias != NULL).
#include "common.cuh"
#include "kernels.h"

namespace ssa {

namespace {
__device__ __forceinline__ float to_float(float v) { return v; }
__device__ __forceinline__ float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }

constexpr int kSumRows = 8;       // key rows in flight per warp (learned summary)
constexpr int kRouteThreads = 256;
constexpr int kBisect = 40;       // bisection steps on tau (interval 1 -> 2^-40)
}  // namespace

// One warp per (b, KV head, complete block); lane owns D / 32 columns.
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
    for (int rr = 0; rr < kSumRows; ++rr) {
      const int r = min(r0 + rr, B - 1);
#pragma unroll
      for (int e = 0; e < E; ++e) k[rr][e] = to_float(base[(size_t)r * D + e]);
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) a = fmaf(q[e], k[rr][e], a);
      z[rr] = a;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int rr = 0; rr < kSumRows; ++rr) z[rr] += __shfl_xor_sync(0xffffffffu, z[rr], o);
#pragma unroll
    for (int rr = 0; rr < kSumRows; ++rr) {
      if (r0 + rr >= B) break;
      const float mn = fmaxf(m, z[rr]);
      const float al = exp2f(m - mn), p = exp2f(z[rr] - mn);
      l = l * al + p;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = fmaf(p, k[rr][e], acc[e] * al);
      m = mn;
    }
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
  const size_t smem = sizeof(float) * ((size_t)d + 2 * (size_t)nq);
  const unsigned grid = (unsigned)((long long)batch * Hkv * nq);
  const float zs = gamma / sqrtf((float)d);
  cudaError_t e = cudaSuccess;
#define SSA_LAUNCH_ROUTE(TT, DD)                                                               \
  e = cudaFuncSetAttribute(entmax_route_kernel<TT, DD>,                                      \
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);           \
  if (e != cudaSuccess) return e;                                                            \
  entmax_route_kernel<TT, DD><<<grid, kRouteThreads, smem, st>>>(                            \
      (const TT*)Q, S, idx, cnt, bias, w, Hq, Hkv, N, B, nq, nfull, max_sel, alpha, zs, sigma)
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
