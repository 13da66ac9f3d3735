// Two-level routing (segments of M blocks, then blocks), one CTA per
// (batch, KV head g, query block i), 256 threads:
//   1. qbar = mean of Q over the block's rows and the group's heads;
//   2. block scores z_j = qbar . S_j / sqrt(d) for the complete blocks j < i;
//   3. segment scores = the mean of their blocks' scores (= qbar . mean summary,
//      by linearity) for the closed segments ((m + 1) M <= i) holding a
//      candidate; warp 0 keeps the top k_seg (ties to the lower index);
//   4. candidates 1 .. i-1 outside the kept and the open segments get -inf;
//      warp 0 keeps the top min(k_blk, pool size) of the rest;
//   5. selection = {0} + kept blocks + {i}, ascending.
// Dynamic shared memory: qbar [d], block scores [nq], segment scores [nq / M + 1].
#include "common.cuh"
#include "kernels.h"

namespace ssa {

namespace {
constexpr int kHierThreads = 256;
__device__ __forceinline__ float tof(float v) { return v; }
__device__ __forceinline__ float tof(__nv_bfloat16 v) { return __bfloat162float(v); }
}  // namespace

template <typename T, int D>
__global__ void __launch_bounds__(kHierThreads) hier_route_kernel(
    const T* __restrict__ Q, const float* __restrict__ S, int32_t* __restrict__ idx,
    int32_t* __restrict__ cnt, int Hq, int Hkv, int N, int B, int nq, int nfull, int M,
    int k_seg, int k_blk, int max_sel, float inv_sqrt_d) {
  extern __shared__ float sm_h[];
  float* qb = sm_h;              // [D]
  float* zb = qb + D;            // [nq] block scores
  float* zs = zb + nq;           // [nq / M + 1] segment scores
  __shared__ uint32_t hist[256];
  __shared__ int32_t kept[64];   // k_seg <= 64
  __shared__ int n_kept, n_pool;
  const int i = blockIdx.x % nq;
  const int bg = blockIdx.x / nq;
  const int b = bg / Hkv, g = bg - b * Hkv;
  const int G = Hq / Hkv;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int r0 = i * B, rows = min(B, N - r0);
  const int nc = min(i, nfull);              // complete blocks before i
  const int nclosed = nc / M;                // closed segments
  // 1. pooled query
  for (int c = t; c < D; c += kHierThreads) {
    float a = 0.f;
    for (int h = 0; h < G; ++h) {
      const T* qh = Q + (((size_t)b * Hq + g * G + h) * N + r0) * D + c;
      for (int r = 0; r < rows; ++r) a += tof(qh[(size_t)r * D]);
    }
    qb[c] = a / (float)(G * rows);
  }
  __syncthreads();
  // 2. block scores, one warp per block
  for (int jb = warp; jb < nc; jb += kHierThreads / 32) {
    const float* sj = S + ((size_t)bg * nfull + jb) * D;
    float a = 0.f;
    for (int c = lane; c < D; c += 32) a = fmaf(qb[c], sj[c], a);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == 0) zb[jb] = a * inv_sqrt_d;
  }
  __syncthreads();
  // 3. segment scores and the kept segments
  for (int m = t; m < nclosed; m += kHierThreads) {
    float a = 0.f;
    for (int e = 0; e < M; ++e) a += zb[m * M + e];
    // a segment holding only the sink block has no candidate
    zs[m] = (m == 0 && M == 1) ? -INFINITY : a / (float)M;
  }
  __syncthreads();
  if (warp == 0) {
    const int n_elig = nclosed - ((M == 1 && nclosed > 0) ? 1 : 0);
    const int ks = min(min(k_seg, n_elig), 64);
    const int nk = warp_select_topk(zs, nclosed, ks, 0, kept, hist);
    if (lane == 0) n_kept = nk;
  }
  __syncthreads();
  // 4. pool: candidates 1 .. i-1 in a kept segment or in no closed segment
  if (t == 0) n_pool = 0;
  __syncthreads();
  for (int jb = 1 + t; jb < i; jb += kHierThreads) {
    bool in_pool = jb >= nclosed * M || jb >= nc;
    if (!in_pool) {
      const int m = jb / M;
      for (int e = 0; e < n_kept; ++e) in_pool |= kept[e] == m;
    }
    if (jb < nc) {
      if (!in_pool) zb[jb] = -INFINITY;
      else atomicAdd(&n_pool, 1);
    }
  }
  __syncthreads();
  // 5. block selection and the ascending list {0} + R + {i}
  int32_t* row = idx + ((size_t)bg * nq + i) * max_sel;
  if (warp == 0) {
    const int ncand = max(nc - 1, 0);  // candidates 1 .. nc-1 (complete blocks before i)
    const int kb = min(k_blk, n_pool);
    int n_sel = 0;
    if (i > 0) {
      const int nr = warp_select_topk(zb + 1, ncand, kb, 1, row + 1, hist);
      __syncwarp();
      if (lane == 0) {
        row[0] = 0;
        row[1 + nr] = i;
      }
      n_sel = nr + 2;
    } else if (lane == 0) {
      row[0] = 0;
      n_sel = 1;
    }
    n_sel = __shfl_sync(0xffffffffu, n_sel, 0);
    for (int p = n_sel + lane; p < max_sel; p += 32) row[p] = -1;
    if (lane == 0) cnt[(size_t)bg * nq + i] = n_sel;
  }
}

cudaError_t launch_hier_route(const void* Q, ssa_dtype dt, const float* S, int batch, int Hq,
                              int Hkv, int N, int d, int B, int M, int k_seg, int k_blk,
                              int max_sel, int32_t* idx, int32_t* cnt, cudaStream_t st) {
  const int nq = (N + B - 1) / B, nfull = N / B;
  const size_t smem = sizeof(float) * ((size_t)d + nq + nq / M + 1);
  const unsigned grid = (unsigned)((long long)batch * Hkv * nq);
  const float isd = 1.0f / sqrtf((float)d);
  cudaError_t e = cudaSuccess;
#define SSA_HIER(TT, DD)                                                                       \
  e = cudaFuncSetAttribute(hier_route_kernel<TT, DD>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                           (int)smem);                                                        \
  if (e != cudaSuccess) return e;                                                             \
  hier_route_kernel<TT, DD><<<grid, kHierThreads, smem, st>>>(                                \
      (const TT*)Q, S, idx, cnt, Hq, Hkv, N, B, nq, nfull, M, k_seg, k_blk, max_sel, isd)
  if (dt == SSA_BF16) {
    if (d == 128) { SSA_HIER(__nv_bfloat16, 128); } else { SSA_HIER(__nv_bfloat16, 64); }
  } else {
    if (d == 128) { SSA_HIER(float, 128); } else { SSA_HIER(float, 64); }
  }
#undef SSA_HIER
  return cudaGetLastError();
}

}  // namespace ssa
