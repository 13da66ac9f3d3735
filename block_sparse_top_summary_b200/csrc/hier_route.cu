// Two-level routing (segments of M blocks, then blocks), one CTA of 256
// threads per (tile of 8 query blocks, batch x KV head g), warp w taking query
// block i = i0 + w:
//   1. qbar = mean of Q over the block's rows and the group's heads, and
//   2. block scores z_j = qbar . S_j / sqrt(d) for the complete blocks j < i,
//      as in the flat routing kernel (route_tile::pool and route_tile::score:
//      the scores are bitwise those of ssa_route);
//   3. segment scores = the mean of their blocks' scores (= qbar . mean
//      summary, by linearity) for the closed segments ((m + 1) M <= i); the
//      warp keeps the top k_seg of those holding a candidate (ties to the
//      lower index);
//   4. candidates 1 .. i-1 outside the kept and the open segments get -inf;
//      the warp keeps the top min(k_blk, pool size) of the rest;
//   5. selection = {0} + kept blocks + {i}, ascending.
// Dynamic shared memory: qbar [8][d], histograms [8][128] words, block scores
// [8][nfull], segment scores [8][nfull / M + 1], kept segments [8][64].
#include "common.cuh"
#include "kernels.h"
#include "route_tile.cuh"

namespace ssa {

using route_tile::TQ;

template <typename T, int D>
__global__ void __launch_bounds__(route_tile::kThreads) hier_route_kernel(
    const T* __restrict__ Q, const float* __restrict__ S, int32_t* __restrict__ idx,
    int32_t* __restrict__ cnt, int Hq, int Hkv, int N, int B, int nq, int nfull, int M,
    int k_seg, int k_blk, int max_sel, int ntiles, int sc_stride, int zs_stride,
    float inv_sqrt_d) {
  extern __shared__ __align__(16) float sm_h[];
  float* qbar = sm_h;                                              // [TQ][D]
  uint32_t* hist = reinterpret_cast<uint32_t*>(qbar + TQ * D);     // [TQ][128]
  float* sc = reinterpret_cast<float*>(hist + TQ * 128);           // [TQ][sc_stride]
  float* zsa = sc + TQ * sc_stride;                                // [TQ][zs_stride]
  int32_t* kepta = reinterpret_cast<int32_t*>(zsa + TQ * zs_stride);  // [TQ][64]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int bg = blockIdx.x;
  const int tile = ntiles - 1 - (int)blockIdx.y;  // late (heavy) tiles first
  const int b = bg / Hkv, g = bg - b * Hkv;
  const int G = Hq / Hkv;
  const int i0 = tile * TQ, i1 = min(i0 + TQ, nq);
  // 1-2. pooled queries and the scores of blocks 0 .. min(i1 - 1, nfull) - 1
  route_tile::pool<T, D>(Q, qbar, b, g, G, Hq, N, B, i0, i1);
  const int nc_tile = min(i1 - 1, nfull);
  route_tile::score<D>(qbar, S, sc, sc_stride, (int64_t)bg * nfull, 0, nc_tile - 1, inv_sqrt_d);
  __syncthreads();
  const int i = i0 + warp;
  if (i >= i1) return;
  float* zb = sc + warp * sc_stride;
  float* zs = zsa + warp * zs_stride;
  int32_t* kept = kepta + warp * 64;
  uint32_t* hw = hist + warp * 128;
  const int nc = min(i, nfull);   // complete blocks before i
  const int nclosed = nc / M;     // closed segments
  // 3. segment scores and the kept segments
  for (int m = lane; m < nclosed; m += 32) {
    float a = 0.f;
    for (int e = 0; e < M; ++e) a += zb[m * M + e];
    // a segment holding only the sink block has no candidate
    zs[m] = (m == 0 && M == 1) ? -INFINITY : a / (float)M;
  }
  __syncwarp();
  const int n_elig = nclosed - ((M == 1 && nclosed > 0) ? 1 : 0);
  const int ks = min(min(k_seg, n_elig), 64);
  const int n_kept = warp_select_topk(zs, nclosed, ks, 0, kept, hw);
  __syncwarp();
  // 4. pool: candidates 1 .. i-1 in a kept segment or in no closed segment
  int n_pool = 0;
  for (int jb0 = 1; jb0 < i; jb0 += 32) {
    const int jb = jb0 + lane;
    bool in_pool = jb >= nclosed * M || jb >= nc;
    if (!in_pool && jb < i) {
      const int m = jb / M;
      for (int e = 0; e < n_kept; ++e) in_pool |= kept[e] == m;
    }
    const bool cand = jb < i && jb < nc;
    if (cand && !in_pool) zb[jb] = -INFINITY;
    n_pool += __popc(__ballot_sync(0xffffffffu, cand && in_pool));
  }
  __syncwarp();
  // 5. block selection and the ascending list {0} + R + {i}
  int32_t* row = idx + ((size_t)bg * nq + i) * max_sel;
  const int ncand = max(nc - 1, 0);  // candidates 1 .. nc-1 (complete blocks before i)
  const int kb = min(k_blk, n_pool);
  int n_sel = 1;
  if (i > 0) {
    const int nr = warp_select_topk(zb + 1, ncand, kb, 1, row + 1, hw);
    __syncwarp();
    if (lane == 0) row[1 + nr] = i;
    n_sel = nr + 2;
  }
  if (lane == 0) {
    row[0] = 0;
    cnt[(size_t)bg * nq + i] = n_sel;
  }
  for (int p = n_sel + lane; p < max_sel; p += 32) row[p] = -1;
}

namespace {
constexpr int kHierThreads = 256;
__device__ __forceinline__ float tof(float v) { return v; }
__device__ __forceinline__ float tof(__nv_bfloat16 v) { return __bfloat162float(v); }
}  // namespace

// The same selection for one query block per CTA, for sizes whose tile of
// score rows does not fit shared memory: dynamic shared memory qbar [d],
// block scores [nq], segment scores [nq / M + 1].  The pooled query and the
// scores are summed in another order than the tiled kernel's (so a near-tie
// may resolve differently).
template <typename T, int D>
__global__ void __launch_bounds__(kHierThreads) hier_route_row_kernel(
    const T* __restrict__ Q, const float* __restrict__ S, int32_t* __restrict__ idx,
    int32_t* __restrict__ cnt, int Hq, int Hkv, int N, int B, int nq, int nfull, int M,
    int k_seg, int k_blk, int max_sel, float inv_sqrt_d) {
  extern __shared__ float sm_h[];
  float* qb = sm_h;              // [D]
  float* zb = qb + D;            // [nq] block scores
  float* zs = zb + nq;           // [nq / M + 1] segment scores
  __shared__ uint32_t hist[128];
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
  const int ntiles = (nq + TQ - 1) / TQ;
  const int sc_stride = nfull > 0 ? nfull : 1;
  const int zs_stride = nfull / M + 1;
  const size_t smem = sizeof(float) * ((size_t)TQ * d + (size_t)TQ * 128 +
                                       (size_t)TQ * sc_stride + (size_t)TQ * zs_stride +
                                       (size_t)TQ * 64);
  const dim3 grid((unsigned)(batch * Hkv), (unsigned)ntiles);
  const float isd = 1.0f / sqrtf((float)d);
  cudaError_t e = cudaSuccess;
  if (smem <= (size_t)200 * 1024) {
#define SSA_HIER(TT, DD)                                                                       \
  e = cudaFuncSetAttribute(hier_route_kernel<TT, DD>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                           (int)smem);                                                        \
  if (e != cudaSuccess) return e;                                                             \
  hier_route_kernel<TT, DD><<<grid, route_tile::kThreads, smem, st>>>(                        \
      (const TT*)Q, S, idx, cnt, Hq, Hkv, N, B, nq, nfull, M, k_seg, k_blk, max_sel, ntiles,  \
      sc_stride, zs_stride, isd)
    if (dt == SSA_BF16) {
      if (d == 128) { SSA_HIER(__nv_bfloat16, 128); } else { SSA_HIER(__nv_bfloat16, 64); }
    } else {
      if (d == 128) { SSA_HIER(float, 128); } else { SSA_HIER(float, 64); }
    }
#undef SSA_HIER
    return cudaGetLastError();
  }
  const size_t smem_row = sizeof(float) * ((size_t)d + nq + nq / M + 1);
  const unsigned grid_row = (unsigned)((long long)batch * Hkv * nq);
#define SSA_HIER_ROW(TT, DD)                                                                    \
  e = cudaFuncSetAttribute(hier_route_row_kernel<TT, DD>,                                      \
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_row);        \
  if (e != cudaSuccess) return e;                                                              \
  hier_route_row_kernel<TT, DD><<<grid_row, kHierThreads, smem_row, st>>>(                     \
      (const TT*)Q, S, idx, cnt, Hq, Hkv, N, B, nq, nfull, M, k_seg, k_blk, max_sel, isd)
  if (dt == SSA_BF16) {
    if (d == 128) { SSA_HIER_ROW(__nv_bfloat16, 128); } else { SSA_HIER_ROW(__nv_bfloat16, 64); }
  } else {
    if (d == 128) { SSA_HIER_ROW(float, 128); } else { SSA_HIER_ROW(float, 64); }
  }
#undef SSA_HIER_ROW
  return cudaGetLastError();
}

}  // namespace ssa
