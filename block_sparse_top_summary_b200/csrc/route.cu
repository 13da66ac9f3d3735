// Stage 1: routing.  Each query block scores the summaries of the complete
// key blocks before it and keeps the top-k; sink block 0 and the diagonal are
// always added (DashAttention page, "Estágio 1" and "Estágio 2", diagonal
// branch; The Sparse Frontier page, RQ2, block-wise prefill selection; GSA
// page, "Componentes Principais" 3).  Query heads of one GQA group share the
// selection: their rows are pooled together (DashAttention page, "Estágio 1",
// GQA handling).
//
// One fused kernel, one CTA of 256 threads per (tile of 8 query blocks,
// batch x KV head):
//   1. pool: warp w streams query block w of the tile (G heads x B rows x d)
//      with coalesced 16-byte loads, 16 in flight per lane, into its fp32
//      mean qbar (the HBM-bound part);
//   2. score: every warp takes 4 candidate summaries at a time; lane l holds
//      d/32 coordinates of each summary and of the 8 qbar rows, so one
//      coalesced load feeds 8*d/32 FMAs (packed in pairs); the 32 partial dot products of a
//      warp step are reduced with a 31-shuffle butterfly that leaves dot
//      product l in lane l; scores land in shared memory (phases 1 and 2 are
//      route_tile::pool and route_tile::score);
//   3. select: warp w selects for query block w of the tile with an exact
//      radix select (ties to the lower index; long rows are first filtered
//      to the candidates at or above the least of the 32 lane maxima, see
//      warp_select_topk) and writes the ascending
//      block list, and, when the caller asks for them, the block's row of
//      scores (-inf where a block is not a candidate).
// Tiles are dispatched heaviest first (late query blocks have the most
// candidates).
#include "common.cuh"
#include "kernels.h"
#include "route_tile.cuh"

namespace ssa {

// Shared memory ahead of the score rows: qbar [TQ][D] while pooling and
// scoring, then the selection histograms [TQ][128] words.
template <int D, int TQ>
constexpr int route_head_words() {
  return TQ * (D > 128 ? D : 128);
}

template <typename T, int D, int TQ, int MINB>
__global__ void __launch_bounds__(256, MINB) route_kernel(const T* __restrict__ Q,
                                                    const float* __restrict__ S,
                                                    int32_t* __restrict__ idx,
                                                    int32_t* __restrict__ cnt,
                                                    float* __restrict__ scores, int Hq, int Hkv,
                                                    int N, int B, int nq, int nfull, int topk,
                                                    int max_sel, int ntiles, int sc_stride,
                                                    float inv_sqrt_d) {
  extern __shared__ __align__(16) float smem[];
  float* qbar = smem;                                             // [TQ][D]
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem);             // [TQ][128], after scoring
  float* sc = smem + route_head_words<D, TQ>();                   // [TQ][sc_stride]
  uint16_t* cand = reinterpret_cast<uint16_t*>(sc + TQ * sc_stride);  // [TQ][kSelCap]

  const int t = threadIdx.x;
  const int lane = t & 31;
  const int warp = t >> 5;
  const int bg = blockIdx.x;  // b * Hkv + g
  const int tile = ntiles - 1 - (int)blockIdx.y;
  const int G = Hq / Hkv;
  const int b = bg / Hkv;
  const int g = bg - b * Hkv;
  const int i0 = tile * TQ;
  const int i1 = min(i0 + TQ, nq);

  // ---- 1. pool Q over (rows of the block) x (heads of the group)
  route_tile::pool<T, D>(Q, qbar, b, g, G, Hq, N, B, i0, i1);

  // ---- 2. scores for candidates j = 1 .. i1-2 against all TQ rows
  const int ncand = max(i1 - 2, 0);
  route_tile::score<D, TQ>(qbar, S, sc, sc_stride, (int64_t)bg * nfull, 1, ncand, inv_sqrt_d);
  __syncthreads();

  // ---- 3. per query block: top-k, then {0} U R U {i} ascending, -1 padded
  {
    const int i = i0 + warp;
    if (i < i1) {
      int32_t* row = idx + ((int64_t)bg * nq + i) * max_sel;
      int n_sel = 1;  // block 0
      if (i >= 1) {
        const int m = warp_select_topk(sc + warp * sc_stride, i - 1, topk, 1, row + 1,
                                       hist + warp * 128, cand + warp * kSelCap);
        n_sel = m + 2;
        __syncwarp();
        if (lane == 0) row[m + 1] = i;
      }
      if (lane == 0) {
        row[0] = 0;
        cnt[(int64_t)bg * nq + i] = n_sel;
      }
      for (int p = n_sel + lane; p < max_sel; p += 32) row[p] = -1;
      if (scores != nullptr) {
        float* srow = scores + ((int64_t)bg * nq + i) * nfull;
        const float* mine = sc + warp * sc_stride;
        for (int j = lane; j < nfull; j += 32)
          srow[j] = (j >= 1 && j <= i - 1) ? mine[j - 1] : -INFINITY;
      }
    }
  }
}

template <typename T, int D, int TQ>
static cudaError_t launch_route_tq(const void* Q, const float* S, int batch, int Hq, int Hkv,
                                   int N, int B, int topk, int max_sel, int32_t* idx, int32_t* cnt,
                                   float* scores, cudaStream_t st) {
  const int nq = (N + B - 1) / B;
  const int nfull = N / B;
  const int ntiles = (nq + TQ - 1) / TQ;
  const int sc_stride = nq > 2 ? nq - 2 : 1;
  const size_t smem = sizeof(float) * ((size_t)route_head_words<D, TQ>() + (size_t)TQ * sc_stride) +
                      sizeof(uint16_t) * (size_t)TQ * kSelCap;
  // two CTAs per SM for tiles of 8 (at most 128 registers); the taller
  // score rows of 4- and 2-block tiles allow one CTA per SM anyway
  constexpr int MINB = TQ == 8 ? 2 : 1;
  cudaError_t e = cudaFuncSetAttribute(route_kernel<T, D, TQ, MINB>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(batch * Hkv, ntiles);
  route_kernel<T, D, TQ, MINB><<<grid, 256, smem, st>>>((const T*)Q, S, idx, cnt, scores, Hq, Hkv, N, B,
                                                  nq, nfull, topk, max_sel, ntiles, sc_stride,
                                                  1.0f / sqrtf((float)D));
  return cudaGetLastError();
}

// Tiles of 8 query blocks while their score rows fit in shared memory, else
// 4 or 2 (the warps past the tile idle in the pooling and selection phases).
template <typename T, int D>
static cudaError_t launch_route_t(const void* Q, const float* S, int batch, int Hq, int Hkv, int N,
                                  int B, int topk, int max_sel, int32_t* idx, int32_t* cnt,
                                  float* scores, cudaStream_t st) {
  const int nq = (N + B - 1) / B;
  const size_t row = sizeof(float) * ((size_t)(D > 128 ? D : 128) + (size_t)(nq > 2 ? nq - 2 : 1)) +
                     sizeof(uint16_t) * kSelCap;
  const size_t limit = (size_t)220 * 1024;
  if (8 * row <= limit)
    return launch_route_tq<T, D, 8>(Q, S, batch, Hq, Hkv, N, B, topk, max_sel, idx, cnt, scores, st);
  if (4 * row <= limit)
    return launch_route_tq<T, D, 4>(Q, S, batch, Hq, Hkv, N, B, topk, max_sel, idx, cnt, scores, st);
  return launch_route_tq<T, D, 2>(Q, S, batch, Hq, Hkv, N, B, topk, max_sel, idx, cnt, scores, st);
}

cudaError_t launch_route(const void* Q, ssa_dtype dt, const float* S, int batch, int Hq, int Hkv,
                         int N, int d, int B, int topk, int max_sel, int32_t* idx, int32_t* cnt,
                         float* scores, cudaStream_t st) {
  if (dt == SSA_BF16) {
    return d == 128 ? launch_route_t<__nv_bfloat16, 128>(Q, S, batch, Hq, Hkv, N, B, topk, max_sel,
                                                         idx, cnt, scores, st)
                    : launch_route_t<__nv_bfloat16, 64>(Q, S, batch, Hq, Hkv, N, B, topk, max_sel,
                                                        idx, cnt, scores, st);
  }
  return d == 128 ? launch_route_t<float, 128>(Q, S, batch, Hq, Hkv, N, B, topk, max_sel, idx, cnt,
                                               scores, st)
                  : launch_route_t<float, 64>(Q, S, batch, Hq, Hkv, N, B, topk, max_sel, idx, cnt,
                                              scores, st);
}

}  // namespace ssa
