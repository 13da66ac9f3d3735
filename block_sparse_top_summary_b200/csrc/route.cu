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
//      coalesced load feeds 8*d/32 FMAs; the 32 partial dot products of a
//      warp step are reduced with a 31-shuffle butterfly that leaves dot
//      product l in lane l; scores land in shared memory;
//   3. select: warp w selects for query block w of the tile with an exact
//      4-pass radix select (ties to the lower index) and writes the ascending
//      block list, and, when the caller asks for them, the block's row of
//      scores (-inf where a block is not a candidate).
// Tiles are dispatched heaviest first (late query blocks have the most
// candidates).
#include "common.cuh"
#include "kernels.h"

namespace ssa {

namespace {

constexpr int TQ = 8;  // query blocks per CTA (= warps per CTA)

// Butterfly reduction of 32 per-lane values: afterwards lane l's v[0] holds
// the warp-wide sum of value index l.
__device__ __forceinline__ float reduce32_transpose(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int half = 16; half >= 1; half >>= 1) {
    const bool upper = (lane & half) != 0;
#pragma unroll
    for (int k = 0; k < half; ++k) {
      const float send = upper ? v[k] : v[k + half];
      const float keep = upper ? v[k + half] : v[k];
      v[k] = keep + __shfl_xor_sync(0xffffffffu, send, half);
    }
  }
  return v[0];
}

}  // namespace

template <typename T, int D>
__global__ void __launch_bounds__(256) route_kernel(const T* __restrict__ Q,
                                                    const float* __restrict__ S,
                                                    int32_t* __restrict__ idx,
                                                    int32_t* __restrict__ cnt,
                                                    float* __restrict__ scores, int Hq, int Hkv,
                                                    int N, int B, int nq, int nfull, int topk,
                                                    int max_sel, int ntiles, int sc_stride,
                                                    float inv_sqrt_d) {
  constexpr int EPC = Vec16<T>::n;
  constexpr int CPR = D / EPC;
  constexpr int SL = D / 32;  // summary coordinates per lane
  extern __shared__ __align__(16) float smem[];
  float* qbar = smem;                                        // [TQ][D]
  uint32_t* hist = reinterpret_cast<uint32_t*>(qbar + TQ * D);  // [TQ][256]
  float* sc = reinterpret_cast<float*>(hist + TQ * 256);     // [TQ][sc_stride]

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

  // ---- 1. pool Q over (rows of the block) x (heads of the group): warp w
  // pools query block i0 + w.  A warp load covers RPW whole rows (16-byte
  // chunk cc of row rs); 16 loads are in flight per lane; rows meet by
  // xor-shuffles at the end, so this phase needs no block barrier.
  {
    constexpr int LPR = CPR < 32 ? CPR : 32;  // lanes per row
    constexpr int RPW = 32 / LPR;             // rows per warp load
    constexpr int U = 16;                     // loads in flight per lane
    const int qi = i0 + warp;
    if (qi < i1) {
      const int rows = min(B, N - qi * B);
      const int R = G * rows;
      const int cc = lane % LPR;
      const int rs = lane / LPR;
      float acc[EPC];
#pragma unroll
      for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
      const T* blk = Q + ((int64_t)(b * Hq + g * G) * N + (int64_t)qi * B) * D + cc * EPC;
      for (int r0 = rs; r0 < R; r0 += RPW * U) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int r = r0 + u * RPW;
          if (r < R) {
            const int h = r / rows;
            v[u] = ldg16_stream(blk + ((int64_t)h * N + (r - h * rows)) * D);
          } else {
            v[u] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          float f[EPC];
          unpack16(v[u], f, (const T*)nullptr);
#pragma unroll
          for (int e = 0; e < EPC; ++e) acc[e] += f[e];
        }
      }
#pragma unroll
      for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
        for (int e = 0; e < EPC; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
      if (rs == 0) {
        const float inv = 1.0f / (float)R;
#pragma unroll
        for (int e = 0; e < EPC; ++e) qbar[warp * D + cc * EPC + e] = acc[e] * inv;
      }
    }
    // CPR > 32 (fp32, d = 128 has CPR = 32): one row per warp load covers d
    static_assert(CPR <= 32, "a row must fit one warp load");
    __syncthreads();
  }

  // ---- 2. scores for candidates j = 1 .. i1-2 against all TQ rows
  const int ncand = max(i1 - 2, 0);
  {
    float qs[TQ][SL];
#pragma unroll
    for (int q = 0; q < TQ; ++q)
#pragma unroll
      for (int e = 0; e < SL; ++e) qs[q][e] = qbar[q * D + lane * SL + e];
    const float* Sg = S + (int64_t)bg * nfull * D + lane * SL;
    // the summary rows of a warp step are loaded one step ahead
    auto load_rows = [&](int j0, float (&sv)[4][SL]) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int j = min(j0 + c, ncand);
        if (SL == 4) {
          const float4 x = __ldg(reinterpret_cast<const float4*>(Sg + (int64_t)j * D));
          sv[c][0] = x.x; sv[c][1] = x.y; sv[c][2 % SL] = x.z; sv[c][3 % SL] = x.w;
        } else {
          const float2 x = __ldg(reinterpret_cast<const float2*>(Sg + (int64_t)j * D));
          sv[c][0] = x.x; sv[c][1 % SL] = x.y;
        }
      }
    };
    constexpr int kStep = 4 * (256 / 32);
    float sv[4][SL];
    if (1 + warp * 4 <= ncand) load_rows(1 + warp * 4, sv);
    for (int j0 = 1 + warp * 4; j0 <= ncand; j0 += kStep) {
      float sn[4][SL];
      if (j0 + kStep <= ncand) load_rows(j0 + kStep, sn);
      float v[32];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int q = 0; q < TQ; ++q) {
          float a = 0.f;
#pragma unroll
          for (int e = 0; e < SL; ++e) a = fmaf(sv[c][e], qs[q][e], a);
          v[c * TQ + q] = a;
        }
      const float dot = reduce32_transpose(v);
      const int c = lane / TQ;
      const int q = lane % TQ;
      const int j = j0 + c;
      if (j <= ncand) sc[q * sc_stride + (j - 1)] = dot * inv_sqrt_d;
#pragma unroll
      for (int c2 = 0; c2 < 4; ++c2)
#pragma unroll
        for (int e = 0; e < SL; ++e) sv[c2][e] = sn[c2][e];
    }
  }
  __syncthreads();

  // ---- 3. per query block: top-k, then {0} U R U {i} ascending, -1 padded
  {
    const int i = i0 + warp;
    if (i < i1) {
      int32_t* row = idx + ((int64_t)bg * nq + i) * max_sel;
      int n_sel = 1;  // block 0
      if (i >= 1) {
        const int m = warp_select_topk(sc + warp * sc_stride, i - 1, topk, 1, row + 1,
                                       hist + warp * 256);
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

template <typename T, int D>
static cudaError_t launch_route_t(const void* Q, const float* S, int batch, int Hq, int Hkv, int N,
                                  int B, int topk, int max_sel, int32_t* idx, int32_t* cnt,
                                  float* scores, cudaStream_t st) {
  const int nq = (N + B - 1) / B;
  const int nfull = N / B;
  const int ntiles = (nq + TQ - 1) / TQ;
  const int sc_stride = nq > 2 ? nq - 2 : 1;
  const size_t smem = sizeof(float) * ((size_t)TQ * D + (size_t)TQ * 256 + (size_t)TQ * sc_stride);
  cudaError_t e = cudaFuncSetAttribute(route_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(batch * Hkv, ntiles);
  route_kernel<T, D><<<grid, 256, smem, st>>>((const T*)Q, S, idx, cnt, scores, Hq, Hkv, N, B,
                                              nq, nfull,
                                              topk, max_sel, ntiles, sc_stride,
                                              1.0f / sqrtf((float)D));
  return cudaGetLastError();
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
