// Phases shared by the routing kernels that take query blocks in tiles of
// TQ (8, or 4 or 2 for long sequences; one warp each), 256 threads per CTA:
// pooling the tile's query blocks, and scoring a range of block summaries
// against all of them.
#pragma once

#include "common.cuh"

namespace ssa {
namespace route_tile {

constexpr int TQ = 8;         // query blocks per CTA (= warps per CTA) unless stated
constexpr int kThreads = 256;

// Butterfly reduction of 32 per-lane values held in lane-permuted order:
// lane l keeps value index m in v[m ^ l].  At each level a lane keeps the
// lower half of its live values and sends the upper half to its partner, so
// no lane-dependent selects are needed; afterwards lane l's v[0] holds the
// warp-wide sum of value index l.
__device__ __forceinline__ float reduce32_permuted(float (&v)[32]) {
#pragma unroll
  for (int half = 16; half >= 1; half >>= 1)
#pragma unroll
    for (int k = 0; k < half; ++k) v[k] += __shfl_xor_sync(0xffffffffu, v[k + half], half);
  return v[0];
}

// qbar[w] = mean of Q over the rows of query block i0 + w and the G heads of
// KV head g, for the tile's query blocks [i0, i1).  Warp w pools query block
// i0 + w: a warp load covers RPW whole rows (16-byte chunk cc of row rs), 16
// loads are in flight per lane, and rows meet by xor-shuffles at the end, so
// no block barrier is needed inside.  Ends with a block barrier.
template <typename T, int D>
__device__ __forceinline__ void pool(const T* __restrict__ Q, float* qbar, int b, int g, int G,
                                     int Hq, int N, int B, int i0, int i1) {
  constexpr int EPC = Vec16<T>::n;
  constexpr int CPR = D / EPC;
  constexpr int LPR = CPR < 32 ? CPR : 32;  // lanes per row
  constexpr int RPW = 32 / LPR;             // rows per warp load
  constexpr int U = 16;                     // loads in flight per lane
  static_assert(CPR <= 32, "a row must fit one warp load");
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
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
  __syncthreads();
}

// sc[q * stride + (j - jlo)] = qbar[q] . S[bg, j] * inv_sqrt_d for j in
// [jlo, jhi] and every row q < NQ of the tile.  Every warp takes CW = 32 / NQ
// summaries at a time; lane l holds d/32 coordinates of each summary and of
// the NQ qbar rows, so one coalesced load feeds NQ*d/32 FMAs, issued two at a
// time on packed fp32 pairs (two qbar rows against one summary coordinate).
// The 32 partial dot products of a warp step are reduced with a 31-shuffle
// butterfly that leaves dot product l in lane l.  Lane l = cx*NQ + qx keeps
// summary c ^ cx in slot c and qbar row q ^ qx in slot q, so that slot pair
// (c, q) lands at position c*NQ + q = m ^ l of the butterfly's input, m the
// product's index (reduce32_permuted).  The summary rows of a step are loaded
// one step ahead.  No barrier inside; the caller synchronises before reading
// sc.
template <int D, int NQ = TQ>
__device__ __forceinline__ void score(const float* qbar, const float* __restrict__ S, float* sc,
                                      int stride, int64_t srow0, int jlo, int jhi,
                                      float inv_sqrt_d) {
  constexpr int SL = D / 32;  // summary coordinates per lane
  constexpr int CW = 32 / NQ; // summaries per warp step
  static_assert(NQ >= 2 && (NQ & (NQ - 1)) == 0 && NQ <= 32, "NQ: a power of two, 2 .. 32");
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int cx = lane / NQ;
  const int qx = lane % NQ;
  // qbar rows in pairs of slots (2p, 2p + 1), one packed register per coordinate
  uint64_t qs[NQ / 2][SL];
#pragma unroll
  for (int p = 0; p < NQ / 2; ++p)
#pragma unroll
    for (int e = 0; e < SL; ++e)
      qs[p][e] = f32x2(qbar[((2 * p) ^ qx) * D + lane * SL + e],
                       qbar[((2 * p + 1) ^ qx) * D + lane * SL + e]);
  const float* Sg = S + srow0 * D + lane * SL;
  auto load_rows = [&](int j0, float (&sv)[CW][SL]) {
#pragma unroll
    for (int c = 0; c < CW; ++c) {
      const int j = min(j0 + (c ^ cx), jhi);
      if (SL == 4) {
        const float4 x = __ldg(reinterpret_cast<const float4*>(Sg + (int64_t)j * D));
        sv[c][0] = x.x; sv[c][1] = x.y; sv[c][2 % SL] = x.z; sv[c][3 % SL] = x.w;
      } else {
        const float2 x = __ldg(reinterpret_cast<const float2*>(Sg + (int64_t)j * D));
        sv[c][0] = x.x; sv[c][1 % SL] = x.y;
      }
    }
  };
  constexpr int kStep = CW * (kThreads / 32);
  float sv[CW][SL];
  if (jlo + warp * CW <= jhi) load_rows(jlo + warp * CW, sv);
  for (int j0 = jlo + warp * CW; j0 <= jhi; j0 += kStep) {
    float sn[CW][SL];
    if (j0 + kStep <= jhi) load_rows(j0 + kStep, sn);
    float v[32];
#pragma unroll
    for (int c = 0; c < CW; ++c)
#pragma unroll
      for (int p = 0; p < NQ / 2; ++p) {
        uint64_t a = 0;
#pragma unroll
        for (int e = 0; e < SL; ++e) {
          const uint64_t x = f32x2(sv[c][e], sv[c][e]);
          asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(a) : "l"(x), "l"(qs[p][e]));
        }
        v[c * NQ + 2 * p] = __uint_as_float((uint32_t)a);
        v[c * NQ + 2 * p + 1] = __uint_as_float((uint32_t)(a >> 32));
      }
    const float dot = reduce32_permuted(v);
    const int c = lane / NQ;
    const int q = lane % NQ;
    const int j = j0 + c;
    if (j <= jhi) sc[q * stride + (j - jlo)] = dot * inv_sqrt_d;
#pragma unroll
    for (int c2 = 0; c2 < CW; ++c2)
#pragma unroll
      for (int e = 0; e < SL; ++e) sv[c2][e] = sn[c2][e];
  }
}

}  // namespace route_tile
}  // namespace ssa
