// Stage 0: block summaries, the mean key of every complete block of B keys
// (DashAttention page, "Estágio 0", uniform mean pooling; GSA page,
// "Componentes Principais" 2, MoBA's mean pooling).
//
// HBM-bound streaming reduction, one warp per block (B x d contiguous
// elements) in a grid-stride loop over blocks.  Lane l owns the 16-byte column
// chunk l % LPR of every (l / LPR)-th row, so each warp load is one fully
// used, coalesced 512-byte request; 8 loads are in flight per lane, and the
// row partials meet by xor-shuffles -- no block barrier, so every warp's
// loads are issued at once.  The d fp32 means are written by the lanes of
// row 0 with coalesced stores.
#include "common.cuh"
#include "kernels.h"

namespace ssa {

template <typename T, int D>
__global__ void __launch_bounds__(256) block_summary_kernel(const T* __restrict__ K,
                                                            float* __restrict__ S,
                                                            int64_t n_units, int nfull, int N,
                                                            int B) {
  constexpr int EPC = Vec16<T>::n;          // elements per 16-byte chunk
  constexpr int CPR = D / EPC;              // chunks per row
  constexpr int LPR = CPR < 32 ? CPR : 32;  // lanes per row
  constexpr int RPW = 32 / LPR;             // rows per warp load
  constexpr int U = 8;                      // loads in flight per lane
  static_assert(CPR <= 32, "a row must fit one warp load");
  const int lane = threadIdx.x & 31;
  const int cc = lane % LPR;
  const int rs = lane / LPR;
  const float inv_b = 1.0f / (float)B;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t u = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); u < n_units;
       u += nwarps) {
    const int64_t head = u / nfull;  // (b * Hkv + g)
    const int j = (int)(u - head * nfull);
    const T* base = K + (head * (int64_t)N + (int64_t)j * B) * D + cc * EPC;
    float acc[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
    for (int r0 = rs; r0 < B; r0 += RPW * U) {
      // rows past the block are clamped into it (so all U loads issue
      // unconditionally) and left out of the sum
      uint4 v[U];
#pragma unroll
      for (int q = 0; q < U; ++q)
        v[q] = ldg16_stream(base + (int64_t)min(r0 + q * RPW, B - 1) * D);
#pragma unroll
      for (int q = 0; q < U; ++q) {
        if (r0 + q * RPW < B) {
          float f[EPC];
          unpack16(v[q], f, (const T*)nullptr);
#pragma unroll
          for (int e = 0; e < EPC; ++e) acc[e] += f[e];
        }
      }
    }
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < EPC; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    if (rs == 0) {
      float4* dst = reinterpret_cast<float4*>(S + u * D + cc * EPC);
#pragma unroll
      for (int e = 0; e < EPC; e += 4)
        dst[e / 4] = make_float4(acc[e] * inv_b, acc[e + 1] * inv_b, acc[e + 2] * inv_b,
                                 acc[e + 3] * inv_b);
    }
  }
}

template <typename T, int D>
static cudaError_t launch_summary_t(const void* K, float* S, int batch, int Hkv, int N, int B,
                                    cudaStream_t st) {
  const int nfull = N / B;
  const int64_t units = (int64_t)batch * Hkv * nfull;
  if (units == 0) return cudaSuccess;
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, block_summary_kernel<T, D>, 256, 0);
  // one warp per block while the blocks fit in one wave, else a grid-stride
  // loop over one full wave
  const int64_t cap = (int64_t)sms * (per_sm > 0 ? per_sm : 1);
  const int64_t want = (units + 7) / 8;
  const int grid = (int)(want < cap ? want : cap);
  block_summary_kernel<T, D><<<grid, 256, 0, st>>>((const T*)K, S, units, nfull, N, B);
  return cudaGetLastError();
}

cudaError_t launch_block_summary(const void* K, ssa_dtype dt, int batch, int Hkv, int N, int d,
                                 int B, float* S, cudaStream_t st) {
  if (dt == SSA_BF16) {
    return d == 128 ? launch_summary_t<__nv_bfloat16, 128>(K, S, batch, Hkv, N, B, st)
                    : launch_summary_t<__nv_bfloat16, 64>(K, S, batch, Hkv, N, B, st);
  }
  return d == 128 ? launch_summary_t<float, 128>(K, S, batch, Hkv, N, B, st)
                  : launch_summary_t<float, 64>(K, S, batch, Hkv, N, B, st);
}

}  // namespace ssa
