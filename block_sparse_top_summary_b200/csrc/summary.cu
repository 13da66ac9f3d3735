// Stage 0: block summaries, the mean key of every complete block of B keys
// (DashAttention page, "Estágio 0", uniform mean pooling; GSA page,
// "Componentes Principais" 2, MoBA's mean pooling).
//
// HBM-bound streaming reduction.  One CTA of 256 threads reduces one block
// (B x d contiguous elements) at a time in a grid-stride loop over blocks.
// Thread t owns the 16-byte column chunk t % CPR and the rows t / CPR + m * RL,
// so every warp load is a fully used, coalesced 512-byte request.  Partial sums
// meet in shared memory; the d fp32 means are written with one coalesced store.
#include "common.cuh"
#include "kernels.h"

namespace ssa {

template <typename T, int D>
__global__ void __launch_bounds__(256) block_summary_kernel(const T* __restrict__ K,
                                                            float* __restrict__ S,
                                                            int64_t n_units, int nfull, int N,
                                                            int B) {
  constexpr int EPC = Vec16<T>::n;  // elements per 16-byte chunk
  constexpr int CPR = D / EPC;      // chunks per row
  constexpr int RL = 256 / CPR;     // row lanes
  __shared__ float red[RL][D];
  const int t = threadIdx.x;
  const int cc = t % CPR;
  const int rl = t / CPR;
  const float inv_b = 1.0f / (float)B;
  for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x) {
    const int64_t head = u / nfull;  // (b * Hkv + g)
    const int j = (int)(u - head * nfull);
    const T* base = K + (head * (int64_t)N + (int64_t)j * B) * D + cc * EPC;
    float acc[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
    // B / RL rows per thread; unrolled by 4 so several loads are in flight.
    int r = rl;
    for (; r + 3 * RL < B; r += 4 * RL) {
      uint4 v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) v[q] = ldg16_stream(base + (int64_t)(r + q * RL) * D);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float f[EPC];
        unpack16(v[q], f, (const T*)nullptr);
#pragma unroll
        for (int e = 0; e < EPC; ++e) acc[e] += f[e];
      }
    }
    for (; r < B; r += RL) {
      float f[EPC];
      unpack16(ldg16_stream(base + (int64_t)r * D), f, (const T*)nullptr);
#pragma unroll
      for (int e = 0; e < EPC; ++e) acc[e] += f[e];
    }
#pragma unroll
    for (int e = 0; e < EPC; ++e) red[rl][cc * EPC + e] = acc[e];
    __syncthreads();
    if (t < D) {
      float s = 0.f;
#pragma unroll 8
      for (int q = 0; q < RL; ++q) s += red[q][t];
      S[u * D + t] = s * inv_b;
    }
    __syncthreads();
  }
}

template <typename T, int D>
static cudaError_t launch_summary_t(const void* K, float* S, int batch, int Hkv, int N, int B,
                                    cudaStream_t st) {
  const int nfull = N / B;
  const int64_t units = (int64_t)batch * Hkv * nfull;
  if (units == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t cap = (int64_t)sms * 8;
  const int grid = (int)(units < cap ? units : cap);
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
