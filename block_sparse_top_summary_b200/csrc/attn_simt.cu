// Stage 2 on the CUDA cores: exact softmax attention over the selected blocks
// (SSA page, "2. Metodologia", sparse stream; DashAttention page, "Estágio 2").
//
// Serves fp32 inputs (where tensor-core tf32 would not meet fp32 accuracy) and
// the bf16 shapes the tensor-core kernel does not cover.  One CTA handles one
// query block of one query head: B rows, D/64 threads per row (each thread
// owns 64 of the d coordinates of its row's q and output).  Keys are visited
// in chunks of 32 staged in shared memory as fp32; logits are computed in the
// log2 domain (q pre-scaled by scale * log2(e)) with an online softmax.  The
// causal mask is applied only on the diagonal block; chunks entirely in the
// future of the block are skipped.
#include "common.cuh"
#include "kernels.h"

namespace ssa {

namespace {
constexpr int KC = 32;  // keys per shared-memory chunk
}

template <typename T, int D>
__global__ void __launch_bounds__(256) attn_simt_kernel(
    const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt,
    const float* __restrict__ bias, T* __restrict__ O, float* __restrict__ lse, int Hq, int Hkv,
    int N, int B, int nq, int max_sel, float scale_log2) {
  constexpr int TPR = D / 64;  // threads per row
  constexpr int EPC = Vec16<T>::n;
  constexpr int CPR = D / EPC;
  __shared__ __align__(16) float Ks[KC][D + 4];
  __shared__ __align__(16) float Vs[KC][D];

  const int i = nq - 1 - (int)blockIdx.x;  // later (longer) query blocks first
  const int bh = blockIdx.y;               // b * Hq + h
  const int b = bh / Hq;
  const int h = bh - b * Hq;
  const int g = h / (Hq / Hkv);
  const int t = threadIdx.x;
  const int r = t / TPR;
  const int part = t % TPR;
  const int nthreads = B * TPR;
  const int qpos = i * B + r;
  const bool row_ok = qpos < N;

  float q[64], o[64];
  {
    const T* qp = Q + ((int64_t)bh * N + (row_ok ? qpos : 0)) * D + part * 64;
#pragma unroll
    for (int c = 0; c < 64 / EPC; ++c) {
      float f[EPC];
      unpack16(ldg16(qp + c * EPC), f, (const T*)nullptr);
#pragma unroll
      for (int e = 0; e < EPC; ++e) q[c * EPC + e] = f[e] * scale_log2;
    }
#pragma unroll
    for (int e = 0; e < 64; ++e) o[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;

  const int64_t kvbase = (int64_t)(b * Hkv + g) * N;
  const int32_t* sel = idx + ((int64_t)(b * Hkv + g) * nq + i) * max_sel;
  const int ns = cnt[(int64_t)(b * Hkv + g) * nq + i];
  const int block_last_row = min(i * B + B, N) - 1;

  const float* brow = bias != nullptr ? bias + ((int64_t)(b * Hkv + g) * nq + i) * max_sel : nullptr;
  for (int s = 0; s < ns; ++s) {
    const int j = sel[s];
    // prior bias of the block (natural log), in the log2 domain of the logits
    const float bj = brow != nullptr ? brow[s] * 1.4426950408889634f : 0.f;
    for (int kc = 0; kc < B; kc += KC) {
      const int kb = j * B + kc;
      if (kb > block_last_row) break;  // the rest of this block is in every row's future
      __syncthreads();
      for (int c = t; c < KC * CPR; c += nthreads) {
        const int kk = c / CPR;
        const int cc = c - kk * CPR;
        float fk[EPC], fv[EPC];
        if (kb + kk < N && kc + kk < B) {
          unpack16(ldg16(K + (kvbase + kb + kk) * D + cc * EPC), fk, (const T*)nullptr);
          unpack16(ldg16(V + (kvbase + kb + kk) * D + cc * EPC), fv, (const T*)nullptr);
        } else {
#pragma unroll
          for (int e = 0; e < EPC; ++e) fk[e] = fv[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < EPC; ++e) {
          Ks[kk][cc * EPC + e] = fk[e];
          Vs[kk][cc * EPC + e] = fv[e];
        }
      }
      __syncthreads();
      float sc[KC];
      float cmax = -INFINITY;
#pragma unroll
      for (int kk = 0; kk < KC; ++kk) {
        const float* kr = &Ks[kk][part * 64];
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < 64; e += 4) {
          const float4 kv = *reinterpret_cast<const float4*>(kr + e);
          a = fmaf(q[e], kv.x, a);
          a = fmaf(q[e + 1], kv.y, a);
          a = fmaf(q[e + 2], kv.z, a);
          a = fmaf(q[e + 3], kv.w, a);
        }
        if (TPR == 2) a += __shfl_xor_sync(0xffffffffu, a, 1);
        // a chunk may reach past block j (B not a multiple of KC): those keys
        // belong to the next block, which this row did not select
        const int kpos = kb + kk;
        sc[kk] = (kpos <= qpos && kc + kk < B) ? a + bj : -INFINITY;
        cmax = fmaxf(cmax, sc[kk]);
      }
      const float mnew = fmaxf(m, cmax);
      if (mnew != -INFINITY) {
        const float alpha = exp2f(m - mnew);  // m = -inf gives 0
        l *= alpha;
#pragma unroll
        for (int e = 0; e < 64; ++e) o[e] *= alpha;
#pragma unroll
        for (int kk = 0; kk < KC; ++kk) {
          const float p = exp2f(sc[kk] - mnew);
          l += p;
          const float* vr = &Vs[kk][part * 64];
#pragma unroll
          for (int e = 0; e < 64; e += 4) {
            const float4 vv = *reinterpret_cast<const float4*>(vr + e);
            o[e] = fmaf(p, vv.x, o[e]);
            o[e + 1] = fmaf(p, vv.y, o[e + 1]);
            o[e + 2] = fmaf(p, vv.z, o[e + 2]);
            o[e + 3] = fmaf(p, vv.w, o[e + 3]);
          }
        }
        m = mnew;
      }
    }
  }

  if (row_ok) {
    const float inv = 1.0f / l;
    T* op = O + ((int64_t)bh * N + qpos) * D + part * 64;
#pragma unroll
    for (int e = 0; e < 64; ++e) store_out(op + e, o[e] * inv);
    if (lse != nullptr && part == 0)
      lse[(int64_t)bh * N + qpos] = (m + log2f(l)) * 0.69314718055994530942f;
  }
}

template <typename T, int D>
static cudaError_t launch_simt_t(const void* Q, const void* K, const void* V, const int32_t* idx,
                                 const int32_t* cnt, const float* bias, int batch, int Hq,
                                 int Hkv, int N, int B, int max_sel, float scale, void* O,
                                 float* lse, cudaStream_t st) {
  const int nq = (N + B - 1) / B;
  dim3 grid(nq, batch * Hq);
  const int threads = B * (D / 64);
  attn_simt_kernel<T, D><<<grid, threads, 0, st>>>(
      (const T*)Q, (const T*)K, (const T*)V, idx, cnt, bias, (T*)O, lse, Hq, Hkv, N, B, nq,
      max_sel, scale * 1.4426950408889634f);
  return cudaGetLastError();
}

cudaError_t launch_attn_simt(const void* Q, const void* K, const void* V, ssa_dtype dt,
                             const int32_t* idx, const int32_t* cnt, const float* bias, int batch,
                             int Hq, int Hkv, int N, int d, int B, int max_sel, float scale,
                             void* O, float* lse, cudaStream_t st) {
  if (dt == SSA_BF16) {
    return d == 128 ? launch_simt_t<__nv_bfloat16, 128>(Q, K, V, idx, cnt, bias, batch, Hq, Hkv, N, B,
                                                        max_sel, scale, O, lse, st)
                    : launch_simt_t<__nv_bfloat16, 64>(Q, K, V, idx, cnt, bias, batch, Hq, Hkv, N, B,
                                                       max_sel, scale, O, lse, st);
  }
  return d == 128 ? launch_simt_t<float, 128>(Q, K, V, idx, cnt, bias, batch, Hq, Hkv, N, B, max_sel,
                                              scale, O, lse, st)
                  : launch_simt_t<float, 64>(Q, K, V, idx, cnt, bias, batch, Hq, Hkv, N, B, max_sel,
                                             scale, O, lse, st);
}

}  // namespace ssa
