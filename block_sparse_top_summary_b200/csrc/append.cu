// Incremental decoding: append one token per sequence to the KV cache and keep
// the cache's block summaries current (DashAttention page, "Contribuições
// Principais" 4, incremental decoding; "Estágio 0", a block's summary is the
// mean of its keys, formed once the block is complete).
//
// One CTA of kAppendThreads threads per sequence, all its KV heads at once.  For a
// sequence holding L tokens (0 <= L < Lmax) every head's new key and value row
// is stored at position L with 16-byte copies, one chunk per thread.  If L + 1
// is a multiple of B, block (L+1)/B - 1 has just become complete: after a
// barrier (the CTA has just stored one of its rows) the threads take (head,
// 16-byte column chunk) pairs, TP threads per pair splitting the block's rows,
// read the rows back through L2, reduce the shares with xor-shuffles and store
// the mean.  The CTA alone owns its sequence's length, which it raises to
// L + 1 last.
#include "common.cuh"
#include "kernels.h"

namespace ssa {

namespace {
constexpr int kAppendThreads = 1024;
}  // namespace

template <typename T, int D>
__global__ void __launch_bounds__(kAppendThreads) decode_append_kernel(
    T* __restrict__ Kc, T* __restrict__ Vc, float* __restrict__ S, int32_t* __restrict__ seqlens,
    const T* __restrict__ k_new, const T* __restrict__ v_new, int Hkv, int Lmax, int B,
    int nfull, CacheMap pm) {
  constexpr int EPC = Vec16<T>::n;  // elements per 16-byte chunk
  constexpr int CPR = D / EPC;      // chunks per row
  const int b = blockIdx.x;
  const int t = threadIdx.x;
  // Thread 0 reads the length once and shares it: thread 0 raises seqlens[b]
  // at the end, and a warp that read it directly after that store would take
  // the new length for the old one.
  __shared__ int s_len;
  if (t == 0) s_len = seqlens[b];
  __syncthreads();
  const int L = s_len;
  if (L < 0 || L >= Lmax) return;  // full cache or invalid length: nothing changes
  // Paged cache: the page of the block that receives the row.  Every thread
  // reads the same table word, so the CTA takes one path.
  int page = -1;
  if (pm.table != nullptr) {
    page = pm.table[(int64_t)b * pm.max_blocks + L / B];
    if (page < 0 || page >= pm.num_pages) return;  // no page for the next block: unchanged
  }
  const int64_t head0 = (int64_t)b * Hkv;
  // element offset of row pos of KV head h: contiguous, or row pos % B of the page
  auto row_at = [&](int h, int pos) -> int64_t {
    return page < 0 ? ((head0 + h) * Lmax + pos) * D
                    : (((int64_t)page * Hkv + h) * B + pos % B) * D;
  };
  // the new rows: chunk w of head h (w < CPR: key, else value)
  for (int e = t; e < Hkv * 2 * CPR; e += kAppendThreads) {
    const int h = e / (2 * CPR), w = e - h * 2 * CPR;
    const int64_t head = head0 + h;
    if (w < CPR) {
      reinterpret_cast<uint4*>(Kc + row_at(h, L))[w] = ldg16(k_new + head * D + w * EPC);
    } else {
      reinterpret_cast<uint4*>(Vc + row_at(h, L))[w - CPR] =
          ldg16(v_new + head * D + (w - CPR) * EPC);
    }
  }
  const int j = (L + 1) / B - 1;
  if ((L + 1) % B != 0 || j >= nfull) {
    if (t == 0) seqlens[b] = L + 1;
    return;
  }
  __syncthreads();  // the new key rows are visible to the whole CTA
  const int P = Hkv * CPR;  // (head, chunk) pairs
  int TP = 1;               // threads per pair (a power of two, at most 32)
  while (TP < 32 && TP * 2 * P <= kAppendThreads) TP *= 2;
  const int part = t % TP;
  for (int p0 = 0; p0 < P; p0 += kAppendThreads / TP) {
    const int pair = p0 + t / TP;
    float acc[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
    const int h = pair / CPR, cc = pair - (pair / CPR) * CPR;
    if (pair < P) {
      const T* src = Kc + row_at(h, j * B) + cc * EPC;
#pragma unroll 8
      for (int r = part; r < B; r += TP) {
        const uint4 v = __ldcg(reinterpret_cast<const uint4*>(src + (int64_t)r * D));
        float f[EPC];
        unpack16(v, f, (const T*)nullptr);
#pragma unroll
        for (int e = 0; e < EPC; ++e) acc[e] += f[e];
      }
    }
#pragma unroll
    for (int o = 1; o < TP; o <<= 1)
#pragma unroll
      for (int e = 0; e < EPC; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    if (pair < P && part == 0) {
      float4* dst = reinterpret_cast<float4*>(S + ((head0 + h) * nfull + j) * D + cc * EPC);
      const float inv = 1.0f / (float)B;
#pragma unroll
      for (int e = 0; e < EPC; e += 4)
        dst[e / 4] = make_float4(acc[e] * inv, acc[e + 1] * inv, acc[e + 2] * inv, acc[e + 3] * inv);
    }
  }
  if (t == 0) seqlens[b] = L + 1;
}

template <typename T, int D>
static cudaError_t launch_append_t(void* Kc, void* Vc, float* S, int32_t* seqlens,
                                   const void* k_new, const void* v_new, int batch, int Hkv,
                                   int Lmax, int B, cudaStream_t st, CacheMap pm) {
  decode_append_kernel<T, D><<<batch, kAppendThreads, 0, st>>>((T*)Kc, (T*)Vc, S, seqlens, (const T*)k_new,
                                                    (const T*)v_new, Hkv, Lmax, B, Lmax / B, pm);
  return cudaGetLastError();
}

cudaError_t launch_decode_append(void* Kc, void* Vc, ssa_dtype dt, float* S, int32_t* seqlens,
                                 const void* k_new, const void* v_new, int batch, int Hkv,
                                 int Lmax, int d, int B, cudaStream_t st, CacheMap pm) {
  if (dt == SSA_BF16) {
    return d == 128 ? launch_append_t<__nv_bfloat16, 128>(Kc, Vc, S, seqlens, k_new, v_new, batch,
                                                          Hkv, Lmax, B, st, pm)
                    : launch_append_t<__nv_bfloat16, 64>(Kc, Vc, S, seqlens, k_new, v_new, batch,
                                                         Hkv, Lmax, B, st, pm);
  }
  return d == 128 ? launch_append_t<float, 128>(Kc, Vc, S, seqlens, k_new, v_new, batch, Hkv, Lmax,
                                                B, st, pm)
                  : launch_append_t<float, 64>(Kc, Vc, S, seqlens, k_new, v_new, batch, Hkv, Lmax,
                                               B, st, pm);
}

}  // namespace ssa
