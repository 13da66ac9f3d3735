// One decode step of block-sparse attention with top-k summary routing
// (DashAttention page, "Contribuições Principais" 4, incremental decoding;
// The Sparse Frontier page, RQ2: decode keeps the whole KV cache and loads
// only the selected blocks, so its cost is memory traffic).
//
// Two launches, both HBM-bound:
//   1. route: one CTA per (sequence, KV head).  The group-mean query scores
//      the summaries of the complete blocks 1 .. last-1 (each warp takes 32
//      summaries per step; lane l holds d/32 coordinates; a 31-shuffle
//      butterfly leaves dot product l in lane l), then one warp runs the exact
//      radix top-k (ties to the lower index).  The block list goes to the
//      scratch area (and to the caller's idx if given).
//   2. split-KV attention: one CTA per (split, sequence, KV head).  Each split
//      owns a contiguous run of the selected blocks; every block's K rows and
//      V rows are contiguous in the BHND cache, so each is fetched with ONE
//      untiled bulk copy (TMA) into shared memory, all issued up front on one
//      mbarrier.  The CTA computes the G heads' logits, a local softmax
//      (max m, sum l, unnormalised o) and writes that partial; the last CTA of
//      a (sequence, KV head) to finish (atomic counter) merges the partials
//      with a log-sum-exp combine and writes O.
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace ssa {

__device__ int g_decode_error = 0;

namespace {

constexpr int kMaxG = 8;            // query heads per KV head handled by the split kernel
constexpr uint32_t kWaitLimit = 1u << 24;  // bounded mbarrier polls

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

// Exclusive prefix sum of one int per thread over a 256-thread block.
__device__ __forceinline__ int block_excl_scan(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int base = 0, all = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const int x = wsum[w];
    base += (w < warp) ? x : 0;
    all += x;
  }
  __syncthreads();
  *total = all;
  return base + incl - v;
}

// Top-k by all 256 threads of the block over n scores in shared memory; same
// result as warp_select_topk: the k highest scores, equal scores going to the
// lower index, written ascending as first + e to out[0 ..).  4-pass MSB-first
// radix select (8 bits per pass) on a shared histogram, then an index-ordered
// compaction (block scans) of the keys above the threshold and the first
// `need` keys equal to it.  Returns the number written.
__device__ int block_select_topk(const float* sc, int n, int k, int first, int32_t* out,
                                 uint32_t* hist, int* sbuf) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  if (k <= 0 || n <= 0) return 0;
  if (k >= n) {
    for (int e = t; e < n; e += 256) out[e] = first + e;
    return n;
  }
  uint32_t prefix = 0, pmask = 0;
  int need = k;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    hist[t] = 0;
    __syncthreads();
    for (int e = t; e < n; e += 256) {
      const uint32_t key = order_key(sc[e]);
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t c[8], local = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        c[q] = hist[255 - (lane * 8 + q)];
        local += c[q];
      }
      uint32_t incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t excl = incl - local;
      if (excl < (uint32_t)need && (uint32_t)need <= incl) {
        uint32_t run = excl;
        for (int q = 0; q < 8; ++q) {
          if (run + c[q] >= (uint32_t)need) {
            sbuf[8] = 255 - (lane * 8 + q);
            sbuf[9] = (int)run;
            break;
          }
          run += c[q];
        }
      }
    }
    __syncthreads();
    prefix |= (uint32_t)sbuf[8] << shift;
    pmask |= 255u << shift;
    need -= sbuf[9];
    __syncthreads();
  }
  // index-ordered compaction: thread t owns the contiguous range [e0, e1)
  const int per = (n + 255) / 256;
  const int e0 = min(t * per, n), e1 = min(e0 + per, n);
  int neq = 0;
  for (int e = e0; e < e1; ++e) neq += (order_key(sc[e]) == prefix);
  int total;
  int eqr = block_excl_scan(neq, sbuf, &total);
  int ntake = 0;
  for (int e = e0; e < e1; ++e) {
    const uint32_t key = order_key(sc[e]);
    if (key > prefix) ++ntake;
    else if (key == prefix) ntake += (eqr++ < need);
  }
  int pos = block_excl_scan(ntake, sbuf, &total);
  eqr = block_excl_scan(neq, sbuf, &total);  // recompute this thread's equal-key rank base
  for (int e = e0; e < e1; ++e) {
    const uint32_t key = order_key(sc[e]);
    bool take = key > prefix;
    if (key == prefix) take = (eqr++ < need);
    if (take) out[pos++] = first + e;
  }
  return k;
}

}  // namespace

// ---------------------------------------------------------------- 1. route
template <typename T, int D>
__global__ void __launch_bounds__(256, 2) decode_route_kernel(
    const T* __restrict__ q, const float* __restrict__ S, const int32_t* __restrict__ seqlens,
    int Hq, int Hkv, int Lmax, int B, int nsum, int kk, int width, int32_t* __restrict__ ws_idx,
    int32_t* __restrict__ ws_cnt, int* __restrict__ ws_ctr, int32_t* __restrict__ idx_out,
    float inv_sqrt_d) {
  constexpr int SL = D / 32;
  extern __shared__ __align__(16) float smem[];
  float* qb = smem;                                          // [D]
  uint32_t* hist = reinterpret_cast<uint32_t*>(qb + D);      // [256]
  float* sc = reinterpret_cast<float*>(hist + 256);          // [nsum]
  const int bg = blockIdx.x;
  const int b = bg / Hkv;
  const int g = bg - b * Hkv;
  const int G = Hq / Hkv;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int L = seqlens[b];
  const bool valid = (L >= 1) && (L <= Lmax);
  const int last = valid ? (L - 1) / B : 0;
  const int n = valid ? max(last - 1, 0) : 0;  // candidates 1 .. last-1
  if (t == 0) ws_ctr[bg] = 0;                   // reset the split counter for pass 2

  if (t < D) {
    float s = 0.f;
    for (int h = 0; h < G; ++h) s += (float)q[((int64_t)b * Hq + g * G + h) * D + t];
    qb[t] = s / (float)G;
  }
  __syncthreads();
  {
    float qs[SL];
#pragma unroll
    for (int e = 0; e < SL; ++e) qs[e] = qb[lane * SL + e];
    const float* Sg = S + (int64_t)bg * nsum * D + lane * SL;
    for (int j0 = 1 + warp * 32; j0 <= n; j0 += 32 * 8) {
      float v[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const int j = min(j0 + c, n);
        float a = 0.f;
        if constexpr (SL == 4) {
          const float4 x = __ldg(reinterpret_cast<const float4*>(Sg + (int64_t)j * D));
          a = fmaf(x.x, qs[0], a);
          a = fmaf(x.y, qs[1], a);
          a = fmaf(x.z, qs[2], a);
          a = fmaf(x.w, qs[3], a);
        } else {
          const float2 x = __ldg(reinterpret_cast<const float2*>(Sg + (int64_t)j * D));
          a = fmaf(x.x, qs[0], a);
          a = fmaf(x.y, qs[1], a);
        }
        v[c] = a;
      }
      const float dot = reduce32_transpose(v);
      const int j = j0 + lane;
      if (j <= n) sc[j - 1] = dot * inv_sqrt_d;
    }
  }
  __syncthreads();
  __shared__ int sbuf[16];
  int32_t* row = ws_idx + (int64_t)bg * width;
  int n_sel = 0;
  if (valid) {
    n_sel = 1;
    if (last >= 1) {
      const int m = block_select_topk(sc, n, kk, 1, row + 1, hist, sbuf);
      if (t == 0) row[m + 1] = last;
      n_sel = m + 2;
    }
    if (t == 0) row[0] = 0;
  }
  for (int p = n_sel + t; p < width; p += 256) row[p] = -1;
  if (t == 0) ws_cnt[bg] = n_sel;
  __syncthreads();
  if (idx_out != nullptr) {
    for (int p = t; p < width; p += 256) idx_out[(int64_t)bg * width + p] = row[p];
  }
}

// -------------------------------------------------------- 2. split-KV attention
// Partial record per (sequence, KV head, split): m[G], l[G], o[G][D] (fp32,
// log2 domain, o unnormalised).
template <int D>
__host__ __device__ constexpr int part_floats(int G) {
  return G * (D + 2);
}

template <typename T, int D, int GP>
__global__ void __launch_bounds__(256) decode_split_kernel(
    const T* __restrict__ q, const T* __restrict__ Kc, const T* __restrict__ Vc,
    const int32_t* __restrict__ seqlens, int Hq, int Hkv, int Lmax, int B, int width, int splits,
    int per_split, const int32_t* __restrict__ ws_idx, const int32_t* __restrict__ ws_cnt,
    float* __restrict__ ws_part, int* __restrict__ ws_ctr, T* __restrict__ O,
    float scale_log2) {
  // logits layout: DL lanes per key, each holding DS coordinates of every
  // head's q; a warp step covers KG keys
  constexpr int DL = 8 * GP / 4;
  constexpr int DS = D / DL;
  constexpr int KG = 32 / DL;
  // P.V layout: lane owns SL output coordinates of every head
  constexpr int SL = D / 32;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const int G = Hq / Hkv;
  const int split = blockIdx.x;
  const int bg = blockIdx.y;
  const int b = bg / Hkv;
  const int g = bg - b * Hkv;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int nk_max = per_split * B;  // keys this CTA can hold

  // shared layout: K rows | V rows | p[nk_max][GP] | ow[8][GP][D] | red
  T* Ks = reinterpret_cast<T*>(smem_raw);
  T* Vs = Ks + (size_t)nk_max * D;
  float* ps = reinterpret_cast<float*>(Vs + (size_t)nk_max * D);
  float* ow = ps + (size_t)nk_max * GP;
  float* red = ow + (size_t)8 * GP * D;  // [8][GP] maxima / sums + [GP] totals
  __shared__ uint64_t bar;
  __shared__ int s_last;

  const int L = seqlens[b];
  const int ns = ws_cnt[bg];
  const int s0 = split * per_split;
  const int s1 = min(s0 + per_split, ns);
  const int64_t kvbase = (int64_t)bg * Lmax;

  // ---- issue every block's K and V bulk copies up front
  int nkeys = 0;  // keys held, in selection order
  if (s0 < s1) {
    if (t == 0) {
      ptx::mbar_init(&bar, 1);
      ptx::fence_mbar_init();
    }
    __syncthreads();
    if (t == 0) {
      uint32_t total = 0;
      for (int s = s0; s < s1; ++s) {
        const int j = ws_idx[(int64_t)bg * width + s];
        total += 2u * (uint32_t)(min(B, L - j * B) * D * (int)sizeof(T));
      }
      ptx::mbar_arrive_expect_tx(&bar, total);
      int off = 0;
      for (int s = s0; s < s1; ++s) {
        const int j = ws_idx[(int64_t)bg * width + s];
        const int rows = min(B, L - j * B);
        const uint32_t bytes = (uint32_t)(rows * D * (int)sizeof(T));
        ptx::bulk_g2s(Ks + (size_t)off * D, Kc + (kvbase + (int64_t)j * B) * D, bytes, &bar);
        ptx::bulk_g2s(Vs + (size_t)off * D, Vc + (kvbase + (int64_t)j * B) * D, bytes, &bar);
        off += rows;
      }
    }
    for (int s = s0; s < s1; ++s) {
      const int j = ws_idx[(int64_t)bg * width + s];
      nkeys += min(B, L - j * B);
    }
  }
  // this lane's slice of every head's query, scaled into the log2 domain
  const int kg = lane / DL, dl = lane % DL;
  uint64_t qr[GP][DS / 2];
#pragma unroll
  for (int h = 0; h < GP; ++h)
#pragma unroll
    for (int e = 0; e < DS / 2; ++e) {
      float lo = 0.f, hi = 0.f;
      if (h < G) {
        const T* qp = q + ((int64_t)b * Hq + g * G + h) * D + dl * DS + 2 * e;
        lo = (float)qp[0] * scale_log2;
        hi = (float)qp[1] * scale_log2;
      }
      qr[h][e] = f32x2(lo, hi);
    }
  bool ok = true;
  if (s0 < s1) ok = ptx::mbar_wait_bounded(&bar, 0, kWaitLimit);
  if (!ok) atomicCAS(&g_decode_error, 0, (int)SSA_ERR_TIMEOUT);
  __syncthreads();

  float* part = ws_part + ((int64_t)bg * splits + split) * part_floats<D>(G);
  // ---- logits
  float mx[GP];
#pragma unroll
  for (int h = 0; h < GP; ++h) mx[h] = -INFINITY;
  if (ok) {
    for (int k0 = warp * KG; k0 < nkeys; k0 += 8 * KG) {
      const int k = k0 + kg;
      const T* kr = Ks + (size_t)min(k, nkeys - 1) * D + dl * DS;
      uint64_t acc[GP];
#pragma unroll
      for (int h = 0; h < GP; ++h) acc[h] = 0;
#pragma unroll
      for (int e = 0; e < DS / 2; ++e) {
        uint64_t kv;
        if constexpr (sizeof(T) == 2) {
          kv = bf16x2_to_f32x2(reinterpret_cast<const uint32_t*>(kr)[e]);
        } else {
          kv = f32x2(reinterpret_cast<const float*>(kr)[2 * e],
                     reinterpret_cast<const float*>(kr)[2 * e + 1]);
        }
#pragma unroll
        for (int h = 0; h < GP; ++h) ffma2(acc[h], kv, qr[h][e]);
      }
      float a[GP];
#pragma unroll
      for (int h = 0; h < GP; ++h) a[h] = f32x2_sum(acc[h]);
#pragma unroll
      for (int o = 1; o < DL; o <<= 1)
#pragma unroll
        for (int h = 0; h < GP; ++h) a[h] += __shfl_xor_sync(0xffffffffu, a[h], o);
      if (dl == 0 && k < nkeys) {
#pragma unroll
        for (int h = 0; h < GP; ++h) {
          ps[k * GP + h] = a[h];
          mx[h] = fmaxf(mx[h], a[h]);
        }
      }
    }
  }
  // CTA max per head: lanes dl == 0 of the key groups, then the warps
#pragma unroll
  for (int o = DL; o < 32; o <<= 1)
#pragma unroll
    for (int h = 0; h < GP; ++h) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], o));
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < GP; ++h) red[warp * GP + h] = mx[h];
  }
  __syncthreads();
  if (t < GP) {
    float mm = -INFINITY;
    for (int w = 0; w < 8; ++w) mm = fmaxf(mm, red[w * GP + t]);
    red[8 * GP + t] = mm;
  }
  __syncthreads();
  // p = 2^(s - m) in place, per-thread sums
  float lloc[GP];
#pragma unroll
  for (int h = 0; h < GP; ++h) lloc[h] = 0.f;
  for (int k = t; k < nkeys; k += 256) {
#pragma unroll
    for (int h = 0; h < GP; ++h) {
      const float p = exp2f(ps[k * GP + h] - red[8 * GP + h]);
      ps[k * GP + h] = p;
      lloc[h] += p;
    }
  }
  // ---- P.V: warp w walks keys w, w+8, ...; lane owns SL coordinates
  uint64_t o2[GP][SL / 2];
#pragma unroll
  for (int h = 0; h < GP; ++h)
#pragma unroll
    for (int e = 0; e < SL / 2; ++e) o2[h][e] = 0;
  __syncthreads();  // p complete
  for (int k = warp; k < nkeys; k += 8) {
    const T* vr = Vs + (size_t)k * D + lane * SL;
    uint64_t vv[SL / 2];
#pragma unroll
    for (int e = 0; e < SL / 2; ++e) {
      if constexpr (sizeof(T) == 2) {
        vv[e] = bf16x2_to_f32x2(reinterpret_cast<const uint32_t*>(vr)[e]);
      } else {
        vv[e] = f32x2(reinterpret_cast<const float*>(vr)[2 * e],
                      reinterpret_cast<const float*>(vr)[2 * e + 1]);
      }
    }
#pragma unroll
    for (int h = 0; h < GP; ++h) {
      const float p = ps[k * GP + h];
      const uint64_t p2 = f32x2(p, p);
#pragma unroll
      for (int e = 0; e < SL / 2; ++e) ffma2(o2[h][e], vv[e], p2);
    }
  }
#pragma unroll
  for (int h = 0; h < GP; ++h)
#pragma unroll
    for (int e = 0; e < SL / 2; ++e) {
      ow[((size_t)warp * GP + h) * D + lane * SL + 2 * e] = __uint_as_float((uint32_t)o2[h][e]);
      ow[((size_t)warp * GP + h) * D + lane * SL + 2 * e + 1] =
          __uint_as_float((uint32_t)(o2[h][e] >> 32));
    }
  // row sums
#pragma unroll
  for (int h = 0; h < GP; ++h) {
    const float w = warp_sum(lloc[h]);
    if (lane == 0) red[warp * GP + h] = w;
  }
  __syncthreads();
  if (t < G) {
    float ll = 0.f;
    for (int w = 0; w < 8; ++w) ll += red[w * GP + t];
    part[t] = red[8 * GP + t];  // m
    part[G + t] = ll;           // l
  }
  for (int e = t; e < G * D; e += 256) {
    const int h = e / D, dd = e - h * D;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += ow[((size_t)w * GP + h) * D + dd];
    part[2 * G + h * D + dd] = s;
  }
  // ---- the last split of this (sequence, KV head) merges the partials
  __threadfence();
  __syncthreads();
  if (t == 0) s_last = (atomicAdd(&ws_ctr[bg], 1) == splits - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float* parts = ws_part + (int64_t)bg * splits * part_floats<D>(G);
  for (int e = t; e < G * D; e += blockDim.x) {
    const int h = e / D, dd = e - h * D;
    T* op = O + ((int64_t)b * Hq + g * G + h) * D + dd;
    if (ns == 0) {
      store_out(op, 0.f);
      continue;
    }
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, __ldcg(parts + (int64_t)s * part_floats<D>(G) + h));
    float num = 0.f, den = 0.f;
    for (int s = 0; s < splits; ++s) {
      const float* ps_ = parts + (int64_t)s * part_floats<D>(G);
      const float ms = __ldcg(ps_ + h);
      if (ms == -INFINITY) continue;
      const float w = exp2f(ms - M);
      den = fmaf(w, __ldcg(ps_ + G + h), den);
      num = fmaf(w, __ldcg(ps_ + 2 * G + h * D + dd), num);
    }
    store_out(op, num / den);
  }
}

DecodePlan plan_decode(int batch, int Hq, int Hkv, int d, int B, int topk, int Lmax) {
  DecodePlan p{};
  p.G = Hq / Hkv;
  p.nblk_max = (Lmax + B - 1) / B;
  p.kk = topk < p.nblk_max ? topk : p.nblk_max;
  p.width = p.kk + 2;
  // about 64 KB of K+V per split (two 32 KB blocks at B=64, d=128, bf16)
  const int blk_bytes = 2 * B * d * 2;
  p.per_split = blk_bytes >= 65536 ? 1 : 65536 / blk_bytes;
  p.splits = (p.width + p.per_split - 1) / p.per_split;
  const size_t bg = (size_t)batch * Hkv;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  p.off_idx = 0;
  p.off_cnt = up(p.off_idx + bg * p.width * sizeof(int32_t));
  p.off_ctr = up(p.off_cnt + bg * sizeof(int32_t));
  p.off_part = up(p.off_ctr + bg * sizeof(int32_t));
  p.bytes = up(p.off_part + bg * p.splits * (size_t)p.G * (d + 2) * sizeof(float));
  return p;
}

template <typename T, int D>
static cudaError_t launch_decode_t(const DecodePlan& p, const void* q, const void* Kc,
                                   const void* Vc, const float* S, const int32_t* seqlens,
                                   int batch, int Hq, int Hkv, int Lmax, int B, float scale,
                                   void* O, int32_t* idx_out, void* ws, cudaStream_t st) {
  char* w = static_cast<char*>(ws);
  int32_t* ws_idx = reinterpret_cast<int32_t*>(w + p.off_idx);
  int32_t* ws_cnt = reinterpret_cast<int32_t*>(w + p.off_cnt);
  int* ws_ctr = reinterpret_cast<int*>(w + p.off_ctr);
  float* ws_part = reinterpret_cast<float*>(w + p.off_part);
  const int nsum = Lmax / B;
  const size_t smem1 = sizeof(float) * (D + 256 + (size_t)(nsum > 0 ? nsum : 1));
  cudaError_t e = cudaFuncSetAttribute(decode_route_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
  if (e != cudaSuccess) return e;
  decode_route_kernel<T, D><<<batch * Hkv, 256, smem1, st>>>(
      (const T*)q, S, seqlens, Hq, Hkv, Lmax, B, nsum, p.kk, p.width, ws_idx, ws_cnt, ws_ctr,
      idx_out, 1.0f / sqrtf((float)D));
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int nk_max = p.per_split * B;
  const int GPv = p.G <= 4 ? 4 : 8;
  const size_t smem2 = 2 * (size_t)nk_max * D * sizeof(T) +
                       sizeof(float) * ((size_t)nk_max * GPv + (size_t)8 * GPv * D + 9 * GPv);
  dim3 grid(p.splits, batch * Hkv);
  const float sl2 = scale * 1.4426950408889634f;
  if (p.G <= 4) {
    e = cudaFuncSetAttribute(decode_split_kernel<T, D, 4>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2);
    if (e != cudaSuccess) return e;
    decode_split_kernel<T, D, 4><<<grid, 256, smem2, st>>>(
        (const T*)q, (const T*)Kc, (const T*)Vc, seqlens, Hq, Hkv, Lmax, B, p.width, p.splits,
        p.per_split, ws_idx, ws_cnt, ws_part, ws_ctr, (T*)O, sl2);
  } else {
    e = cudaFuncSetAttribute(decode_split_kernel<T, D, 8>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2);
    if (e != cudaSuccess) return e;
    decode_split_kernel<T, D, 8><<<grid, 256, smem2, st>>>(
        (const T*)q, (const T*)Kc, (const T*)Vc, seqlens, Hq, Hkv, Lmax, B, p.width, p.splits,
        p.per_split, ws_idx, ws_cnt, ws_part, ws_ctr, (T*)O, sl2);
  }
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodePlan& p, const void* q, const void* Kc, const void* Vc,
                          ssa_dtype dt, const float* S, const int32_t* seqlens, int batch, int Hq,
                          int Hkv, int Lmax, int d, int B, float scale, void* O, int32_t* idx_out,
                          void* ws, cudaStream_t st) {
  if (dt == SSA_BF16) {
    return d == 128 ? launch_decode_t<__nv_bfloat16, 128>(p, q, Kc, Vc, S, seqlens, batch, Hq, Hkv,
                                                          Lmax, B, scale, O, idx_out, ws, st)
                    : launch_decode_t<__nv_bfloat16, 64>(p, q, Kc, Vc, S, seqlens, batch, Hq, Hkv,
                                                         Lmax, B, scale, O, idx_out, ws, st);
  }
  return d == 128 ? launch_decode_t<float, 128>(p, q, Kc, Vc, S, seqlens, batch, Hq, Hkv, Lmax, B,
                                                scale, O, idx_out, ws, st)
                  : launch_decode_t<float, 64>(p, q, Kc, Vc, S, seqlens, batch, Hq, Hkv, Lmax, B,
                                               scale, O, idx_out, ws, st);
}

int read_and_reset_decode_error() {
  int v = 0;
  cudaMemcpyFromSymbol(&v, g_decode_error, sizeof(int));
  const int z = 0;
  cudaMemcpyToSymbol(g_decode_error, &z, sizeof(int));
  return v;
}

}  // namespace ssa
