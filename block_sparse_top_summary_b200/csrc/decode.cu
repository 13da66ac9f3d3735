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
//   2. split-KV attention, a persistent streaming kernel (one CTA per SM).
//      The selected blocks of all (sequence, KV head) pairs are cut into
//      units of at most 32 KB of K + V rows; each CTA owns an equal
//      contiguous run of units.  A producer warp copies each unit into a
//      ring of shared stages.  bf16: one TMA tensor box per 64 columns
//      (128-byte swizzle), and each of four consumer warps takes whole units
//      on mma.sync tensor-core tiles (the group's heads are the rows).  fp32:
//      one untiled bulk copy each for the K rows and the V rows, and sixteen
//      consumer warps split every unit's keys in fp32 FMA.  Every consumer
//      warp keeps its own online softmax (max m, sum l, unnormalised o).
//      Where the run leaves a (sequence, KV head) the warps are merged; a
//      pair split between CTAs is finished by the last of them (atomic
//      counter) with a log-sum-exp combine of the partial records.
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "tmap.h"

namespace ssa {

__device__ int g_decode_error = 0;

namespace {


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

// Scores of GG query heads against the summaries 1 .. n in one sweep: a warp
// step takes 32 / GG summaries, lane l holding d/32 coordinates of each; the
// butterfly leaves the dot product of (summary c, head h) in lane c GG + h.
// Each dot product is formed in the order of the single-head sweep.
// sc[h n + (j - 1)] for head h and summary j.
template <int GG, int D>
__device__ __forceinline__ void score_heads(const float* qg, const float* __restrict__ Sh, int n,
                                            float* sc, float inv_sqrt_d) {
  constexpr int SL = D / 32;
  constexpr int CPS = 32 / GG;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float qs[GG][SL];
#pragma unroll
  for (int h = 0; h < GG; ++h)
#pragma unroll
    for (int e = 0; e < SL; ++e) qs[h][e] = qg[h * D + lane * SL + e];
  const float* Sg = Sh + lane * SL;
  for (int j0 = 1 + warp * CPS; j0 <= n; j0 += CPS * 8) {
    float v[32];
#pragma unroll
    for (int c = 0; c < CPS; ++c) {
      const int j = min(j0 + c, n);
      float x[SL];
      if constexpr (SL == 4) {
        const float4 y = __ldg(reinterpret_cast<const float4*>(Sg + (int64_t)j * D));
        x[0] = y.x; x[1] = y.y; x[2 % SL] = y.z; x[3 % SL] = y.w;
      } else {
        const float2 y = __ldg(reinterpret_cast<const float2*>(Sg + (int64_t)j * D));
        x[0] = y.x; x[1 % SL] = y.y;
      }
#pragma unroll
      for (int h = 0; h < GG; ++h) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < SL; ++e) a = fmaf(x[e], qs[h][e], a);
        v[c * GG + h] = a;
      }
    }
    const float dot = reduce32_transpose(v);
    const int c = lane / GG, h = lane - (lane / GG) * GG;
    const int j = j0 + c;
    if (j <= n) sc[(size_t)h * n + (j - 1)] = dot * inv_sqrt_d;
  }
}

// ---------------------------------------------------------------- 1. route
template <typename T, int D>
__global__ void __launch_bounds__(256, 2) decode_route_kernel(
    const T* __restrict__ q, const float* __restrict__ S, const int32_t* __restrict__ seqlens,
    int Hq, int Hkv, int Lmax, int B, int nsum, int kk, int width, int32_t* __restrict__ ws_idx,
    int32_t* __restrict__ ws_cnt, int* __restrict__ ws_ctr, int32_t* __restrict__ idx_out,
    float inv_sqrt_d, int kv_div, int head_width, int gsweep) {
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

  // scores of the candidates against qb, into sc
  auto score = [&]() {
    float qs[SL];
#pragma unroll
    for (int e = 0; e < SL; ++e) qs[e] = qb[lane * SL + e];
    // the summaries of the unit's cache head (units are query heads when kv_div > 1)
    const int64_t hc = (int64_t)b * (Hkv / kv_div) + g / kv_div;
    const float* Sg = S + hc * nsum * D + lane * SL;
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
  };
  __shared__ int sbuf[16];
  int32_t* row = ws_idx + (int64_t)bg * width;
  // {0} + top-k of the candidates (scores at scs) + {last} into row[0 ..);
  // returns the count
  auto select = [&](const float* scs) -> int {
    int n_sel = 0;
    if (valid) {
      n_sel = 1;
      if (last >= 1) {
        const int m = block_select_topk(scs, n, kk, 1, row + 1, hist, sbuf);
        if (t == 0) row[m + 1] = last;
        n_sel = m + 2;
      }
      if (t == 0) row[0] = 0;
    }
    return n_sel;
  };

  if (head_width == 0) {
    // one selection per KV head from the group-mean query
    if (t < D) {
      float s = 0.f;
      for (int h = 0; h < G; ++h) s += (float)q[((int64_t)b * Hq + g * G + h) * D + t];
      qb[t] = s / (float)G;
    }
    __syncthreads();
    score();
    __syncthreads();
    const int n_sel = select(sc);
    for (int p = n_sel + t; p < width; p += 256) row[p] = -1;
    if (t == 0) ws_cnt[bg] = n_sel;
    __syncthreads();
    if (idx_out != nullptr) {
      for (int p = t; p < width; p += 256) idx_out[(int64_t)bg * width + p] = row[p];
    }
    return;
  }

  // one selection per query head; the row then holds their union, ascending,
  // each entry j | (mask of the heads that chose j) << 24
  // (gsweep > 1: the G heads scored in one sweep over the summaries into
  // sc[G][n]; else one sweep per head)
  uint8_t* hm = reinterpret_cast<uint8_t*>(sc + (size_t)gsweep * (nsum > 0 ? nsum : 1));
  float* qg = reinterpret_cast<float*>(hm + (((size_t)nsum + 2 + 15) & ~(size_t)15));  // [G][D]
  for (int j = t; j < nsum + 2; j += 256) hm[j] = 0;
  if (gsweep > 1) {
    for (int e = t; e < G * D; e += 256) qg[e] = (float)q[((int64_t)b * Hq + g * G) * D + e];
    __syncthreads();
    const float* Sh = S + ((int64_t)b * Hkv + g) * nsum * D;
    if (G == 2) score_heads<2, D>(qg, Sh, n, sc, inv_sqrt_d);
    else if (G == 4) score_heads<4, D>(qg, Sh, n, sc, inv_sqrt_d);
    else score_heads<8, D>(qg, Sh, n, sc, inv_sqrt_d);
  }
  for (int h = 0; h < G; ++h) {
    __syncthreads();  // the previous head's list is consumed
    if (gsweep == 1) {
      if (t < D) qb[t] = (float)q[((int64_t)b * Hq + g * G + h) * D + t];
      __syncthreads();
      score();
      __syncthreads();
    }
    const int n_sel = select(gsweep > 1 ? sc + (size_t)h * n : sc);
    __syncthreads();
    for (int p = t; p < n_sel; p += 256) hm[row[p]] |= (uint8_t)(1u << h);
    if (idx_out != nullptr) {
      int32_t* orow = idx_out + ((int64_t)b * Hq + g * G + h) * head_width;
      for (int p = t; p < head_width; p += 256) orow[p] = p < n_sel ? row[p] : -1;
    }
  }
  __syncthreads();
  __shared__ int wsum[8];
  int total = 0;
  const int nb = valid ? last + 1 : 0;  // blocks 0 .. last
  for (int base = 0; base < nb; base += 256) {
    const int j = base + t;
    const int mask = j < nb ? (int)hm[j] : 0;
    int tot = 0;
    const int off = block_excl_scan(mask != 0 ? 1 : 0, wsum, &tot);
    if (mask != 0) row[total + off] = j | (mask << 24);
    total += tot;
  }
  for (int p = total + t; p < width; p += 256) row[p] = -1;
  if (t == 0) ws_cnt[bg] = total;
}

// -------------------------------------------------------- 2. split-KV attention
// Partial record per (sequence, KV head, part): m[G], l[G], o[G][D] (fp32,
// log2 domain, o unnormalised).
template <int D>
__host__ __device__ constexpr int part_floats(int G) {
  return G * (D + 2);
}

namespace {

constexpr int kCW = 16;                         // consumer warps
constexpr int kMW = 8;                          // merge slots (consumer warps fold in pairs)
constexpr int kStreamThreads = 32 * (kCW + 1);  // + one producer warp
constexpr int kMaxStages = 8;
constexpr unsigned long long kWaitNs = 1000000000ull;  // 1 s per bounded wait

// Layout constants of the streaming kernel.
template <typename T, int D, int GP>
struct StreamShape {
  // logits: DL lanes per key, each holding DS coordinates of every head's
  // query; a warp step covers KG keys.  A lane reads its coordinates as NV
  // vectors of VB bytes at vector indices dl, dl + DL, ... of the row, so the
  // DL lanes of a key read consecutive 16-byte words (no bank conflicts).
  // After the reduction R lanes hold each head's dot product.
  static constexpr int DL = 4 * GP < 32 ? 4 * GP : 32;
  static constexpr int R = DL / GP;
  static constexpr int KG = 32 / DL;
  static constexpr int DS = D / DL;
  static constexpr int VB = DS * (int)sizeof(T) < 16 ? DS * (int)sizeof(T) : 16;
  static constexpr int EV = VB / (int)sizeof(T);
  static constexpr int NV = DS / EV;
  // P.V: lane owns SL consecutive output coordinates of every head
  static constexpr int SL = D / 32;
  // most keys of one unit (32 KB of K + V) and of one warp's share of it
  static constexpr int CKM = 32768 / (2 * D * (int)sizeof(T));
  static constexpr int KWM = CKM / kCW;
  static_assert(KWM >= 1 && KWM <= 16, "per-warp scratch holds 16 keys");
  // per-warp scratch: logits s[16][GP] | p pairs [16][GP] | alpha[GP] (+pad)
  static constexpr int kPwBytes = 16 * GP * 4 + 16 * GP * 8 + 32;
};

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait by one thread: false when the CTA aborted or the wait expired
// (then the CTA aborts and the device error word is set).
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > kWaitNs) {
        *abort = 1;
        atomicCAS(&g_decode_error, 0, (int)SSA_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Warp-uniform bounded wait: lane 0 polls, every lane then observes the
// completed phase itself (acquire order for its own shared-memory reads).
__device__ __forceinline__ bool warp_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = wait_bounded(bar, parity, abort) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) ptx::mbar_try_wait(bar, parity);
  return ok != 0;
}

// Warp-uniform bounded wait until the shared word `tag` equals `want`
// (acquire order); false when the CTA aborted or the wait expired.
__device__ __forceinline__ bool warp_wait_tag(const int* tag, int want, volatile int* abort) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0 && ptx::ld_acquire_s32(tag) != want) {
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
      if (ptx::ld_acquire_s32(tag) == want) break;
      if ((it & 255u) == 0) {
        if (*abort) {
          ok = 0;
          break;
        }
        if (globaltimer_ns() - t0 > kWaitNs) {
          *abort = 1;
          atomicCAS(&g_decode_error, 0, (int)SSA_ERR_TIMEOUT);
          ok = 0;
          break;
        }
      }
    }
  }
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kCW * 32) : "memory");
}

__device__ __forceinline__ void mma_consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(4 * 32) : "memory");
}

template <int VB>
__device__ __forceinline__ void ld_vec(const void* p, uint32_t (&w)[VB / 4]) {
  if constexpr (VB == 16) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (VB == 8) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x; w[1] = v.y;
  } else {
    w[0] = *reinterpret_cast<const uint32_t*>(p);
  }
}

// Words of T elements -> packed fp32 pairs.
template <typename T, int NW>
__device__ __forceinline__ void to_pairs(const uint32_t (&w)[NW], uint64_t* out) {
  if constexpr (sizeof(T) == 2) {
#pragma unroll
    for (int e = 0; e < NW; ++e) out[e] = bf16x2_to_f32x2(w[e]);
  } else {
#pragma unroll
    for (int e = 0; e < NW / 2; ++e) out[e] = ((uint64_t)w[2 * e + 1] << 32) | w[2 * e];
  }
}

// CTA whose unit range [floor(x U / grid), floor((x+1) U / grid)) holds unit u.
__device__ __forceinline__ int cta_of_unit(long long u, long long U, long long grid) {
  return (int)(((u + 1) * grid + U - 1) / U - 1);
}

}  // namespace

// Persistent streaming split-KV kernel.  The selected blocks of all
// (sequence, KV head) pairs form one list of units (a unit is up to CK keys
// of one block, K rows and V rows each contiguous in the cache); CTA x takes
// the contiguous range [x U / grid, (x+1) U / grid) of that list, so every CTA
// streams the same number of bytes.  Warp kCW issues one bulk copy for the K
// rows and one for the V rows of each unit into a ring of `stages` shared
// stages (full / empty mbarriers); the kCW consumer warps each take CK / kCW
// keys of every unit and keep their own online softmax (m, l, o).  When the
// range leaves a (sequence, KV head), the warps' states are merged; if the
// pair lies wholly inside this CTA's range O is written directly, otherwise
// the CTA writes a partial record and the last of the pair's CTAs (atomic
// counter) merges the records with a log-sum-exp combine.
template <typename T, int D, int GP>
__global__ void __launch_bounds__(kStreamThreads, 1) decode_stream_kernel(
    const T* __restrict__ q, const T* __restrict__ Kc, const T* __restrict__ Vc,
    const int32_t* __restrict__ seqlens, int Hq, int Hkv, int Lmax, int B, int width, int CK,
    int subs, int stages, int stage_bytes, long long U, int parts_max,
    const int32_t* __restrict__ ws_idx, const int32_t* __restrict__ ws_cnt,
    float* __restrict__ ws_part, int* __restrict__ ws_ctr, T* __restrict__ O, float scale_log2,
    CacheMap pm) {
  using SH = StreamShape<T, D, GP>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ uint64_t full[kMaxStages], empty[kMaxStages];
  __shared__ int info[kMaxStages];  // rows held by each stage
  __shared__ int s_abort, s_last;

  const int G = Hq / Hkv;
  const int Ubg = width * subs;
  const long long grid = gridDim.x;
  const long long u0 = (long long)blockIdx.x * U / grid;
  const long long u1 = ((long long)blockIdx.x + 1) * U / grid;
  const int nunits = (int)(u1 - u0);
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  volatile int* abort = &s_abort;

  unsigned char* stage0 = smem_raw;
  float* ow = reinterpret_cast<float*>(smem_raw + (size_t)stages * stage_bytes);  // [kMW][GP][D]
  float* mw = ow + kMW * GP * D;                                                  // [kMW][GP]
  float* lw = mw + kMW * GP;                                                      // [kMW][GP]
  unsigned char* pwbase = reinterpret_cast<unsigned char*>(lw + kMW * GP);

  if (t == 0) {
    for (int s = 0; s < stages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], kCW);
    }
    s_abort = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();

  if (warp == kCW) {
    // ------------------------------------------------------------ producer
    // Lane i resolves unit base + i (block index, rows, cache offset); the
    // next batch of 32 is resolved while this one is issued.
    auto resolve = [&](long long u, long long& src, int& rows) {
      src = 0;
      rows = 0;
      if (u >= u1) return;
      const int bg = (int)(u / Ubg);
      const int rem = (int)(u - (long long)bg * Ubg);
      const int s = rem / subs, r = rem - s * subs;
      if (s >= ws_cnt[bg]) return;
      const int j = ws_idx[(int64_t)bg * width + s];
      const int L = seqlens[bg / Hkv];
      const int k0 = j * B + r * CK;
      const int rr = min(CK, min(L, (j + 1) * B) - k0);
      if (rr <= 0) return;
      const int b = bg / Hkv, g = bg - b * Hkv;
      const int Hc = Hkv / pm.kv_div, gc = g / pm.kv_div;  // the cache's head
      if (pm.table != nullptr) {
        // the block's page; a missing page reads as an empty unit
        const int page = j < pm.max_blocks ? pm.table[(int64_t)b * pm.max_blocks + j] : -1;
        if (page < 0 || page >= pm.num_pages) return;
        src = (((int64_t)page * Hc + gc) * B + r * CK) * D;
      } else {
        src = (((int64_t)b * Hc + gc) * Lmax + k0) * D;
      }
      rows = rr;
    };
    long long src_n;
    int rows_n;
    resolve(u0 + lane, src_n, rows_n);
    int issued = 0;
    bool ok = true;
    for (int base = 0; ok && base < nunits; base += 32) {
      const long long src_c = src_n;
      const int rows_c = rows_n;
      resolve(u0 + base + 32 + lane, src_n, rows_n);
      const int cnt = min(32, nunits - base);
      for (int i = 0; i < cnt; ++i) {
        const int n = base + i;
        const int st = n % stages;
        const long long src = __shfl_sync(0xffffffffu, src_c, i);
        const int rows = __shfl_sync(0xffffffffu, rows_c, i);
        if (n >= stages && !(ok = warp_wait_bounded(&empty[st], ((n / stages) - 1) & 1, abort)))
          break;
        if (lane == 0) {
          info[st] = rows;
          unsigned char* dst = stage0 + (size_t)st * stage_bytes;
          if (rows > 0) {
            const uint32_t bytes = (uint32_t)rows * D * (uint32_t)sizeof(T);
            ptx::mbar_arrive_expect_tx(&full[st], 2 * bytes);
            ptx::bulk_g2s(dst, Kc + src, bytes, &full[st]);
            ptx::bulk_g2s(dst + (size_t)CK * D * sizeof(T), Vc + src, bytes, &full[st]);
          } else {
            ptx::mbar_arrive(&full[st]);
          }
        }
        issued = n + 1;
      }
    }
    // every copy issued lands before the CTA may exit (also after an abort)
    if (lane == 0) {
      volatile int no_abort = 0;
      for (int n = max(0, issued - stages); n < issued; ++n)
        wait_bounded(&full[n % stages], (uint32_t)(n / stages) & 1u, &no_abort);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int kg = lane / SH::DL, dl = lane % SH::DL;
  const int KW = CK / kCW;  // keys of each unit this warp takes (CK is a multiple of 16)
  float* pws = reinterpret_cast<float*>(pwbase + warp * SH::kPwBytes);
  uint64_t* pwp = reinterpret_cast<uint64_t*>(pwbase + warp * SH::kPwBytes + 16 * GP * 4);
  float* pwa = reinterpret_cast<float*>(pwbase + warp * SH::kPwBytes + 16 * GP * 12);

  uint64_t qr[GP][SH::DS / 2];
  uint64_t o2[GP][SH::SL / 2];
  float m_run = -INFINITY, l_run = 0.f;
  int cur = -1;

  for (int n = 0; n <= nunits; ++n) {
    const int bg = n < nunits ? (int)((u0 + n) / Ubg) : -2;
    if (bg != cur) {
      if (cur >= 0) {
        // ---- end of a (sequence, KV head): merge the warps' states.  First
        // warps kMW.. publish and warp w < kMW folds in warp w + kMW; then
        // warps < kMW publish and every thread merges the kMW slots.
        float l = l_run;
#pragma unroll
        for (int o = GP; o < 32; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        const int slot = warp & (kMW - 1);
        auto publish = [&]() {
          if (lane < GP) {
            mw[slot * GP + lane] = m_run;
            lw[slot * GP + lane] = l;
          }
#pragma unroll
          for (int h = 0; h < GP; ++h)
#pragma unroll
            for (int e = 0; e < SH::SL / 2; ++e)
              *reinterpret_cast<uint64_t*>(ow + ((size_t)slot * GP + h) * D + lane * SH::SL + 2 * e) =
                  o2[h][e];
        };
        if (warp >= kMW) publish();
        __syncwarp();
        consumer_sync();
        if (warp < kMW) {
          float m_new = m_run, l_new = l;
#pragma unroll
          for (int h = 0; h < GP; ++h) {
            const float ma = __shfl_sync(0xffffffffu, m_run, h);  // lane h keeps head h
            const float mb = mw[slot * GP + h];
            const float M = fmaxf(ma, mb);
            const float sa = ma == -INFINITY ? 0.f : ex2_approx(ma - M);
            const float sb = mb == -INFINITY ? 0.f : ex2_approx(mb - M);
#pragma unroll
            for (int e = 0; e < SH::SL / 2; ++e) {
              const uint64_t ob =
                  *reinterpret_cast<const uint64_t*>(ow + ((size_t)slot * GP + h) * D + lane * SH::SL + 2 * e);
              const float lo = __uint_as_float((uint32_t)o2[h][e]) * sa + __uint_as_float((uint32_t)ob) * sb;
              const float hi = __uint_as_float((uint32_t)(o2[h][e] >> 32)) * sa +
                               __uint_as_float((uint32_t)(ob >> 32)) * sb;
              o2[h][e] = f32x2(lo, hi);
            }
            if (h == lane % GP) {
              m_new = M;
              l_new = l * sa + lw[slot * GP + h] * sb;
            }
          }
          m_run = m_new;
          l = l_new;
          __syncwarp();
          publish();
        }
        __syncwarp();
        consumer_sync();
        const int b = cur / Hkv, g = cur - b * Hkv;
        const long long uf = (long long)cur * Ubg;
        const int xf = cta_of_unit(uf, U, grid);
        const int nparts = cta_of_unit(uf + Ubg - 1, U, grid) - xf + 1;
        float* part = ws_part + ((int64_t)cur * parts_max + (blockIdx.x - xf)) * part_floats<D>(G);
        for (int e = t; e < G * D; e += kCW * 32) {
          const int h = e / D, dd = e - h * D;
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < kMW; ++w) M = fmaxf(M, mw[w * GP + h]);
          float num = 0.f, den = 0.f;
#pragma unroll
          for (int w = 0; w < kMW; ++w) {
            const float mwv = mw[w * GP + h];
            if (mwv == -INFINITY) continue;
            const float sc = exp2f(mwv - M);
            num = fmaf(sc, ow[((size_t)w * GP + h) * D + dd], num);
            den = fmaf(sc, lw[w * GP + h], den);
          }
          if (nparts == 1) {
            store_out(O + ((int64_t)b * Hq + g * G + h) * D + dd, den > 0.f ? num / den : 0.f);
          } else {
            part[2 * G + h * D + dd] = num;
            if (dd == 0) {
              part[h] = M;
              part[G + h] = den;
            }
          }
        }
        if (nparts > 1) __threadfence();
        consumer_sync();
        if (nparts > 1) {
          if (t == 0) s_last = (atomicAdd(&ws_ctr[cur], 1) == nparts - 1);
          consumer_sync();
          if (s_last) {
            __threadfence();
            const float* parts = ws_part + (int64_t)cur * parts_max * part_floats<D>(G);
            for (int e = t; e < G * D; e += kCW * 32) {
              const int h = e / D, dd = e - h * D;
              float M = -INFINITY;
              for (int p = 0; p < nparts; ++p)
                M = fmaxf(M, __ldcg(parts + (int64_t)p * part_floats<D>(G) + h));
              float num = 0.f, den = 0.f;
              for (int p = 0; p < nparts; ++p) {
                const float* pp = parts + (int64_t)p * part_floats<D>(G);
                const float mp = __ldcg(pp + h);
                if (mp == -INFINITY) continue;
                const float sc = exp2f(mp - M);
                den = fmaf(sc, __ldcg(pp + G + h), den);
                num = fmaf(sc, __ldcg(pp + 2 * G + h * D + dd), num);
              }
              store_out(O + ((int64_t)b * Hq + g * G + h) * D + dd, den > 0.f ? num / den : 0.f);
            }
          }
        }
      }
      if (n == nunits) break;
      // ---- start of a (sequence, KV head): its query slice, fresh state
      cur = bg;
      {
        const int b = bg / Hkv, g = bg - b * Hkv;
#pragma unroll
        for (int h = 0; h < GP; ++h)
#pragma unroll
          for (int m = 0; m < SH::NV; ++m) {
            uint64_t pr[SH::EV / 2];
            if (h < G) {
              uint32_t w[SH::VB / 4];
              ld_vec<SH::VB>(q + ((int64_t)b * Hq + g * G + h) * D + (dl + SH::DL * m) * SH::EV, w);
              to_pairs<T, SH::VB / 4>(w, pr);
            } else {
#pragma unroll
              for (int e = 0; e < SH::EV / 2; ++e) pr[e] = 0;
            }
#pragma unroll
            for (int e = 0; e < SH::EV / 2; ++e) {
              const float lo = __uint_as_float((uint32_t)pr[e]) * scale_log2;
              const float hi = __uint_as_float((uint32_t)(pr[e] >> 32)) * scale_log2;
              qr[h][m * (SH::EV / 2) + e] = f32x2(lo, hi);
            }
          }
#pragma unroll
        for (int h = 0; h < GP; ++h)
#pragma unroll
          for (int e = 0; e < SH::SL / 2; ++e) o2[h][e] = 0;
        m_run = -INFINITY;
        l_run = 0.f;
      }
    }

    // ---- one unit
    const int st = n % stages;
    if (warp_wait_bounded(&full[st], (uint32_t)(n / stages) & 1u, abort)) {
      const int rows = info[st];
      const int kw0 = warp * KW;
      const int kwv = min(KW, rows - kw0);
      if (kwv > 0) {
        const T* Ks = reinterpret_cast<const T*>(stage0 + (size_t)st * stage_bytes);
        const T* Vs = Ks + (size_t)CK * D;
        // logits of this warp's keys, log2 domain.  The loops run to the
        // compile-time maximum KWM with rows clamped into the unit, so they
        // unroll and their shared loads overlap; keys >= kwv are masked.
#pragma unroll
        for (int sp = 0; sp < SH::KWM; sp += SH::KG) {
          const int kl = sp + kg;
          const bool valid = kl < kwv;
          const T* kr = Ks + (size_t)(kw0 + min(kl, kwv - 1)) * D;
          uint64_t acc[GP];
#pragma unroll
          for (int h = 0; h < GP; ++h) acc[h] = 0;
#pragma unroll
          for (int m = 0; m < SH::NV; ++m) {
            uint32_t w[SH::VB / 4];
            ld_vec<SH::VB>(kr + (dl + SH::DL * m) * SH::EV, w);
            uint64_t kv[SH::EV / 2];
            to_pairs<T, SH::VB / 4>(w, kv);
#pragma unroll
            for (int e = 0; e < SH::EV / 2; ++e)
#pragma unroll
              for (int h = 0; h < GP; ++h) ffma2(acc[h], kv[e], qr[h][m * (SH::EV / 2) + e]);
          }
          float a[GP];
#pragma unroll
          for (int h = 0; h < GP; ++h) a[h] = f32x2_sum(acc[h]);
          // reduce-scatter over the DL lanes of the key: lane dl ends with
          // head dl / R (the R lanes of a head hold the same sum)
#pragma unroll
          for (int c = GP, msk = SH::DL / 2; c > 1; c >>= 1, msk >>= 1) {
            const bool upper = (dl & msk) != 0;
#pragma unroll
            for (int k = 0; k < c / 2; ++k) {
              const float send = upper ? a[k] : a[k + c / 2];
              const float keep = upper ? a[k + c / 2] : a[k];
              a[k] = keep + __shfl_xor_sync(0xffffffffu, send, msk);
            }
          }
          float s = a[0];
#pragma unroll
          for (int msk = SH::R / 2; msk >= 1; msk >>= 1) s += __shfl_xor_sync(0xffffffffu, s, msk);
          if (dl % SH::R == 0) pws[kl * GP + dl / SH::R] = valid ? s : -INFINITY;
        }
        __syncwarp();
        // online softmax: lane keeps head lane % GP; its elements are
        // e = lane + 32 i (key e / GP)
        constexpr int NEL = SH::KWM * GP;         // elements of the warp's keys
        constexpr int NE = (NEL + 31) / 32;
        float sv[NE];
        float cm = -INFINITY;
#pragma unroll
        for (int i2 = 0; i2 < NE; ++i2) {
          const int e = lane + 32 * i2;
          sv[i2] = (NEL % 32 == 0 || e < NEL) ? pws[e] : -INFINITY;
          cm = fmaxf(cm, sv[i2]);
        }
#pragma unroll
        for (int o = GP; o < 32; o <<= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
        const float m_new = fmaxf(m_run, cm);          // finite: the warp has a valid key
        const float alpha = ex2_approx(m_run - m_new);  // 0 on the first unit
        l_run *= alpha;
#pragma unroll
        for (int i2 = 0; i2 < NE; ++i2) {
          const float p = ex2_approx(sv[i2] - m_new);  // 0 for masked keys
          l_run += p;
          const int e = lane + 32 * i2;
          if (NEL % 32 == 0 || e < NEL) pwp[e] = f32x2(p, p);
        }
        if (lane < GP) pwa[lane] = alpha;
        m_run = m_new;
        __syncwarp();
#pragma unroll
        for (int h = 0; h < GP; ++h) {
          const float al = pwa[h];
#pragma unroll
          for (int e = 0; e < SH::SL / 2; ++e) {
            const float lo = __uint_as_float((uint32_t)o2[h][e]) * al;
            const float hi = __uint_as_float((uint32_t)(o2[h][e] >> 32)) * al;
            o2[h][e] = f32x2(lo, hi);
          }
        }
        // P.V over this warp's keys (masked keys have p = 0 and are skipped)
#pragma unroll
        for (int kl = 0; kl < SH::KWM; ++kl) {
          uint32_t w[SH::SL * (int)sizeof(T) / 4];
          ld_vec<SH::SL * (int)sizeof(T)>(Vs + (size_t)(kw0 + min(kl, kwv - 1)) * D + lane * SH::SL,
                                          w);
          uint64_t vv[SH::SL / 2];
          to_pairs<T, SH::SL * (int)sizeof(T) / 4>(w, vv);
          const ulonglong2* pp = reinterpret_cast<const ulonglong2*>(pwp + kl * GP);
          if (kl < kwv) {
#pragma unroll
            for (int h2 = 0; h2 < GP / 2; ++h2) {
              const ulonglong2 p2 = pp[h2];
#pragma unroll
              for (int e = 0; e < SH::SL / 2; ++e) {
                ffma2(o2[2 * h2][e], vv[e], p2.x);
                ffma2(o2[2 * h2 + 1][e], vv[e], p2.y);
              }
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&empty[st]);
  }
}

// ------------------------------------------------- 2b. split-KV attention, bf16
// The same unit stream as decode_stream_kernel, with the two contractions of
// a unit on mma.sync tensor-core tiles (m16n8k16, bf16 in, fp32 accumulate):
//   S = Qg . K^T  (rows: the G <= 8 query heads of the group, rows 8-15 zero)
//   O += P . V    (P rounded to bf16, as in the prefill kernel)
// A unit's K and V rows arrive as 64-column boxes with the 128-byte swizzle
// (TMA tensor copies), so the ldmatrix row reads are conflict-free.  One
// consumer warp takes a whole unit (units n = warp mod kMmaCW) and keeps its
// own online softmax; P.V reuses the S accumulators as A fragments directly.
namespace {

constexpr int kMmaCW = 4;                          // consumer warps
constexpr int kMmaThreads = 32 * (kMmaCW + 1);     // + one producer warp

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// d += A . B for one m16n8k16 tile with A rows 8-15 zero (a1 = a3 = 0).
__device__ __forceinline__ void mma_rows8(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(kMmaThreads, 1) decode_mma_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ seqlens, int Hq, int Hkv,
    int Lmax, int B, int width, int CK, int subs, int stages, long long U, int parts_max,
    const int32_t* __restrict__ ws_idx, const int32_t* __restrict__ ws_cnt,
    float* __restrict__ ws_part, int* __restrict__ ws_ctr, __nv_bfloat16* __restrict__ O,
    float scale_log2, CacheMap pm) {
  constexpr int CKM = 32768 / (4 * D);  // most keys per unit (32 KB of K + V)
  constexpr int NT = CKM / 8;           // S column tiles
  constexpr int KS = D / 16;            // k steps of S
  constexpr int ON = D / 8;             // O column tiles
  constexpr int NB = D / 64;            // 64-column boxes per row block
  constexpr float kLazy = 8.0f;         // rescale O only when the max grows by more (log2)
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t full[kMaxStages], empty[kMaxStages];
  __shared__ int info[kMaxStages];
  __shared__ int tag[kMaxStages];  // unit each stage was last refilled for
  __shared__ int s_abort, s_last;

  const int G = Hq / Hkv;
  const int Ubg = width * subs;
  const int tile_bytes = CK * D * 2;  // K (or V) rows of one unit
  const int stage_bytes = 2 * tile_bytes;
  const long long grid = gridDim.x;
  const long long u0 = (long long)blockIdx.x * U / grid;
  const long long u1 = ((long long)blockIdx.x + 1) * U / grid;
  const int nunits = (int)(u1 - u0);
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  volatile int* abort = &s_abort;
  float* ow = reinterpret_cast<float*>(base + (size_t)stages * stage_bytes);  // [kMmaCW][8][D]
  float* mw = ow + kMmaCW * 8 * D;                                              // [kMmaCW][8]
  float* lw = mw + kMmaCW * 8;                                                  // [kMmaCW][8]

  if (t == 0) {
    for (int s = 0; s < stages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
      tag[s] = -1;
    }
    s_abort = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();

  if (warp == kMmaCW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tmK);
      ptx::prefetch_tmap(&tmV);
    }
    // tensor-map coordinates of a unit: row y, head z (contiguous: z = the
    // cache head b * Hc + gc; paged: y within the block's page, z = page * Hc
    // + gc)
    // rows: the unit's key rows, with the mask of the query heads that chose
    // the block in bits 16-23 (0: every head)
    auto resolve = [&](long long u, int& y, int& z, int& rows) {
      y = 0;
      z = 0;
      rows = 0;
      if (u >= u1) return;
      const int bg = (int)(u / Ubg);
      const int rem = (int)(u - (long long)bg * Ubg);
      const int s = rem / subs, r = rem - s * subs;
      if (s >= ws_cnt[bg]) return;
      const int ent = ws_idx[(int64_t)bg * width + s];
      const int j = ent & 0xFFFFFF;
      const int hmask = (int)((unsigned)ent >> 24);
      const int L = seqlens[bg / Hkv];
      const int k0 = j * B + r * CK;
      const int rr = min(CK, min(L, (j + 1) * B) - k0);
      if (rr <= 0) return;
      const int b = bg / Hkv, g = bg - b * Hkv;
      const int Hc = Hkv / pm.kv_div, gc = g / pm.kv_div;  // the cache's head
      if (pm.table != nullptr) {
        const int page = j < pm.max_blocks ? pm.table[(int64_t)b * pm.max_blocks + j] : -1;
        if (page < 0 || page >= pm.num_pages) return;
        y = r * CK;
        z = page * Hc + gc;
      } else {
        y = k0;
        z = b * Hc + gc;
      }
      rows = rr | (hmask << 16);
    };
    int y_n, z_n, rows_n;
    resolve(u0 + lane, y_n, z_n, rows_n);
    int issued = 0;
    bool ok = true;
    for (int b0 = 0; ok && b0 < nunits; b0 += 32) {
      const int y_c = y_n, z_c = z_n, rows_c = rows_n;
      resolve(u0 + b0 + 32 + lane, y_n, z_n, rows_n);
      const int cntb = min(32, nunits - b0);
      for (int i = 0; i < cntb; ++i) {
        const int n = b0 + i;
        const int st = n % stages;
        const int y = __shfl_sync(0xffffffffu, y_c, i);
        const int z = __shfl_sync(0xffffffffu, z_c, i);
        const int rows = __shfl_sync(0xffffffffu, rows_c, i);
        if (n >= stages && !(ok = warp_wait_bounded(&empty[st], ((n / stages) - 1) & 1, abort)))
          break;
        if (lane == 0) {
          info[st] = rows;
          ptx::st_release_s32(&tag[st], n);
          if ((rows & 0xFFFF) > 0) {
            unsigned char* dst = base + (size_t)st * stage_bytes;
            // whole boxes land (rows past the sequence are masked, rows past
            // the cache read as zeros), so the byte count is fixed
            ptx::mbar_arrive_expect_tx(&full[st], (uint32_t)stage_bytes);
            for (int bx = 0; bx < NB; ++bx) {
              ptx::tma_load_3d(dst + bx * CK * 128, &tmK, bx * 64, y, z, &full[st]);
              ptx::tma_load_3d(dst + tile_bytes + bx * CK * 128, &tmV, bx * 64, y, z, &full[st]);
            }
          } else {
            ptx::mbar_arrive(&full[st]);
          }
        }
        issued = n + 1;
      }
    }
    // every copy issued lands before the CTA may exit (also after an abort)
    if (lane == 0) {
      volatile int no_abort = 0;
      for (int n = max(0, issued - stages); n < issued; ++n)
        wait_bounded(&full[n % stages], (uint32_t)(n / stages) & 1u, &no_abort);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int gr = lane >> 2;  // fragment row = query head of the group (valid if < G)
  const int tq = lane & 3;
  uint32_t qa[KS][2];        // A fragments of q: columns 16 ks + 2 tq (+8)
  float oc[ON][4];           // O accumulators (elements 2, 3: rows 8-15, stay 0)
  float m_run = -INFINITY, l_run = 0.f;
  int cur = -1;
  // ldmatrix lane roles: matrix lane >> 3, row lane & 7
  const int lm = lane >> 3, lr = lane & 7;

  for (int n = 0; n <= nunits; ++n) {
    const int bg = n < nunits ? (int)((u0 + n) / Ubg) : -2;
    if (bg != cur) {
      if (cur >= 0) {
        // ---- end of a (sequence, KV head): merge the consumer warps
        float l = l_run;
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        if (tq == 0) {
          mw[warp * 8 + gr] = m_run;
          lw[warp * 8 + gr] = l;
        }
#pragma unroll
        for (int nt = 0; nt < ON; ++nt)
          *reinterpret_cast<float2*>(ow + ((size_t)warp * 8 + gr) * D + nt * 8 + 2 * tq) =
              make_float2(oc[nt][0], oc[nt][1]);
        __syncwarp();
        mma_consumer_sync();
        const int b = cur / Hkv, g = cur - b * Hkv;
        const long long uf = (long long)cur * Ubg;
        const int xf = cta_of_unit(uf, U, grid);
        const int nparts = cta_of_unit(uf + Ubg - 1, U, grid) - xf + 1;
        float* part = ws_part + ((int64_t)cur * parts_max + (blockIdx.x - xf)) * part_floats<D>(G);
        for (int e = t; e < G * D; e += kMmaCW * 32) {
          const int h = e / D, dd = e - h * D;
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < kMmaCW; ++w) M = fmaxf(M, mw[w * 8 + h]);
          float num = 0.f, den = 0.f;
#pragma unroll
          for (int w = 0; w < kMmaCW; ++w) {
            const float mwv = mw[w * 8 + h];
            if (mwv == -INFINITY) continue;
            const float sc = ex2_approx(mwv - M);
            num = fmaf(sc, ow[((size_t)w * 8 + h) * D + dd], num);
            den = fmaf(sc, lw[w * 8 + h], den);
          }
          if (nparts == 1) {
            store_out(O + ((int64_t)b * Hq + g * G + h) * D + dd, den > 0.f ? num / den : 0.f);
          } else {
            part[2 * G + h * D + dd] = num;
            if (dd == 0) {
              part[h] = M;
              part[G + h] = den;
            }
          }
        }
        if (nparts > 1) __threadfence();
        mma_consumer_sync();
        if (nparts > 1) {
          if (t == 0) s_last = (atomicAdd(&ws_ctr[cur], 1) == nparts - 1);
          mma_consumer_sync();
          if (s_last) {
            __threadfence();
            const float* parts = ws_part + (int64_t)cur * parts_max * part_floats<D>(G);
            for (int e = t; e < G * D; e += kMmaCW * 32) {
              const int h = e / D, dd = e - h * D;
              float M = -INFINITY;
              for (int p = 0; p < nparts; ++p)
                M = fmaxf(M, __ldcg(parts + (int64_t)p * part_floats<D>(G) + h));
              float num = 0.f, den = 0.f;
              for (int p = 0; p < nparts; ++p) {
                const float* pp = parts + (int64_t)p * part_floats<D>(G);
                const float mp = __ldcg(pp + h);
                if (mp == -INFINITY) continue;
                const float sc = ex2_approx(mp - M);
                den = fmaf(sc, __ldcg(pp + G + h), den);
                num = fmaf(sc, __ldcg(pp + 2 * G + h * D + dd), num);
              }
              store_out(O + ((int64_t)b * Hq + g * G + h) * D + dd, den > 0.f ? num / den : 0.f);
            }
          }
        }
      }
      if (n == nunits) break;
      // ---- start of a (sequence, KV head): the group's query rows, fresh state
      cur = bg;
      {
        const int b = bg / Hkv, g = bg - b * Hkv;
        const bool has = gr < G;
        const uint32_t* qp = reinterpret_cast<const uint32_t*>(
            q + ((int64_t)b * Hq + g * G + (has ? gr : 0)) * D + 2 * tq);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          qa[ks][0] = has ? qp[ks * 8] : 0u;
          qa[ks][1] = has ? qp[ks * 8 + 4] : 0u;
        }
#pragma unroll
        for (int nt = 0; nt < ON; ++nt) oc[nt][0] = oc[nt][1] = oc[nt][2] = oc[nt][3] = 0.f;
        m_run = -INFINITY;
        l_run = 0.f;
      }
    }
    if (n % kMmaCW != warp) continue;

    // ---- one unit
    // Stage st holds units n - stages, n, n + stages ... and the unit before
    // this one there belongs to another warp when kMmaCW does not divide
    // stages.  A parity wait cannot tell that unit's phase, still open, from
    // this unit's, complete; the producer tags the stage with n only after
    // that unit was consumed, so wait for the tag first.
    const int st = n % stages;
    if (warp_wait_tag(&tag[st], n, abort) &&
        warp_wait_bounded(&full[st], (uint32_t)(n / stages) & 1u, abort)) {
      const int rows = info[st] & 0xFFFF;
      const unsigned hmask = (unsigned)info[st] >> 16;
      // a query head that did not choose this block sees none of its keys
      const bool row_on = hmask == 0u || ((hmask >> gr) & 1u) != 0u;
      if (rows > 0) {
        unsigned char* stg = base + (size_t)st * stage_bytes;
        const uint32_t sK = ptx::smem_u32(stg);
        const uint32_t sV = sK + tile_bytes;
        const int np = CK / 16;  // 16-key groups in the unit
        if (rows < CK) {
          // V rows past the sequence may hold anything: make them zero so
          // that P = 0 times them stays 0
          for (int e = lane; e < (CK - rows) * NB * 8; e += 32) {
            const int rr = rows + e / (NB * 8), c = e % (NB * 8);
            *reinterpret_cast<uint4*>(stg + tile_bytes + (c >> 3) * CK * 128 + rr * 128 +
                                      (c & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          __syncwarp();
        }
        // S = q . K^T
        float sc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
        for (int p = 0; p < NT / 2; ++p) {
          if (p < np) {
            const int key = 16 * p + (lm >> 1) * 8 + lr;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
              const int chunk = ((2 * ks) & 7) + (lm & 1);
              const uint32_t addr = sK + (ks >> 2) * CK * 128 + key * 128 + ((chunk ^ (key & 7)) << 4);
              uint32_t r0, r1, r2, r3;
              ldsm_x4(addr, r0, r1, r2, r3);
              mma_rows8(sc[2 * p], qa[ks][0], qa[ks][1], r0, r1);
              mma_rows8(sc[2 * p + 1], qa[ks][0], qa[ks][1], r2, r3);
            }
          }
        }
        // online softmax for row gr (log2 domain); keys >= rows are masked
        float cm = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int key = nt * 8 + 2 * tq + e;
            const float x = (key < rows && row_on) ? sc[nt][e] * scale_log2 : -INFINITY;
            sc[nt][e] = x;
            cm = fmaxf(cm, x);
          }
        cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 1));
        cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 2));
        if (cm > m_run + kLazy) {  // lazy: P stays below 2^kLazy otherwise
          const float alpha = ex2_approx(m_run - cm);  // 0 on the first unit
          l_run *= alpha;
#pragma unroll
          for (int nt = 0; nt < ON; ++nt) {
            oc[nt][0] *= alpha;
            oc[nt][1] *= alpha;
          }
          m_run = cm;
        }
        __syncwarp();  // reconverge before the warp-collective mma.sync below
        uint32_t pa[NT / 2][2];
        // a row with no key yet (m_run = -inf) has every x = -inf here: P = 0
        const float mr = m_run == -INFINITY ? 0.f : m_run;
#pragma unroll
        for (int p = 0; p < NT / 2; ++p) {
          const float p0 = ex2_approx(sc[2 * p][0] - mr), p1 = ex2_approx(sc[2 * p][1] - mr);
          const float p2 = ex2_approx(sc[2 * p + 1][0] - mr);
          const float p3 = ex2_approx(sc[2 * p + 1][1] - mr);
          l_run += (p0 + p1) + (p2 + p3);
          pa[p][0] = pack_bf16x2(p0, p1);
          pa[p][1] = pack_bf16x2(p2, p3);
        }
        // O += P . V
#pragma unroll
        for (int p = 0; p < NT / 2; ++p) {
          if (p < np) {
            const int key = 16 * p + (lm & 1) * 8 + lr;
#pragma unroll
            for (int qd = 0; qd < ON / 2; ++qd) {
              const int chunk = 2 * qd + (lm >> 1);
              const uint32_t addr =
                  sV + (chunk >> 3) * CK * 128 + key * 128 + (((chunk & 7) ^ (key & 7)) << 4);
              uint32_t r0, r1, r2, r3;
              ldsm_x4_t(addr, r0, r1, r2, r3);
              mma_rows8(oc[2 * qd], pa[p][0], pa[p][1], r0, r1);
              mma_rows8(oc[2 * qd + 1], pa[p][0], pa[p][1], r2, r3);
            }
          }
        }
        if (rows < CK) ptx::fence_proxy_async_smem();  // generic zero stores before the next TMA
      }
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&empty[st]);
  }
}

namespace {

// Unit geometry of the streaming kernel for one element size.
struct StreamGeom {
  int ck, subs, ubg;
  long long units;
  int parts_max;
};

constexpr int kStageTarget = 32768;  // bytes of K + V per stage
constexpr int kGridMax = 512;        // upper bound on the streaming grid

StreamGeom stream_geom(int bg, int width, int d, int B, int esize) {
  StreamGeom s{};
  int ck = kStageTarget / (2 * d * esize);
  ck = ck < B ? ck : B;
  s.ck = ck;
  s.subs = (B + ck - 1) / ck;
  s.ubg = width * s.subs;
  s.units = (long long)bg * s.ubg;
  // every CTA range holds at least lr units (grid <= kGridMax), so one
  // (sequence, KV head) meets at most ceil(ubg / lr) + 1 ranges
  const long long lr = s.units / kGridMax > 0 ? s.units / kGridMax : 1;
  const long long pm = (s.ubg + lr - 1) / lr + 1;
  s.parts_max = (int)(pm < s.ubg ? pm : s.ubg);
  return s;
}

}  // namespace

DecodePlan plan_decode(int batch, int Hq, int Hkv, int d, int B, int topk, int Lmax) {
  DecodePlan p{};
  p.G = Hq / Hkv;
  p.nblk_max = (Lmax + B - 1) / B;
  p.kk = topk < p.nblk_max ? topk : p.nblk_max;
  p.width = p.kk + 2;
  const int bgn = batch * Hkv;
  const StreamGeom s2 = stream_geom(bgn, p.width, d, B, 2);
  const StreamGeom s4 = stream_geom(bgn, p.width, d, B, 4);
  p.parts_max = s2.parts_max > s4.parts_max ? s2.parts_max : s4.parts_max;
  const size_t bg = (size_t)bgn;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  p.off_idx = 0;
  p.off_cnt = up(p.off_idx + bg * p.width * sizeof(int32_t));
  p.off_ctr = up(p.off_cnt + bg * sizeof(int32_t));
  p.off_part = up(p.off_ctr + bg * sizeof(int32_t));
  p.bytes = up(p.off_part + bg * p.parts_max * (size_t)p.G * (d + 2) * sizeof(float));
  return p;
}

DecodePlan plan_decode_union(int batch, int Hq, int Hkv, int d, int B, int topk, int Lmax) {
  DecodePlan p{};
  p.G = Hq / Hkv;
  p.nblk_max = (Lmax + B - 1) / B;
  p.kk = topk < p.nblk_max ? topk : p.nblk_max;
  p.head_width = p.kk + 2;
  const int uw = p.G * p.kk + 2;  // the union of the heads' lists (sink and last shared)
  p.width = uw < p.nblk_max ? uw : (p.nblk_max > 2 ? p.nblk_max : 2);
  const int bgn = batch * Hkv;
  const StreamGeom s2 = stream_geom(bgn, p.width, d, B, 2);
  p.parts_max = s2.parts_max;
  const size_t bg = (size_t)bgn;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  p.off_idx = 0;
  p.off_cnt = up(p.off_idx + bg * p.width * sizeof(int32_t));
  p.off_ctr = up(p.off_cnt + bg * sizeof(int32_t));
  p.off_part = up(p.off_ctr + bg * sizeof(int32_t));
  p.bytes = up(p.off_part + bg * p.parts_max * (size_t)p.G * (d + 2) * sizeof(float));
  return p;
}

template <typename T, int D, int GP>
static cudaError_t launch_stream(const DecodePlan& p, const void* q, const void* Kc, const void* Vc,
                                 const int32_t* seqlens, int batch, int Hq, int Hkv, int Lmax,
                                 int B, float scale, void* O, int32_t* ws_idx, int32_t* ws_cnt,
                                 int* ws_ctr, float* ws_part, cudaStream_t st, CacheMap pm) {
  using SH = StreamShape<T, D, GP>;
  const StreamGeom s = stream_geom(batch * Hkv, p.width, D, B, (int)sizeof(T));
  const int stage_bytes = 2 * s.ck * D * (int)sizeof(T);
  const size_t fixed = sizeof(float) * ((size_t)kMW * GP * D + 2 * (size_t)kMW * GP) +
                       (size_t)kCW * SH::kPwBytes;
  const size_t budget = 225 * 1024;
  int stages = (int)((budget - fixed) / (size_t)stage_bytes);
  stages = stages > kMaxStages ? kMaxStages : stages;
  if (stages < 2) return cudaErrorInvalidConfiguration;
  const size_t smem = (size_t)stages * stage_bytes + fixed;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  long long grid = sms < kGridMax ? sms : kGridMax;
  if (grid > s.units) grid = s.units;
  if (grid < 1) return cudaSuccess;
  e = cudaFuncSetAttribute(decode_stream_kernel<T, D, GP>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  decode_stream_kernel<T, D, GP><<<(unsigned)grid, kStreamThreads, smem, st>>>(
      (const T*)q, (const T*)Kc, (const T*)Vc, seqlens, Hq, Hkv, Lmax, B, p.width, s.ck, s.subs,
      stages, stage_bytes, s.units, p.parts_max, ws_idx, ws_cnt, ws_part, ws_ctr, (T*)O,
      scale * 1.4426950408889634f, pm);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_mma(const DecodePlan& p, const void* q, const void* Kc, const void* Vc,
                              const int32_t* seqlens, int batch, int Hq, int Hkv, int Lmax, int B,
                              float scale, void* O, int32_t* ws_idx, int32_t* ws_cnt, int* ws_ctr,
                              float* ws_part, cudaStream_t st, CacheMap pm) {
  const StreamGeom s = stream_geom(batch * Hkv, p.width, D, B, 2);
  const int stage_bytes = 4 * s.ck * D;
  const size_t fixed = sizeof(float) * ((size_t)kMmaCW * 8 * D + 2 * (size_t)kMmaCW * 8);
  const size_t budget = 224 * 1024;  // dynamic shared memory, the 1 KB alignment slack included
  int stages = (int)((budget - 1024 - fixed) / (size_t)stage_bytes);
  stages = stages > kMaxStages ? kMaxStages : stages;
  if (stages < 2) return cudaErrorInvalidConfiguration;
  const size_t smem = 1024 + (size_t)stages * stage_bytes + fixed;
  CUtensorMap mk, mv;
  // contiguous: (d, Lmax, batch * Hkv); paged: (d, B, num_pages * Hkv)
  const int Hc = Hkv / pm.kv_div;  // the cache's heads
  const int rows_dim = pm.table != nullptr ? B : Lmax;
  const int heads_dim = pm.table != nullptr ? pm.num_pages * Hc : batch * Hc;
  if (!make_bf16_map(&mk, Kc, D, rows_dim, heads_dim, s.ck) ||
      !make_bf16_map(&mv, Vc, D, rows_dim, heads_dim, s.ck))
    return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  long long grid = sms < kGridMax ? sms : kGridMax;
  if (grid > s.units) grid = s.units;
  if (grid < 1) return cudaSuccess;
  e = cudaFuncSetAttribute(decode_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
  if (e != cudaSuccess) return e;
  decode_mma_kernel<D><<<(unsigned)grid, kMmaThreads, smem, st>>>(
      mk, mv, (const __nv_bfloat16*)q, seqlens, Hq, Hkv, Lmax, B, p.width, s.ck, s.subs, stages,
      s.units, p.parts_max, ws_idx, ws_cnt, ws_part, ws_ctr, (__nv_bfloat16*)O,
      scale * 1.4426950408889634f, pm);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t launch_decode_t(const DecodePlan& p, const void* q, const void* Kc,
                                   const void* Vc, const float* S, const int32_t* seqlens,
                                   int batch, int Hq, int Hkv, int Lmax, int B, float scale,
                                   void* O, int32_t* idx_out, void* ws, cudaStream_t st,
                                   CacheMap pm) {
  char* w = static_cast<char*>(ws);
  int32_t* ws_idx = reinterpret_cast<int32_t*>(w + p.off_idx);
  int32_t* ws_cnt = reinterpret_cast<int32_t*>(w + p.off_cnt);
  int* ws_ctr = reinterpret_cast<int*>(w + p.off_ctr);
  float* ws_part = reinterpret_cast<float*>(w + p.off_part);
  const int nsum = Lmax / B;
  // the union of the heads' selections is streamed by the bf16 split pass only,
  // whose rows are the group's (at most 8) query heads
  if (p.head_width > 0 && (sizeof(T) != 2 || p.G > 8 || pm.kv_div != 1)) return cudaErrorInvalidValue;
  // union: the G heads' scores in one sweep when they fit beside the rest
  const size_t nsc = (size_t)(nsum > 0 ? nsum : 1);
  const int gsweep = (p.head_width > 0 && (p.G == 2 || p.G == 4 || p.G == 8) &&
                      sizeof(float) * p.G * (nsc + D) <= (size_t)160 * 1024)
                         ? p.G
                         : 1;
  const size_t smem1 = sizeof(float) * (D + 256 + gsweep * nsc) +
                       (p.head_width > 0 ? (((size_t)nsum + 2 + 15) & ~(size_t)15) : 0) +
                       (gsweep > 1 ? sizeof(float) * p.G * D : 0);
  cudaError_t e = cudaFuncSetAttribute(decode_route_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
  if (e != cudaSuccess) return e;
  decode_route_kernel<T, D><<<batch * Hkv, 256, smem1, st>>>(
      (const T*)q, S, seqlens, Hq, Hkv, Lmax, B, nsum, p.kk, p.width, ws_idx, ws_cnt, ws_ctr,
      idx_out, 1.0f / sqrtf((float)D), pm.kv_div, p.head_width, gsweep);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if constexpr (sizeof(T) == 2) {
    return launch_mma<D>(p, q, Kc, Vc, seqlens, batch, Hq, Hkv, Lmax, B, scale, O, ws_idx, ws_cnt,
                         ws_ctr, ws_part, st, pm);
  } else {
    return p.G <= 4 ? launch_stream<T, D, 4>(p, q, Kc, Vc, seqlens, batch, Hq, Hkv, Lmax, B, scale,
                                             O, ws_idx, ws_cnt, ws_ctr, ws_part, st, pm)
                    : launch_stream<T, D, 8>(p, q, Kc, Vc, seqlens, batch, Hq, Hkv, Lmax, B, scale,
                                             O, ws_idx, ws_cnt, ws_ctr, ws_part, st, pm);
  }
}

cudaError_t launch_decode(const DecodePlan& p, const void* q, const void* Kc, const void* Vc,
                          ssa_dtype dt, const float* S, const int32_t* seqlens, int batch, int Hq,
                          int Hkv, int Lmax, int d, int B, float scale, void* O, int32_t* idx_out,
                          void* ws, cudaStream_t st, CacheMap pm) {
  if (dt == SSA_BF16) {
    return d == 128 ? launch_decode_t<__nv_bfloat16, 128>(p, q, Kc, Vc, S, seqlens, batch, Hq, Hkv,
                                                          Lmax, B, scale, O, idx_out, ws, st, pm)
                    : launch_decode_t<__nv_bfloat16, 64>(p, q, Kc, Vc, S, seqlens, batch, Hq, Hkv,
                                                         Lmax, B, scale, O, idx_out, ws, st, pm);
  }
  return d == 128 ? launch_decode_t<float, 128>(p, q, Kc, Vc, S, seqlens, batch, Hq, Hkv, Lmax, B,
                                                scale, O, idx_out, ws, st, pm)
                  : launch_decode_t<float, 64>(p, q, Kc, Vc, S, seqlens, batch, Hq, Hkv, Lmax, B,
                                               scale, O, idx_out, ws, st, pm);
}

cudaError_t decode_error_word(int** word) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(word), g_decode_error);
}

int read_and_reset_decode_error() {
  int v = 0;
  cudaMemcpyFromSymbol(&v, g_decode_error, sizeof(int));
  const int z = 0;
  cudaMemcpyToSymbol(g_decode_error, &z, sizeof(int));
  return v;
}

}  // namespace ssa
