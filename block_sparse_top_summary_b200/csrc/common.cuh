// Device helpers shared by the kernels of the block-sparse attention library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssa.h"

namespace ssa {

constexpr int kWarp = 32;

// Elements of T in one 16-byte vector load.
template <typename T>
struct Vec16 {
  static constexpr int n = 16 / sizeof(T);
};

// Unpack one 16-byte chunk into floats (exact for fp32 and bf16).
__device__ __forceinline__ void unpack16(const uint4& v, float* out, const float*) {
  out[0] = __uint_as_float(v.x);
  out[1] = __uint_as_float(v.y);
  out[2] = __uint_as_float(v.z);
  out[3] = __uint_as_float(v.w);
}

__device__ __forceinline__ void bf16x2_to_f(uint32_t w, float& lo, float& hi) {
  lo = __uint_as_float(w << 16);
  hi = __uint_as_float(w & 0xffff0000u);
}

__device__ __forceinline__ void unpack16(const uint4& v, float* out, const __nv_bfloat16*) {
  bf16x2_to_f(v.x, out[0], out[1]);
  bf16x2_to_f(v.y, out[2], out[3]);
  bf16x2_to_f(v.z, out[4], out[5]);
  bf16x2_to_f(v.w, out[6], out[7]);
}

__device__ __forceinline__ uint4 ldg16(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// Streaming 16-byte load that does not allocate in L1.
__device__ __forceinline__ uint4 ldg16_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void store_out(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// acc += a * b on two fp32 lanes at once (one packed f32x2 FMA).
__device__ __forceinline__ void ffma2(uint64_t& acc, uint64_t a, uint64_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}

// Two bf16 (low half first) as a packed fp32 pair.
__device__ __forceinline__ uint64_t bf16x2_to_f32x2(uint32_t w) {
  return ((uint64_t)(w & 0xffff0000u) << 32) | (uint64_t)(w << 16);
}

__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  return ((uint64_t)__float_as_uint(hi) << 32) | (uint64_t)__float_as_uint(lo);
}

__device__ __forceinline__ float f32x2_sum(uint64_t v) {
  return __uint_as_float((uint32_t)v) + __uint_as_float((uint32_t)(v >> 32));
}

// Order-preserving map from fp32 to uint32: a > b (as floats, no NaN) iff key(a) > key(b).
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Capacity of the candidate list that warp_select_topk may use to filter a
// long row before its radix passes.
constexpr int kSelCap = 256;

// Top-k selection by one warp over n candidate scores held in shared memory.
//
// Candidate e (0 <= e < n) is block index first + e.  The k highest scores
// are kept, equal scores going to the lower index; the chosen block indices
// are written to out[0 ..) in ascending order and their number returned.
// hist: 128 words of shared memory private to this warp (256 bins of 16
// bits, two to a word).  n must be below 65536, so that no bin overflows.
// cand: kSelCap entries of shared memory private to this warp, or null.
//
// The k-th largest key is found by an MSB-first radix select, 8 bits per pass,
// stopping early once the threshold bin holds exactly the keys still needed;
// the compaction pass then walks the candidates in index order and takes every
// key above the threshold prefix plus the first `need` keys equal to it.
//
// With a cand buffer, k <= 32 and n >= 64, the row is filtered first: lane l
// takes the maximum key of candidates l, l + 32, ...; T is the least of these
// 32 maxima, so at least 32 >= k candidates have a key >= T, the k-th largest
// key is >= T, and every candidate that can be taken (ties at the k-th key
// included) is >= T.  The candidates >= T are listed in index order and the
// radix passes run on that list alone, starting below the leading bits that
// all its keys share (those of T and of the row maximum).  A list longer than
// kSelCap falls back to the whole row.  Both routes take the same set.
__device__ __forceinline__ int warp_select_topk(const float* sc, int n, int k, int first,
                                                int32_t* out, uint32_t* hist,
                                                uint16_t* cand = nullptr) {
  const int lane = threadIdx.x & 31;
  if (k <= 0 || n <= 0) return 0;
  if (k >= n) {
    for (int e = lane; e < n; e += 32) out[e] = first + e;
    return n;
  }
  // the list: candidate t < m is element cand[t] (or t itself without a list)
  int m = n;
  bool listed = false;
  uint32_t prefix = 0, pmask = 0;
  int lo = 32;  // bits [0, lo) of the keys are still open
  if (cand != nullptr && k <= 32 && n >= 64) {
    uint32_t lmax = 0;
    for (int e = lane; e < n; e += 32) lmax = max(lmax, order_key(sc[e]));
    const uint32_t T = __reduce_min_sync(0xffffffffu, lmax);
    const uint32_t M = __reduce_max_sync(0xffffffffu, lmax);
    int pos = 0;
    for (int base = 0; base < n && pos <= kSelCap; base += 32) {
      const int e = base + lane;
      const bool in = e < n && order_key(sc[e]) >= T;
      const uint32_t im = __ballot_sync(0xffffffffu, in);
      const int at = pos + __popc(im & lanemask_lt());
      if (in && at < kSelCap) cand[at] = (uint16_t)e;
      pos += __popc(im);
    }
    if (pos <= kSelCap) {
      listed = true;
      m = pos;
      lo = 32 - __clz(T ^ M);
      pmask = lo == 32 ? 0u : ~((1u << lo) - 1u);
      prefix = M & pmask;
    }
    __syncwarp();
  }
  auto elem = [&](int t) { return listed ? (int)cand[t] : t; };
  int need = k;  // how many of the keys matching `prefix` are still to be taken
#pragma unroll 1
  for (int hi = lo; hi > 0; hi -= 8) {
    // digit bits [shift, shift + 8); any of them at or above hi are fixed by
    // the prefix and equal in every key still in play
    const int shift = hi > 8 ? hi - 8 : 0;
    for (int b = lane; b < 128; b += 32) hist[b] = 0;
    __syncwarp();
    for (int base = 0; base < m; base += 32) {
      const int t = base + lane;
      const bool ok = t < m;
      const uint32_t key = ok ? order_key(sc[elem(t)]) : 0u;
      const bool hit = ok && ((key & pmask) == prefix);
      const uint32_t digit = (key >> shift) & 255u;
      const uint32_t act = __ballot_sync(0xffffffffu, hit);
      if (hit) {
        const uint32_t peers = __match_any_sync(act, digit);
        if ((peers & lanemask_lt()) == 0)
          atomicAdd(&hist[digit >> 1], (uint32_t)__popc(peers) << ((digit & 1u) * 16u));
      }
    }
    __syncwarp();
    // Find the digit dd with  sum_{b > dd} hist[b] < need <= sum_{b >= dd} hist[b].
    // Lane L owns bins 255-8L-7 .. 255-8L (descending), scanned high to low.
    uint32_t c[8];
    uint32_t local = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int bin = 255 - (lane * 8 + q);
      c[q] = (hist[bin >> 1] >> ((bin & 1) * 16)) & 0xffffu;
      local += c[q];
    }
    uint32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t excl = incl - local;  // count in bins above this lane's range
    const bool mine = (excl < (uint32_t)need) && ((uint32_t)need <= incl);
    const uint32_t who = __ballot_sync(0xffffffffu, mine);
    const int src = __ffs(who) - 1;
    uint32_t dd = 0, above = 0, in_bin = 0;
    if (lane == src) {
      uint32_t run = excl;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (run + c[q] >= (uint32_t)need) {
          dd = 255u - (uint32_t)(lane * 8 + q);
          above = run;
          in_bin = c[q];
          break;
        }
        run += c[q];
      }
    }
    dd = __shfl_sync(0xffffffffu, dd, src);
    above = __shfl_sync(0xffffffffu, above, src);
    in_bin = __shfl_sync(0xffffffffu, in_bin, src);
    prefix |= dd << shift;
    pmask |= 255u << shift;
    need -= (int)above;
    __syncwarp();
    // every key with this prefix is taken: no tie below it can matter
    if (in_bin == (uint32_t)need) break;
  }
  // Take every key whose masked value is above prefix, and the first `need`
  // keys equal to it in ascending index order (all of them when the passes
  // stopped early).
  int pos = 0, eq_seen = 0;
  for (int base = 0; base < m; base += 32) {
    const int t = base + lane;
    const bool ok = t < m;
    const int e = ok ? elem(t) : 0;
    const uint32_t key = ok ? (order_key(sc[e]) & pmask) : 0u;
    const bool gt = ok && key > prefix;
    const bool eq = ok && key == prefix;
    const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_seen + __popc(eqm & lanemask_lt());
    const bool take = gt || (eq && eq_rank < need);
    const uint32_t tm = __ballot_sync(0xffffffffu, take);
    if (take) out[pos + __popc(tm & lanemask_lt())] = first + e;
    pos += __popc(tm);
    eq_seen += __popc(eqm);
  }
  return pos;
}

}  // namespace ssa
