// Stage 2 on the tensor cores: exact softmax attention over the selected KV
// blocks (SSA page, "2. Metodologia", sparse stream; DashAttention page,
// "Estágio 2", a FlashAttention-style kernel iterating only the active blocks,
// here written for sm_100a).
//
// Work item: 256 query rows that share one block selection, i.e. (batch, KV
// head g, query block i, group of 256/B query heads of g).  They form two
// M-tiles of 128 rows (B = 64: two heads x 64 rows; B = 128: one head x 128
// rows).  The selected blocks are visited in chunks of 128 keys (two blocks at
// B = 64, one at B = 128; an odd last block is paired with an all-zero
// out-of-range box whose keys are masked).  One persistent CTA per SM runs a
// sequence of work items back to back, the heaviest first within each group
// of (batch, KV head) pairs.
//
// Roles (576 threads, 18 warps):
//   warp 0      TMA producer: Q of each work item (8 boxes of 64 x 64 bf16,
//               128-byte swizzle), then K and V of every chunk into a 2-stage
//               ring;
//   warp 1      TMEM owner (512 columns) and MMA issuer (one thread):
//               S_t = Q_t K^T  (tcgen05.mma kind::f16, M=128 N=128 K=16, A and B
//               from shared memory), O_t += P_t V (A = P from TMEM, B = V from
//               shared memory, MN-major);
//   warps 2-9   softmax of tile 0, warps 10-17 softmax of tile 1: two threads
//               per row (row = TMEM lane, each thread one 64-key half); read S
//               (tcgen05.ld), mask (only the last chunk holds the diagonal
//               block), exchange the half-row maxima through shared memory,
//               online softmax in the log2 domain (P is computed against a
//               reference max; O in TMEM is rescaled only when the row max
//               exceeds it by more than 2^64),
//               write P as bf16 pairs into the first 32 columns of the thread's
//               own S half (tcgen05.st), and finally normalise O and store it.
//               With a routing prior (DashAttention's stage 2) each half's
//               block adds its offset to the scaled logits.
// TMEM columns: S of tile t at 128 t (P of keys 0-63 at 128 t, of keys 64-127
// at 128 t + 64), O of tile t at 256 + 128 t.
// Every mbarrier wait is bounded in time; on expiry the CTA records
// SSA_ERR_TIMEOUT in the device error word, stops issuing work, drains what it
// issued and frees its TMEM.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "ssa_debug.h"
#include "tmap.h"

namespace ssa {

__device__ int g_attn_tc_error = 0;

namespace {

constexpr int kThreads = 576;
constexpr int kNS = 2;                      // K/V pipeline stages
constexpr uint32_t kQBytes = 65536;         // 2 tiles x 128 rows x 128 d x 2 B
constexpr uint32_t kKVBytes = 32768;        // 128 keys x 128 d x 2 B (K or V)
constexpr uint32_t kSmemBytes = kQBytes + 2 * kNS * kKVBytes;
constexpr uint32_t kTmemCols = 512;
constexpr unsigned long long kWaitNs = 1000000000ull;  // 1 s per wait


struct __align__(8) Shared {
  uint64_t q_full;           // Q of the current work item has landed
  uint64_t q_empty;          // every S of the previous work item has completed
  uint64_t k_full[kNS];
  uint64_t v_full[kNS];
  uint64_t kv_empty[kNS];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done[2];
  uint64_t o_free[2];   // per tile: the epilogue has read O (256 arrivals)
  uint64_t drain;
  uint64_t mx_full[2];  // per tile: both half-row maxima of the chunk are written
  uint64_t l_full[2];   // per tile: both half-row sums are written (epilogue)
  float mx[2][2][2][128];  // [chunk parity][tile][half][row]
  float lx[2][2][128];     // [tile][half][row]
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait: false when the CTA aborted or the wait expired (then the CTA
// aborts and the device error word is set).
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort,
                                         unsigned long long limit_ns = kWaitNs) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort) return false;
      if (globaltimer() - t0 > limit_ns) {
        *abort = 1;
        atomicCAS(&g_attn_tc_error, 0, (int)SSA_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Warp-uniform bounded wait: lane 0 polls, the result is broadcast, so the
// warp stays converged for the .sync.aligned tcgen05 instructions that follow.
__device__ __forceinline__ bool warp_wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = wait_bar(bar, parity, abort) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) ptx::mbar_try_wait(bar, parity);  // completed phase: gives every lane acquire order
  return ok != 0;
}

// Shared-memory matrix descriptor: 128-byte swizzle, sm_100 version 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) |
         ((uint64_t)(sbo >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: bf16 x bf16 -> f32, M = 128, N = 128.
constexpr uint32_t kIdescQK = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) |
                              ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = kIdescQK | (1u << 16);  // B (= V) MN-major

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x on the special-function unit (flushes results below 2^-126 to 0; 2^-inf = 0).
__device__ __forceinline__ float ex2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// (a, b) = (a * s + c, b * s + c) with one packed f32x2 FMA; s2 = {s, s}, c2 = {c, c}.
__device__ __forceinline__ void fma2(float& a, float& b, uint64_t s2, uint64_t c2) {
  asm("{\n\t.reg .b64 x;\n\tmov.b64 x, {%0, %1};\n\tfma.rn.f32x2 x, x, %2, %3;\n\t"
      "mov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a), "+f"(b)
      : "l"(s2), "l"(c2));
}

// acc += {a, b} with one packed f32x2 add.
__device__ __forceinline__ void add2(uint64_t& acc, float a, float b) {
  asm("{\n\t.reg .b64 x;\n\tmov.b64 x, {%1, %2};\n\tadd.f32x2 %0, %0, x;\n\t}"
      : "+l"(acc)
      : "f"(a), "f"(b));
}

__device__ __forceinline__ uint64_t pack2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}

__device__ __forceinline__ float sum2(uint64_t r) {
  float a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
  return a + b;
}

// bf16 pair {lo, hi} (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Max of 32 values (2 independent 3-input max chains) folded into m.
__device__ __forceinline__ float max32(const uint32_t (&v)[32], float m) {
  float a0 = m, a1 = -INFINITY;
#pragma unroll
  for (int n = 0; n < 32; n += 4) {
    a0 = max3f(a0, __uint_as_float(v[n]), __uint_as_float(v[n + 1]));
    a1 = max3f(a1, __uint_as_float(v[n + 2]), __uint_as_float(v[n + 3]));
  }
  return fmaxf(a0, a1);
}

// Columns n (0..31) of a 32-column slice starting at column `col0` whose key is
// masked (causal diagonal or the missing half of an odd chunk) become -inf.
template <int B>
__device__ __forceinline__ void mask32(uint32_t (&v)[32], int col0, const int (&lim)[2]) {
#pragma unroll
  for (int n = 0; n < 32; ++n) {
    const int col = col0 + n;
    const bool valid = (B == 64) ? ((col & 63) <= lim[col >> 6]) : (col <= lim[0]);
    if (!valid) v[n] = __float_as_uint(-INFINITY);
  }
}

// Eight 32-bit words w[o .. o+7] to global memory in one 32-byte store (p
// 32-byte aligned).
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&w)[16], int o) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[o]),
               "r"(w[o + 1]), "r"(w[o + 2]), "r"(w[o + 3]), "r"(w[o + 4]), "r"(w[o + 5]),
               "r"(w[o + 6]), "r"(w[o + 7])
               : "memory");
}

// p = 2^(s * scale - m) for 32 raw scores, packed as 16 bf16 pairs into w;
// adds the (fp32) p to acc.
__device__ __forceinline__ void exp_pack32(const uint32_t (&v)[32], uint32_t (&w)[16], uint64_t s2,
                                           uint64_t c2, uint64_t& acc) {
#pragma unroll
  for (int n = 0; n < 32; n += 2) {
    float a = __uint_as_float(v[n]), b = __uint_as_float(v[n + 1]);
    fma2(a, b, s2, c2);
    a = ex2_mufu(a);
    b = ex2_mufu(b);
    add2(acc, a, b);
    w[n >> 1] = cvt_bf16x2(a, b);
  }
}


}  // namespace

// Work item w.  The (batch, KV head) pairs are taken in groups of `kvg`
// (the last group may be smaller); within a group, the heaviest query blocks
// (the latest) come first.  A group's K and V are what the CTAs read at one
// time, so the host sizes it to stay near the L2.
struct Item {
  int b, g, i, h0, bg;
};

__device__ __forceinline__ Item item_of(int w, int subs, int nbg, int Hkv, int G, int nq, int HPI,
                                        int kvg) {
  Item it;
  const int per_grp = kvg * subs * nq;
  const int grp = w / per_grp;
  const int rem = w - grp * per_grp;
  const int gn = min(kvg, nbg - grp * kvg);  // pairs in this group
  const int per_i = gn * subs;
  it.i = nq - 1 - rem / per_i;
  const int rem2 = rem - (rem / per_i) * per_i;
  it.bg = grp * kvg + rem2 / subs;
  const int sub = rem2 - (rem2 / subs) * subs;
  it.b = it.bg / Hkv;
  it.g = it.bg - it.b * Hkv;
  it.h0 = it.g * G + sub * HPI;
  return it;
}

template <int B>
__device__ __forceinline__ int chunks_of(int ns) {
  return ns <= 0 ? 0 : (B == 64) ? (ns + 1) / 2 : ns;
}

// Persistent kernel: CTA x runs work items x, x + gridDim.x, ...  Every
// per-chunk mbarrier phase is counted by the CTA's running chunk index, so
// the pipeline flows from one item into the next: Q of the next item loads
// once the last S of the current one completes, its first S runs while the
// current item's epilogue reads O, and its first P.V waits only for that
// epilogue (o_free).
// PRIOR: the kernel adds a routing prior per selected block (the bias
// argument); the plain kernel is compiled without that code.  At most 96
// registers per thread: the 18 warps of a CTA share four register quarters of
// the SM, one of which holds 5 of them (5 x 32 x 96 fits 16K).
template <int B, bool PRIOR>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ cnt, const float* __restrict__ bias,
    __nv_bfloat16* __restrict__ O, float* __restrict__ lse,
    int Hq, int Hkv, int N, int nq, int nbg, int max_sel, float scale_log2, int kvg) {
  constexpr int HPT = 128 / B;      // query heads per M-tile
  constexpr int HPI = 2 * HPT;      // query heads per work item
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* Qs = base;
  unsigned char* Ks = base + kQBytes;
  unsigned char* Vs = Ks + kNS * kKVBytes;
  Shared* sh = reinterpret_cast<Shared*>(Vs + kNS * kKVBytes);

  const int G = Hq / Hkv;
  const int subs = G / HPI;
  const int W = nq * subs * nbg;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort = &sh->abort;
  auto ns_of = [&](int w) -> int {
    if (w >= W) return 0;
    const Item it = item_of(w, subs, nbg, Hkv, G, nq, HPI, kvg);
    return cnt[(int64_t)it.bg * nq + it.i];
  };

  if (threadIdx.x == 0) {
    ptx::mbar_init(&sh->q_full, 1);
    ptx::mbar_init(&sh->q_empty, 1);
    for (int s = 0; s < kNS; ++s) {
      ptx::mbar_init(&sh->k_full[s], 1);
      ptx::mbar_init(&sh->v_full[s], 1);
      ptx::mbar_init(&sh->kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      ptx::mbar_init(&sh->s_full[t], 1);
      ptx::mbar_init(&sh->p_full[t], 256);
      ptx::mbar_init(&sh->o_done[t], 1);
      ptx::mbar_init(&sh->o_free[t], 256);
      ptx::mbar_init(&sh->mx_full[t], 256);
      ptx::mbar_init(&sh->l_full[t], 256);
    }
    ptx::mbar_init(&sh->drain, 1);
    sh->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&sh->tmem_base, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (whole warp)
    if (lane == 0) {
      ptx::prefetch_tmap(&tmQ);
      ptx::prefetch_tmap(&tmK);
      ptx::prefetch_tmap(&tmV);
    }
    int gc = 0, kq = 0;
    bool ok = true;
    for (int w = blockIdx.x; ok && w < W; w += gridDim.x) {
      const Item it = item_of(w, subs, nbg, Hkv, G, nq, HPI, kvg);
      const int ns = cnt[(int64_t)it.bg * nq + it.i];
      const int nch = chunks_of<B>(ns);
      if (nch == 0) continue;
      const int32_t* row = idx + ((int64_t)it.bg * nq + it.i) * max_sel;
      int sbase = 0;
      int selv = lane < ns ? row[lane] : 0;  // lane p holds entry sbase + p
      // Q of this item once the previous item's S MMAs are done with Q
      if (kq > 0 && !(ok = warp_wait_bar(&sh->q_empty, (kq - 1) & 1, abort))) break;
      if (lane == 0) {
        ptx::mbar_arrive_expect_tx(&sh->q_full, kQBytes);
        for (int t = 0; t < 2; ++t)
          for (int hh = 0; hh < HPT; ++hh)
            for (int rg = 0; rg < B / 64; ++rg)
              for (int c = 0; c < 2; ++c)
                ptx::tma_load_3d(Qs + t * 32768 + c * 16384 + (hh * B + rg * 64) * 128, &tmQ,
                                 c * 64, it.i * B + rg * 64, it.b * Hq + it.h0 + t * HPT + hh,
                                 &sh->q_full);
      }
      ++kq;
      for (int c = 0; c < nch; ++c, ++gc) {
        const int s = gc % kNS;
        if (gc >= kNS && !(ok = warp_wait_bar(&sh->kv_empty[s], ((gc / kNS) - 1) & 1, abort))) break;
        const int p0 = (B == 64) ? 2 * c : c;  // first selection entry of the chunk
        if (p0 >= sbase + 32) {                // next 32 entries (p0 - sbase is even for B = 64)
          sbase += 32;
          selv = sbase + lane < ns ? row[sbase + lane] : 0;
        }
        const int j0 = __shfl_sync(0xffffffffu, selv, p0 - sbase);
        const int j1 = (B == 64) ? __shfl_sync(0xffffffffu, selv, p0 + 1 - sbase) : 0;
        if (lane == 0) {
          int y[2];
          if (B == 64) {
            y[0] = j0 * 64;
            y[1] = p0 + 1 < ns ? j1 * 64 : nq * B;  // past the end: zero box
          } else {
            y[0] = j0 * 128;
            y[1] = j0 * 128 + 64;
          }
          ptx::mbar_arrive_expect_tx(&sh->k_full[s], kKVBytes);
          for (int kg = 0; kg < 2; ++kg)
            for (int cc = 0; cc < 2; ++cc)
              ptx::tma_load_3d(Ks + s * kKVBytes + cc * 16384 + kg * 8192, &tmK, cc * 64, y[kg],
                               it.b * Hkv + it.g, &sh->k_full[s]);
          ptx::mbar_arrive_expect_tx(&sh->v_full[s], kKVBytes);
          for (int kg = 0; kg < 2; ++kg)
            for (int cc = 0; cc < 2; ++cc)
              ptx::tma_load_3d(Vs + s * kKVBytes + cc * 16384 + kg * 8192, &tmV, cc * 64, y[kg],
                               it.b * Hkv + it.g, &sh->v_full[s]);
        }
      }
    }
    if (!ok && lane == 0) {
      // let every issued copy land before the CTA's shared memory goes away
      volatile int no_abort = 0;
      for (int c = (gc > kNS ? gc - kNS : 0); c < gc; ++c) {
        const int s = c % kNS;
        const uint32_t ph = (c / kNS) & 1;
        wait_bar(&sh->k_full[s], ph, &no_abort);
        wait_bar(&sh->v_full[s], ph, &no_abort);
      }
      if (kq > 0) wait_bar(&sh->q_full, (kq - 1) & 1, &no_abort);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t qa = ptx::smem_u32(Qs);
      const uint32_t ka = ptx::smem_u32(Ks);
      const uint32_t va = ptx::smem_u32(Vs);
      bool any = false, ok = true;
      auto issue_qk = [&](int t, int s) {
        ptx::tc_fence_after();
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          ptx::mma_ss(tmem + t * 128, sdesc(qa + t * 32768 + off, 16, 1024),
                      sdesc(ka + s * kKVBytes + off, 16, 1024), kIdescQK, kk > 0);
        }
        ptx::mma_commit(&sh->s_full[t]);
      };
      auto issue_pv = [&](int t, int s, int c) {
        ptx::tc_fence_after();
        for (int kk = 0; kk < 8; ++kk)
          ptx::mma_ts(tmem + 256 + t * 128, tmem + t * 128 + (kk >> 2) * 64 + (kk & 3) * 8,
                      sdesc(va + s * kKVBytes + kk * 2048, 16384, 1024), kIdescPV,
                      (c > 0 || kk > 0) ? 1u : 0u);
        ptx::mma_commit(&sh->o_done[t]);
      };
      int gc = 0, kq = 0;
      int ns_next = ns_of(blockIdx.x);
      for (int w = blockIdx.x; ok && w < W; w += gridDim.x) {
        const int ns = ns_next;
        ns_next = ns_of(w + gridDim.x);
        const int nch = chunks_of<B>(ns);
        if (nch == 0) continue;
        if (!(ok = wait_bar(&sh->q_full, kq & 1, abort))) break;
        if (!(ok = wait_bar(&sh->k_full[gc % kNS], (gc / kNS) & 1, abort))) break;
        // S of the new item overwrites P of the previous one: issued after
        // its P.V, and tcgen05 MMAs of one thread run in issue order
        issue_qk(0, gc % kNS);
        issue_qk(1, gc % kNS);
        any = true;
        if (nch == 1) ptx::mma_commit(&sh->q_empty);
        for (int c = 0; c < nch; ++c) {
          const int g = gc + c;
          const int s = g % kNS;
          if (!(ok = wait_bar(&sh->v_full[s], (g / kNS) & 1, abort))) break;
          if (!(ok = wait_bar(&sh->p_full[0], g & 1, abort))) break;
          if (c == 0 && kq > 0 && !(ok = wait_bar(&sh->o_free[0], (kq - 1) & 1, abort))) break;
          issue_pv(0, s, c);
          const bool more = c + 1 < nch;
          const int s1 = (g + 1) % kNS;
          if (more) {
            if (!(ok = wait_bar(&sh->k_full[s1], ((g + 1) / kNS) & 1, abort))) break;
            issue_qk(0, s1);
          }
          if (!(ok = wait_bar(&sh->p_full[1], g & 1, abort))) break;
          if (c == 0 && kq > 0 && !(ok = wait_bar(&sh->o_free[1], (kq - 1) & 1, abort))) break;
          issue_pv(1, s, c);
          ptx::mma_commit(&sh->kv_empty[s]);
          if (more) {
            issue_qk(1, s1);
            if (c + 2 == nch) ptx::mma_commit(&sh->q_empty);  // last S of the item issued
          }
        }
        gc += nch;
        ++kq;
      }
      if (any) {
        // every MMA issued by this thread has completed once `drain` flips
        ptx::mma_commit(&sh->drain);
        volatile int no_abort = 0;
        wait_bar(&sh->drain, 0, &no_abort);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int t = (warp - 2) >> 3;          // M-tile
    const int half = ((warp - 2) >> 2) & 1; // key half of the chunk: columns 64 half ..
    const int quarter = warp & 3;           // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;      // row in the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128 + half * 64;
    const uint32_t tO = tmem + lane_off + 256 + t * 128 + half * 64;
    bool ok = true;
    const bool o_al32 = (reinterpret_cast<uintptr_t>(O) & 31u) == 0;
    int gc = 0, kq = 0;
    int ns_next = ns_of(blockIdx.x);
    for (int w = blockIdx.x; ok && w < W; w += gridDim.x) {
      const int ns = ns_next;
      ns_next = ns_of(w + gridDim.x);
      const int nch = chunks_of<B>(ns);
      if (nch == 0) continue;
      const Item it = item_of(w, subs, nbg, Hkv, G, nq, HPI, kvg);
      const int hh = r / B;
      const int pos = it.i * B + (r % B);
      const int h = it.h0 + t * HPT + hh;
      // the routing prior of each selected block (natural log)
      const float* brow = PRIOR ? bias + ((int64_t)it.bg * nq + it.i) * max_sel : nullptr;
      float m_used = -INFINITY, l = 0.f;
      for (int c = 0; c < nch; ++c) {
        const int g = gc + c;
        // this half's block: entry 2c + half (B = 64) or c (B = 128); its
        // prior joins the logits in the log2 domain
        const int ent = (B == 64) ? 2 * c + half : c;
        const float bh = (PRIOR && ent < ns) ? brow[ent] * 1.4426950408889634f : 0.f;
        if (!(ok = warp_wait_bar(&sh->s_full[t], g & 1, abort))) break;
        ptx::tc_fence_after();
        const bool last = (c == nch - 1);
        // causal mask / missing block, only in the chunk holding the diagonal.
        // Selections are ascending and end with the diagonal block, so the
        // last chunk is (diagonal, missing) when ns is odd and (full,
        // diagonal) when it is even (B = 64), or the diagonal (B = 128).
        // Key column n (0..127) of block half kg is valid iff (n mod 64) <=
        // lim[kg] (B = 64), or n <= lim[0] (B = 128).
        int lim[2] = {127, 127};
        if (last) {
          if (B == 64) {
            if (ns & 1) {
              lim[0] = r & 63;
              lim[1] = -1;
            } else {
              lim[0] = 63;
              lim[1] = r & 63;
            }
          } else {
            lim[0] = lim[1] = r;
          }
        }
        // pass 1: this half's maximum, then the other half's through shared memory
        float pm = -INFINITY;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint32_t v[32];
          ptx::tmem_ld32(tS + q * 32, v);
          ptx::tmem_wait_ld();
          if (last) mask32<B>(v, half * 64 + q * 32, lim);
          pm = max32(v, pm);
        }
        // the half's max of the scaled logits (with the prior), exchanged
        const float pmb = PRIOR ? pm * scale_log2 + bh : pm * scale_log2;
        sh->mx[g & 1][t][half][r] = pmb;
        ptx::mbar_arrive(&sh->mx_full[t]);
        // The two halves of a row must use one reference max.  From chunk 1
        // on, P is computed optimistically with the current reference m_used
        // while the other half's maximum is in flight; the pass is redone only
        // if the row max exceeds m_used by more than 2^kSlack (then P, l and O
        // would leave a comfortable fp32 / bf16 range).  Chunk 0 waits for the
        // exchange first.
        constexpr float kSlack = 64.0f;
        float rmax = -INFINITY;
        bool have_rmax = false;
        if (c == 0) {
          if (!(ok = warp_wait_bar(&sh->mx_full[t], g & 1, abort))) break;
          rmax = fmaxf(pmb, sh->mx[g & 1][t][half ^ 1][r]);
          m_used = rmax;
          have_rmax = true;
        }
        bool need = false;
        float alpha = 1.0f;
        uint64_t acc = 0;
        uint32_t w0[16], w1[16];  // P of this half, stored only once it is final
        for (int attempt = 0; attempt < 2; ++attempt) {
          const float mu = (m_used == -INFINITY) ? 0.f : m_used;
          const uint64_t s2 = pack2(scale_log2, scale_log2);
          const float cst = PRIOR ? bh - mu : -mu;
          const uint64_t c2 = pack2(cst, cst);
          // pass 2: p = 2^(s*scale - m) as bf16 pairs (S stays intact until
          // the pairs are stored, so a redo can read it again)
          acc = 0;
          {
            uint32_t v[32];
            ptx::tmem_ld32(tS, v);
            ptx::tmem_wait_ld();
            if (last) mask32<B>(v, half * 64, lim);
            exp_pack32(v, w0, s2, c2, acc);
            ptx::tmem_ld32(tS + 32, v);
            ptx::tmem_wait_ld();
            if (last) mask32<B>(v, half * 64 + 32, lim);
            exp_pack32(v, w1, s2, c2, acc);
          }
          if (!have_rmax) {
            if (!(ok = warp_wait_bar(&sh->mx_full[t], g & 1, abort))) break;
            rmax = fmaxf(pmb, sh->mx[g & 1][t][half ^ 1][r]);
            have_rmax = true;
          }
          // both halves of a row see the same rmax and m_used, so they decide
          // alike; the redo itself is warp-uniform (the loads and shuffles it
          // runs are warp-collective), rows that do not need it recompute the
          // same values
          const bool my_need = attempt == 0 && c > 0 && rmax > m_used + kSlack;
          if (my_need) {
            need = true;
            alpha = ex2_mufu(m_used - rmax);
            l *= alpha;
            m_used = rmax;
          }
          if (__any_sync(0xffffffffu, my_need)) continue;  // redo pass 2
          break;
        }
        if (!ok) break;
        // P words land on this half's first 32 S columns, all consumed by now
        ptx::tmem_st16(tS, w0);
        ptx::tmem_st16(tS + 16, w1);
        l += sum2(acc);
        if (__any_sync(0xffffffffu, need)) {
          // O must hold P.V of the previous chunk before it is rescaled (S of
          // this chunk was issued after it); P.V of this chunk is not issued
          // before this thread arrives on p_full.
          if (!(ok = warp_wait_bar(&sh->o_done[t], (g - 1) & 1, abort))) break;
          ptx::tc_fence_after();
#pragma unroll 1
          for (int q = 0; q < 2; ++q) {
            uint32_t ov[32];
            ptx::tmem_ld32(tO + q * 32, ov);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            ptx::tmem_st32(tO + q * 32, ov);
          }
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&sh->p_full[t]);
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      sh->lx[t][half][r] = l;
      ptx::mbar_arrive(&sh->l_full[t]);
      if (!(ok = warp_wait_bar(&sh->l_full[t], kq & 1, abort))) break;
      // S of the item's last chunk was issued after the P.V before it, so
      // o_done is at the phase of the last P.V or past it: one parity wait.
      if (!(ok = warp_wait_bar(&sh->o_done[t], (gc + nch - 1) & 1, abort))) break;
      ptx::tc_fence_after();
      const float lrow = sh->lx[t][0][r] + sh->lx[t][1][r];
      const float inv = 1.0f / lrow;
      const bool store = pos < N;
      __nv_bfloat16* orow = O + (((int64_t)it.b * Hq + h) * N + (store ? pos : 0)) * 128 + half * 64;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t ov[32];
        ptx::tmem_ld32(tO + q * 32, ov);
        ptx::tmem_wait_ld();
        uint32_t wv[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          wv[e] = cvt_bf16x2(__uint_as_float(ov[2 * e]) * inv, __uint_as_float(ov[2 * e + 1]) * inv);
        if (store) {
          if (o_al32) {
            // 32-byte stores: every write fills a whole sector
            st_global_v8(orow + q * 32, wv, 0);
            st_global_v8(orow + q * 32 + 16, wv, 8);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_uint4(wv[4 * e], wv[4 * e + 1], wv[4 * e + 2], wv[4 * e + 3]);
          }
        }
      }
      // O of this tile is read: the next item's first P.V may overwrite it
      ptx::tc_fence_before();
      ptx::mbar_arrive(&sh->o_free[t]);
      if (store && half == 0 && lse != nullptr)
        lse[((int64_t)it.b * Hq + h) * N + pos] = (m_used + log2f(lrow)) * 0.69314718055994530942f;
      gc += nch;
      ++kq;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- test hooks
// One thread waits on an mbarrier that nothing arrives on; the bounded wait
// expires and records SSA_ERR_TIMEOUT.
__global__ void wait_timeout_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    ptx::fence_mbar_init();
    abort_flag = 0;
    wait_bar(&bar, 0, &abort_flag, limit_ns);
  }
}

// ---------------------------------------------------------------- host side
namespace {

template <int B>
cudaError_t launch_tc_t(const void* Q, const void* K, const void* V, const int32_t* idx,
                        const int32_t* cnt, const float* bias, int batch, int Hq, int Hkv, int N,
                        int max_sel, float scale, void* O, float* lse, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_bf16_map(&mq, Q, 128, N, batch * Hq, 64) ||
      !make_bf16_map(&mk, K, 128, N, batch * Hkv, 64) ||
      !make_bf16_map(&mv, V, 128, N, batch * Hkv, 64))
    return cudaErrorInvalidValue;
  const int nq = (N + B - 1) / B;
  const int G = Hq / Hkv;
  const int subs = G / (2 * (128 / B));
  const long long items = (long long)nq * subs * batch * Hkv;
  if (items <= 0) return cudaSuccess;
  if (items > (1ll << 30)) return cudaErrorInvalidValue;
  const size_t smem = 1024 + kSmemBytes + sizeof(Shared);
  auto kern = bias != nullptr ? attn_tc_kernel<B, true> : attn_tc_kernel<B, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int grid = (int)(items < sms ? items : sms);  // one persistent CTA per SM
  // (batch, KV head) pairs per group of items: all of them while their K and
  // V fit in twice the L2 (126 MB), else two at a time
  const int nbg = batch * Hkv;
  const double kv_bytes = 2.0 * N * 128 * 2;  // K and V of one pair
  const int kvg = (nbg * kv_bytes <= 2.0 * 126e6) ? nbg : (nbg < 2 ? nbg : 2);
  kern<<<grid, kThreads, smem, st>>>(mq, mk, mv, idx, cnt, bias, (__nv_bfloat16*)O, lse,
                                                  Hq, Hkv, N, nq, nbg, max_sel,
                                                  scale * 1.4426950408889634f, kvg);
  return cudaGetLastError();
}

}  // namespace

bool attn_tc_supported(ssa_dtype dt, int Hq, int Hkv, int d, int B) {
  if (dt != SSA_BF16 || d != 128 || (B != 64 && B != 128)) return false;
  if (Hkv <= 0 || Hq % Hkv != 0) return false;
  return ((Hq / Hkv) * B) % 256 == 0;
}

cudaError_t launch_attn_tc(const void* Q, const void* K, const void* V, const int32_t* idx,
                           const int32_t* cnt, const float* bias, int batch, int Hq, int Hkv,
                           int N, int B, int max_sel, float scale, void* O, float* lse,
                           cudaStream_t st) {
  if (max_sel > 8192) return cudaErrorInvalidValue;
  return B == 64 ? launch_tc_t<64>(Q, K, V, idx, cnt, bias, batch, Hq, Hkv, N, max_sel, scale, O,
                                   lse, st)
                 : launch_tc_t<128>(Q, K, V, idx, cnt, bias, batch, Hq, Hkv, N, max_sel, scale, O,
                                    lse, st);
}

cudaError_t attn_tc_error_word(int** word) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(word), g_attn_tc_error);
}

int read_and_reset_attn_tc_error() {
  int v = 0;
  cudaMemcpyFromSymbol(&v, g_attn_tc_error, sizeof(int));
  const int z = 0;
  cudaMemcpyToSymbol(g_attn_tc_error, &z, sizeof(int));
  return v;
}

}  // namespace ssa

extern "C" ssa_status ssa_debug_wait_timeout(int limit_us, ssa_stream stream) {
  if (limit_us < 1 || limit_us > 1000000) return SSA_ERR_INVALID_ARG;
  ssa::wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      (unsigned long long)limit_us * 1000ull);
  return cudaGetLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}
