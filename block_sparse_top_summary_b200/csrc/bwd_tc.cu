// The backward pass of stage 2 on the tensor cores (tcgen05 + TMA + TMEM), the
// gradients with the selection held fixed (DashAttention page, "Declaração do
// Problema" 2; SSA page, "1. Definição do Problema" 2).
//
// ---- dQ
// Work item (as in the tcgen05 forward): the 256 query rows that share one
// selection, (batch, KV head g, query block i, group of 256/B query heads),
// as two M-tiles of 128 rows.  The selected blocks are visited in chunks of
// 64 keys (one block at B = 64, half a block at B = 128).  Per chunk and tile:
//   S  = Q K^T,  dP = dO V^T        (M = 128, N = 64, K = d; A and B from smem)
//   dS = exp2(S c - lse2) * (dP - delta)   (one thread per row, fp32, into
//        bf16 pairs over the first 32 columns of S)
//   dQ += dS K                      (A = dS from TMEM, B = K MN-major)
// TMEM (512 columns): tile t: S at 128 t, dP at 128 t + 64, dQ at 256 + 128 t.
// Roles (320 threads): warp 0 TMA producer (Q and dO of the item, then K and V
// of each chunk into a 2-stage ring); warp 1 TMEM owner and MMA issuer (one
// thread), which alternates the tiles so that one tile's dS is formed while
// the other tile's MMAs run; warps 2-5 tile 0, 6-9 tile 1, one thread per row
// (TMEM lane).
// One work item per CTA.  Every mbarrier wait is bounded; on expiry the CTA
// records SSA_ERR_TIMEOUT, stops issuing, drains what it issued and frees TMEM.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "tmap.h"

namespace ssa {

__device__ int g_bwd_tc_error = 0;

namespace {

constexpr int kThreadsTc = 320;
constexpr uint32_t kTileBytes = 32768;   // 128 rows x 128 d x 2 B
constexpr uint32_t kChunkBytes = 16384;  // 64 keys x 128 d x 2 B (K or V)
constexpr uint32_t kTmemColsTc = 512;
constexpr unsigned long long kWaitNsTc = 1000000000ull;
constexpr float kLog2eTc = 1.4426950408889634f;

struct __align__(8) SharedTc {
  uint64_t q_full;      // Q and dO of the item have landed
  uint64_t kv_full[2];  // K and V of a chunk have landed
  uint64_t kv_empty[2]; // the chunk's MMAs are done with K and V
  uint64_t s_full[2];   // per tile: S and dP of the chunk are in TMEM
  uint64_t p_full[2];   // per tile: dS of the chunk is in TMEM (128 arrivals)
  uint64_t o_done;      // every dQ MMA has completed
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool wait_tc(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = gtimer();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort) return false;
      if (gtimer() - t0 > kWaitNsTc) {
        *abort = 1;
        atomicCAS(&g_bwd_tc_error, 0, (int)SSA_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool warp_wait_tc(uint64_t* bar, uint32_t parity, volatile int* abort) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = wait_tc(bar, parity, abort) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) ptx::mbar_try_wait(bar, parity);
  return ok != 0;
}

__device__ __forceinline__ uint64_t sdesc_tc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) |
         ((uint64_t)(sbo >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// kind::f16, bf16 x bf16 -> f32, M = 128: N = 64 (S, dP), N = 128 with B MN-major (dQ)
constexpr uint32_t kIdescN64 = (1u << 4) | (1u << 7) | (1u << 10) | ((64u >> 3) << 17) |
                               ((128u >> 4) << 24);
constexpr uint32_t kIdescDQ = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) |
                              ((128u >> 4) << 24) | (1u << 16);

__device__ __forceinline__ uint32_t pack_bf16_tc(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

}  // namespace

template <int B>
__global__ void __launch_bounds__(kThreadsTc, 1) bwd_dq_tc_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmG,
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const float* __restrict__ lse, const float* __restrict__ delta,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt, int Hq, int Hkv, int N,
    int nq, int max_sel, float scale, __nv_bfloat16* __restrict__ dQ) {
  constexpr int HPT = 128 / B;  // query heads per M-tile
  constexpr int HPI = 2 * HPT;  // query heads per work item
  constexpr int CPB = B / 64;   // 64-key chunks per block
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* Qs = base;                       // 2 tiles
  unsigned char* Gs = Qs + 2 * kTileBytes;        // dO, 2 tiles
  unsigned char* Ks = Gs + 2 * kTileBytes;        // 2 stages
  unsigned char* Vs = Ks + 2 * kChunkBytes;       // 2 stages
  SharedTc* sh = reinterpret_cast<SharedTc*>(Vs + 2 * kChunkBytes);

  const int G = Hq / Hkv;
  const int subs = G / HPI;
  // item: query block i (late blocks first), (batch, KV head), head group
  const int w = blockIdx.x;
  const int nbg = gridDim.x / (nq * subs);
  const int per_i = subs * nbg;
  const int i = nq - 1 - w / per_i;
  const int rem = w - (w / per_i) * per_i;
  const int bg = rem / subs;
  const int sub = rem - bg * subs;
  const int b = bg / Hkv, g = bg - b * Hkv;
  const int h0 = g * G + sub * HPI;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &sh->abort;
  const int ns = min(max(cnt[(int64_t)bg * nq + i], 0), max_sel);
  const int32_t* row = idx + ((int64_t)bg * nq + i) * max_sel;
  const int nch = ns * CPB;

  if (threadIdx.x == 0) {
    ptx::mbar_init(&sh->q_full, 1);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&sh->kv_full[s], 1);
      ptx::mbar_init(&sh->kv_empty[s], 1);
      ptx::mbar_init(&sh->s_full[s], 1);
      ptx::mbar_init(&sh->p_full[s], 128);
    }
    ptx::mbar_init(&sh->o_done, 1);
    ptx::mbar_init(&sh->drain, 1);
    sh->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&sh->tmem_base, kTmemColsTc);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int issued = 0;
    bool ok = true;
    if (lane == 0 && nch > 0) {
      ptx::mbar_arrive_expect_tx(&sh->q_full, 4 * kTileBytes);
      for (int t = 0; t < 2; ++t)
        for (int hh = 0; hh < HPT; ++hh)
          for (int rg = 0; rg < B / 64; ++rg)
            for (int c = 0; c < 2; ++c) {
              const uint32_t off = t * kTileBytes + c * 16384 + (hh * B + rg * 64) * 128;
              const int z = b * Hq + h0 + t * HPT + hh;
              ptx::tma_load_3d(Qs + off, &tmQ, c * 64, i * B + rg * 64, z, &sh->q_full);
              ptx::tma_load_3d(Gs + off, &tmG, c * 64, i * B + rg * 64, z, &sh->q_full);
            }
    }
    for (int c = 0; ok && c < nch; ++c) {
      const int s = c & 1;
      if (c >= 2 && !(ok = warp_wait_tc(&sh->kv_empty[s], ((c >> 1) - 1) & 1, abort))) break;
      if (lane == 0) {
        const int j = row[c / CPB];
        const int y = j * B + (c % CPB) * 64;
        ptx::mbar_arrive_expect_tx(&sh->kv_full[s], 2 * kChunkBytes);
        for (int cc = 0; cc < 2; ++cc) {
          ptx::tma_load_3d(Ks + s * kChunkBytes + cc * 8192, &tmK, cc * 64, y, bg, &sh->kv_full[s]);
          ptx::tma_load_3d(Vs + s * kChunkBytes + cc * 8192, &tmV, cc * 64, y, bg, &sh->kv_full[s]);
        }
      }
      issued = c + 1;
    }
    if (lane == 0) {
      // every issued copy lands before the CTA's shared memory goes away
      volatile int no_abort = 0;
      for (int c = (issued > 2 ? issued - 2 : 0); c < issued; ++c)
        wait_tc(&sh->kv_full[c & 1], (c >> 1) & 1, &no_abort);
      if (nch > 0) wait_tc(&sh->q_full, 0, &no_abort);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t qa = ptx::smem_u32(Qs), ga = ptx::smem_u32(Gs);
      const uint32_t ka = ptx::smem_u32(Ks), va = ptx::smem_u32(Vs);
      bool ok = nch == 0 || wait_tc(&sh->q_full, 0, abort);
      // S and dP of tile t for chunk c into TMEM (commits s_full[t])
      auto issue_sdp = [&](int t, int c) {
        const int s = c & 1;
        ptx::tc_fence_after();
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t oq = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t ok2 = (kk >> 2) * 8192 + (kk & 3) * 32;
          ptx::mma_ss(tmem + t * 128, sdesc_tc(qa + t * kTileBytes + oq, 16, 1024),
                      sdesc_tc(ka + s * kChunkBytes + ok2, 16, 1024), kIdescN64, kk > 0);
          ptx::mma_ss(tmem + t * 128 + 64, sdesc_tc(ga + t * kTileBytes + oq, 16, 1024),
                      sdesc_tc(va + s * kChunkBytes + ok2, 16, 1024), kIdescN64, kk > 0);
        }
        ptx::mma_commit(&sh->s_full[t]);
      };
      // dQ_t += dS_t K of chunk c (A = dS from TMEM, B = K MN-major)
      auto issue_dq = [&](int t, int c) {
        const int s = c & 1;
        ptx::tc_fence_after();
        for (int kk = 0; kk < 4; ++kk)
          ptx::mma_ts(tmem + 256 + t * 128, tmem + t * 128 + kk * 8,
                      sdesc_tc(ka + s * kChunkBytes + kk * 2048, 8192, 1024), kIdescDQ,
                      (c > 0 || kk > 0) ? 1u : 0u);
      };
      // The two tiles alternate: while one tile's dS is formed, the tensor
      // cores run the other tile's dQ and next S / dP.  S / dP of chunk c + 1
      // overwrite dS of chunk c, so they are issued after that dQ (MMAs of
      // one thread run in issue order).
      if (ok && nch > 0) {
        if ((ok = wait_tc(&sh->kv_full[0], 0, abort))) {
          issue_sdp(0, 0);
          issue_sdp(1, 0);
        }
      }
      for (int c = 0; ok && c < nch; ++c) {
        const int s = c & 1;
        const bool more = c + 1 < nch;
        if (!(ok = wait_tc(&sh->p_full[0], c & 1, abort))) break;
        issue_dq(0, c);
        if (more) {
          if (!(ok = wait_tc(&sh->kv_full[(c + 1) & 1], ((c + 1) >> 1) & 1, abort))) break;
          issue_sdp(0, c + 1);
        }
        if (!(ok = wait_tc(&sh->p_full[1], c & 1, abort))) break;
        issue_dq(1, c);
        ptx::mma_commit(&sh->kv_empty[s]);  // K(c), V(c) read by every MMA of chunk c
        if (more) issue_sdp(1, c + 1);
      }
      if (ok && nch > 0) ptx::mma_commit(&sh->o_done);
      // every issued MMA completes before TMEM is freed
      ptx::mma_commit(&sh->drain);
      volatile int no_abort = 0;
      wait_tc(&sh->drain, 0, &no_abort);
    }
  } else {
    // ------------------------------------------------------------ dS rows
    const int t = (warp - 2) >> 2;
    const int quarter = warp & 3;        // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;   // row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tQ = tmem + lane_off + 256 + t * 128;
    const int hh = r / B;
    const int pos = i * B + (r % B);
    const int h = h0 + t * HPT + hh;
    const int64_t rowi = ((int64_t)b * Hq + h) * N + pos;
    const bool valid = pos < N;
    const float l2 = valid ? lse[rowi] * kLog2eTc : INFINITY;
    const float dl = valid ? delta[rowi] : 0.f;
    const uint64_t c2 = ptx::f2_pack(scale * kLog2eTc, scale * kLog2eTc);
    const uint64_t nl2 = ptx::f2_pack(-l2, -l2), ndl = ptx::f2_pack(-dl, -dl);
    bool ok = true;
    for (int c = 0; c < nch; ++c) {
      if (!(ok = warp_wait_tc(&sh->s_full[t], c & 1, abort))) break;
      ptx::tc_fence_after();
      const int k0 = row[c / CPB] * B + (c % CPB) * 64;  // first key of the chunk
      uint32_t wv[32];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t sv[32], pv[32];
        ptx::tmem_ld32(tS + q * 32, sv);
        ptx::tmem_ld32(tS + 64 + q * 32, pv);
        ptx::tmem_wait_ld();
        const int kmax = pos - k0 - q * 32;  // columns past it are keys after the query
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float p0, p1, d0, d1;
          ptx::f2_unpack(ptx::f2_fma(ptx::f2_pack(__uint_as_float(sv[2 * e]),
                                                  __uint_as_float(sv[2 * e + 1])),
                                     c2, nl2),
                         p0, p1);
          p0 = 2 * e <= kmax ? ptx::ex2_ftz(p0) : 0.f;
          p1 = 2 * e + 1 <= kmax ? ptx::ex2_ftz(p1) : 0.f;
          ptx::f2_unpack(ptx::f2_mul(ptx::f2_pack(p0, p1),
                                     ptx::f2_add(ptx::f2_pack(__uint_as_float(pv[2 * e]),
                                                              __uint_as_float(pv[2 * e + 1])),
                                                 ndl)),
                         d0, d1);
          wv[q * 16 + e] = pack_bf16_tc(d0, d1);
        }
      }
      // dS words over the first 32 S columns of this row (already read)
      uint32_t w0[16], w1[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        w0[e] = wv[e];
        w1[e] = wv[16 + e];
      }
      ptx::tmem_st16(tS, w0);
      ptx::tmem_st16(tS + 16, w1);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&sh->p_full[t]);
    }
    if (ok && nch > 0 && warp_wait_tc(&sh->o_done, 0, abort)) {
      ptx::tc_fence_after();
      __nv_bfloat16* out = dQ + rowi * 128;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t ov[32];
        ptx::tmem_ld32(tQ + q * 32, ov);
        ptx::tmem_wait_ld();
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(out + q * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(
                pack_bf16_tc(__uint_as_float(ov[8 * e]) * scale, __uint_as_float(ov[8 * e + 1]) * scale),
                pack_bf16_tc(__uint_as_float(ov[8 * e + 2]) * scale, __uint_as_float(ov[8 * e + 3]) * scale),
                pack_bf16_tc(__uint_as_float(ov[8 * e + 4]) * scale, __uint_as_float(ov[8 * e + 5]) * scale),
                pack_bf16_tc(__uint_as_float(ov[8 * e + 6]) * scale, __uint_as_float(ov[8 * e + 7]) * scale));
        }
      }
    } else if (valid && nch == 0) {
      // no selected block: the row's gradient is zero
      uint4* dst = reinterpret_cast<uint4*>(dQ + rowi * 128);
      for (int e = 0; e < 16; ++e) dst[e] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemColsTc);
  }
}

// Host side: maps and launch.  Shapes as attn_tc_supported: bf16, d = 128,
// B in {64, 128}, (Hq / Hkv) * B a multiple of 256.
cudaError_t launch_bwd_dq_tc(const void* Q, const void* K, const void* V, const void* dO,
                             const float* lse, const float* delta, const int32_t* idx,
                             const int32_t* cnt, int batch, int Hq, int Hkv, int N, int B,
                             int max_sel, float scale, void* dQ, cudaStream_t st) {
  CUtensorMap mq, mg, mk, mv;
  if (!make_bf16_map(&mq, Q, 128, N, batch * Hq, 64) ||
      !make_bf16_map(&mg, dO, 128, N, batch * Hq, 64) ||
      !make_bf16_map(&mk, K, 128, N, batch * Hkv, 64) ||
      !make_bf16_map(&mv, V, 128, N, batch * Hkv, 64))
    return cudaErrorInvalidValue;
  const int nq = (N + B - 1) / B;
  const int G = Hq / Hkv;
  const int subs = G / (2 * (128 / B));
  const long long items = (long long)batch * Hkv * nq * subs;
  if (items <= 0) return cudaSuccess;
  const size_t smem = 1024 + 4 * (size_t)kTileBytes + 4 * (size_t)kChunkBytes + sizeof(SharedTc);
  cudaError_t e;
  if (B == 64) {
    e = cudaFuncSetAttribute(bwd_dq_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    bwd_dq_tc_kernel<64><<<(unsigned)items, kThreadsTc, smem, st>>>(
        mq, mg, mk, mv, lse, delta, idx, cnt, Hq, Hkv, N, nq, max_sel, scale,
        (__nv_bfloat16*)dQ);
  } else {
    e = cudaFuncSetAttribute(bwd_dq_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    bwd_dq_tc_kernel<128><<<(unsigned)items, kThreadsTc, smem, st>>>(
        mq, mg, mk, mv, lse, delta, idx, cnt, Hq, Hkv, N, nq, max_sel, scale,
        (__nv_bfloat16*)dQ);
  }
  return cudaGetLastError();
}

cudaError_t bwd_tc_error_word(int** word) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(word), g_bwd_tc_error);
}

int read_and_reset_bwd_tc_error() {
  int v = 0;
  cudaMemcpyFromSymbol(&v, g_bwd_tc_error, sizeof(int));
  const int z = 0;
  cudaMemcpyToSymbol(g_bwd_tc_error, &z, sizeof(int));
  return v;
}


// ---------------------------------------------------------------- dK, dV
// One CTA per (batch, KV head, key block j) at B = 64, over every query block
// i whose selection holds j, 128 query rows (two heads) per step:
//   S = Q K^T, dP = dO V^T      (M = 128 rows, N = 64 keys) into TMEM, 2 buffers
//   P, dS as bf16 rows (128-byte swizzle) into shared memory, 2 buffers
//   dV^T += dO^T P, dK^T += Q^T dS   (M = d = 128, N = 64; A and B MN-major)
// Roles (320 threads): warp 0 TMA producer (K and V once, Q and dO per step
// into a 2-stage ring); warp 1 TMEM owner and MMA issuer, S and dP one step
// ahead of dV and dK; warps 2-9 form P and dS, two warps per TMEM lane
// quarter, one per half of the keys, so a step's P and dS are formed while
// the previous step's dV / dK MMAs run.

namespace {

constexpr int kThreadsKv = 320;
constexpr uint32_t kTile = 32768;    // 128 rows x 128 d x 2 B (Q or dO)
constexpr uint32_t kBlk = 16384;     // 64 keys x 128 d x 2 B (K or V)
constexpr uint32_t kPd = 16384;      // 128 query rows x 64 keys x 2 B (P or dS)
constexpr unsigned long long kWaitKv = 1000000000ull;
constexpr float kL2e = 1.4426950408889634f;

struct __align__(8) SharedKv {
  uint64_t kv_full;
  uint64_t qd_full[2], qd_empty[2];
  uint64_t s_full[2];
  uint64_t pd_full[2];   // P and dS of the step are in shared memory (256 arrivals)
  uint64_t pd_empty[2];  // the step's dV / dK MMAs are done reading them
  uint64_t done, drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ unsigned long long gt() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool wkv(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = gt();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort) return false;
      if (gt() - t0 > kWaitKv) {
        *abort = 1;
        atomicCAS(&g_bwd_tc_error, 0, (int)SSA_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool warp_wkv(uint64_t* bar, uint32_t parity, volatile int* abort) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = wkv(bar, parity, abort) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) ptx::mbar_try_wait(bar, parity);
  return ok != 0;
}

__device__ __forceinline__ uint64_t sd(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) |
         ((uint64_t)(sbo >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// kind::f16, bf16 -> f32, M = 128, N = 64; the second with A and B MN-major
constexpr uint32_t kIdS = (1u << 4) | (1u << 7) | (1u << 10) | ((64u >> 3) << 17) |
                          ((128u >> 4) << 24);
constexpr uint32_t kIdT = kIdS | (1u << 15) | (1u << 16);

__device__ __forceinline__ uint32_t pk(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

}  // namespace

__global__ void __launch_bounds__(kThreadsKv, 1) bwd_dkv_tc_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmG,
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const float* __restrict__ lse, const float* __restrict__ delta, int batch, int Hq, int Hkv,
    int N, int nq, float scale, __nv_bfloat16* __restrict__ dK, __nv_bfloat16* __restrict__ dV,
    float* __restrict__ sink_part, int sink_qr, int sink_nsplit,
    const uint32_t* __restrict__ hitmask, int nwin) {
  constexpr int B = 64;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* Ks = base;
  unsigned char* Vs = Ks + kBlk;
  unsigned char* Qs = Vs + kBlk;          // 2 stages
  unsigned char* Gs = Qs + 2 * kTile;     // 2 stages
  unsigned char* Ps = Gs + 2 * kTile;     // P, 2 buffers
  unsigned char* Ds = Ps + 2 * kPd;       // dS, 2 buffers
  SharedKv* sh = reinterpret_cast<SharedKv*>(Ds + 2 * kPd);

  const int nbg = batch * Hkv;
  // The CTAs of one (batch, KV head) pair are consecutive, so the Q and dO
  // tiles that the running CTAs re-read are one pair's (L2-sized) rather than
  // every pair's.  Within a pair: sink_nsplit CTAs take the sink column (key
  // block 0, in every selection) in ranges of sink_qr query blocks and write
  // fp32 partial sums; then one CTA per key block j >= 1 over every query
  // block i >= j, early (most selected) blocks first.
  const int per_bg = sink_nsplit + nq - 1;
  const int bg = blockIdx.x / per_bg;
  const int r_bg = blockIdx.x - bg * per_bg;
  const bool sink = r_bg < sink_nsplit;
  const int rg = r_bg;  // sink range (sink CTAs only)
  int j, i_lo, i_hi;
  if (sink) {
    j = 0;
    i_lo = rg * sink_qr;
    i_hi = min(nq, i_lo + sink_qr);
  } else {
    j = 1 + (r_bg - sink_nsplit);
    i_lo = j;
    i_hi = nq;
  }
  const int b = bg / Hkv, g = bg - b * Hkv;
  const int G = Hq / Hkv;
  const int tiles = G / 2;  // 128-row tiles per query block: two heads each
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &sh->abort;
  const uint32_t* mrow = hitmask + ((int64_t)bg * nq + j) * nwin;
  auto win_bits = [&](int base) -> unsigned {
    unsigned m = __ldg(mrow + (base >> 5));
    const int lo = i_lo - base, hi = i_hi - base;
    if (lo > 0) m &= lo >= 32 ? 0u : (~0u << lo);
    if (hi < 32) m &= hi <= 0 ? 0u : ((1u << hi) - 1u);
    return m;
  };

  if (threadIdx.x == 0) {
    ptx::mbar_init(&sh->kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&sh->qd_full[s], 1);
      ptx::mbar_init(&sh->qd_empty[s], 1);
      ptx::mbar_init(&sh->s_full[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&sh->pd_full[s], 256);
      ptx::mbar_init(&sh->pd_empty[s], 1);
    }
    ptx::mbar_init(&sh->done, 1);
    ptx::mbar_init(&sh->drain, 1);
    sh->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&sh->tmem_base, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::mbar_arrive_expect_tx(&sh->kv_full, 2 * kBlk);
      for (int cc = 0; cc < 2; ++cc) {
        ptx::tma_load_3d(Ks + cc * 8192, &tmK, cc * 64, j * B, bg, &sh->kv_full);
        ptx::tma_load_3d(Vs + cc * 8192, &tmV, cc * 64, j * B, bg, &sh->kv_full);
      }
    }
    int n = 0;
    bool ok = true;
    for (int base_i = i_lo & ~31; ok && base_i < i_hi; base_i += 32) {
      unsigned m = win_bits(base_i);
      while (ok && m) {
        const int i = base_i + __ffs(m) - 1;
        m &= m - 1;
        for (int tt = 0; ok && tt < tiles; ++tt, ++n) {
          const int s = n & 1;
          if (n >= 2 && !(ok = warp_wkv(&sh->qd_empty[s], ((n >> 1) - 1) & 1, abort))) break;
          if (lane == 0) {
            ptx::mbar_arrive_expect_tx(&sh->qd_full[s], 2 * kTile);
            for (int hh = 0; hh < 2; ++hh)
              for (int c = 0; c < 2; ++c) {
                const uint32_t off = s * kTile + c * 16384 + hh * B * 128;
                const int z = b * Hq + g * G + tt * 2 + hh;
                ptx::tma_load_3d(Qs + off, &tmQ, c * 64, i * B, z, &sh->qd_full[s]);
                ptx::tma_load_3d(Gs + off, &tmG, c * 64, i * B, z, &sh->qd_full[s]);
              }
          }
        }
      }
    }
    if (lane == 0) {
      volatile int no_abort = 0;
      for (int c = (n > 2 ? n - 2 : 0); c < n; ++c) wkv(&sh->qd_full[c & 1], (c >> 1) & 1, &no_abort);
      wkv(&sh->kv_full, 0, &no_abort);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t ka = ptx::smem_u32(Ks), va = ptx::smem_u32(Vs);
    const uint32_t qa = ptx::smem_u32(Qs), ga = ptx::smem_u32(Gs);
    const uint32_t pa = ptx::smem_u32(Ps), da = ptx::smem_u32(Ds);
    bool ok = warp_wkv(&sh->kv_full, 0, abort);
    int n = 0;  // steps whose S / dP are issued
    int m_done = 0;  // steps whose dV / dK are issued
    auto issue_s = [&](int st) {
      const int s = st & 1;
      if (lane == 0) {
        ptx::tc_fence_after();
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t oq = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t okv = (kk >> 2) * 8192 + (kk & 3) * 32;
          ptx::mma_ss(tmem + s * 128, sd(qa + s * kTile + oq, 16, 1024), sd(ka + okv, 16, 1024),
                      kIdS, kk > 0);
          ptx::mma_ss(tmem + s * 128 + 64, sd(ga + s * kTile + oq, 16, 1024),
                      sd(va + okv, 16, 1024), kIdS, kk > 0);
        }
        ptx::mma_commit(&sh->s_full[s]);
      }
      __syncwarp();
    };
    auto issue_dkv = [&](int st) {
      const int s = st & 1;
      if (lane == 0) {
        ptx::tc_fence_after();
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t acc = (st > 0 || kk > 0) ? 1u : 0u;
          ptx::mma_ss(tmem + 256, sd(ga + s * kTile + kk * 2048, 16384, 1024),
                      sd(pa + s * kPd + kk * 2048, 16384, 1024), kIdT, acc);
          ptx::mma_ss(tmem + 320, sd(qa + s * kTile + kk * 2048, 16384, 1024),
                      sd(da + s * kPd + kk * 2048, 16384, 1024), kIdT, acc);
        }
        ptx::mma_commit(&sh->pd_empty[s]);
        ptx::mma_commit(&sh->qd_empty[s]);
      }
      __syncwarp();
    };
    // S / dP of a step are issued once its Q and dO have landed and its TMEM
    // buffer is free (the P / dS of step n - 2 formed); dV / dK of a step once
    // its P and dS are in shared memory.  Neither waits for the other, so the
    // Q / dO stage of step n is released (its dV / dK done) while the load of
    // step n + 1 is still in flight.  Query blocks are found 32 at a time.
    int known = 0;                // steps found so far
    int next_i = i_lo & ~31;      // first query block not yet scanned
    unsigned long long t_last = 0;
    uint32_t idle = 0;
    while (ok) {
      if (n >= known && next_i < i_hi) {
        known += __popc(win_bits(next_i)) * tiles;
        next_i += 32;
        continue;
      }
      if (m_done >= known) break;  // every window scanned, every step issued
      bool progress = false;
      if (n < known && n <= m_done + 1) {
        int rdy = 0;
        if (lane == 0) rdy = ptx::mbar_test_wait(&sh->qd_full[n & 1], (n >> 1) & 1) ? 1 : 0;
        if (__shfl_sync(0xffffffffu, rdy, 0)) {
          issue_s(n);
          ++n;
          progress = true;
        }
      }
      if (m_done < n) {
        int rdy = 0;
        if (lane == 0) rdy = ptx::mbar_test_wait(&sh->pd_full[m_done & 1], (m_done >> 1) & 1) ? 1 : 0;
        if (__shfl_sync(0xffffffffu, rdy, 0)) {
          issue_dkv(m_done);
          ++m_done;
          progress = true;
        }
      }
      if (progress) {
        idle = 0;
      } else if ((++idle & 255u) == 1u) {
        int stop = 0;
        if (lane == 0) {
          const unsigned long long now = gt();
          if (idle == 1u) t_last = now;
          if (*abort) {
            stop = 1;
          } else if (now - t_last > kWaitKv) {
            *abort = 1;
            atomicCAS(&g_bwd_tc_error, 0, (int)SSA_ERR_TIMEOUT);
            stop = 1;
          }
        }
        if (__shfl_sync(0xffffffffu, stop, 0)) ok = false;
      }
    }
    if (lane == 0) {
      if (ok && n > 0) ptx::mma_commit(&sh->done);
      ptx::mma_commit(&sh->drain);
      volatile int no_abort = 0;
      wkv(&sh->drain, 0, &no_abort);
    }
  } else {
    // ------------------------------------------------------------ query rows
    // warps 2-9: two warps per TMEM lane quarter, each taking half of the
    // step's 64 keys (q = key half)
    const int quarter = warp & 3;
    const int q = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;  // query row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint64_t c2 = ptx::f2_pack(scale * kL2e, scale * kL2e);
    // Steps in issue order: query blocks i ascending (set bits of the hit
    // mask), then the two-head tiles t of each.  The next step's lse and
    // delta are loaded one step ahead, so their latency overlaps this step.
    int base = i_lo & ~31;
    unsigned m = base < i_hi ? win_bits(base) : 0u;
    int i = -1, t = tiles - 1;
    auto advance = [&]() {
      if (i >= 0 && t + 1 < tiles) {
        ++t;
        return;
      }
      t = 0;
      while (m == 0u) {
        base += 32;
        if (base >= i_hi) {
          i = -1;
          return;
        }
        m = win_bits(base);
      }
      i = base + __ffs(m) - 1;
      m &= m - 1;
    };
    auto row_of = [&](int ii, int tt) -> int64_t {
      return ((int64_t)b * Hq + g * G + tt * 2 + r / B) * N + ii * B + (r % B);
    };
    advance();
    float lse_n = 0.f, dl_n = 0.f;
    bool valid_n = false;
    if (i >= 0) {
      valid_n = i * B + (r % B) < N;
      if (valid_n) {
        lse_n = lse[row_of(i, t)];
        dl_n = delta[row_of(i, t)];
      }
    }
    int n = 0;
    bool ok = true;
    while (ok && i >= 0) {
      const int ci = i, s = n & 1;
      const int pos = ci * B + (r % B);
      const float l2 = valid_n ? lse_n * kL2e : INFINITY;
      const float dl = valid_n ? dl_n : 0.f;
      advance();
      if (i >= 0) {
        valid_n = i * B + (r % B) < N;
        if (valid_n) {
          lse_n = lse[row_of(i, t)];
          dl_n = delta[row_of(i, t)];
        }
      }
      if (!(ok = warp_wkv(&sh->s_full[s], (n >> 1) & 1, abort))) break;
      // the dV / dK MMAs of step n - 2 are done with this P / dS buffer
      if (n >= 2 && !(ok = warp_wkv(&sh->pd_empty[s], ((n >> 1) - 1) & 1, abort))) break;
      ptx::tc_fence_after();
      unsigned char* prow = Ps + s * kPd + r * 128;
      unsigned char* drow = Ds + s * kPd + r * 128;
      uint32_t sv[32], pv[32], pw[16], dw[16];
      ptx::tmem_ld32(tmem + lane_off + s * 128 + q * 32, sv);
      ptx::tmem_ld32(tmem + lane_off + s * 128 + 64 + q * 32, pv);
      ptx::tmem_wait_ld();
      // only the diagonal block (i = j) has keys after the query
      const int kmax = ci == j ? pos - j * B - q * 32 : 64;
      const uint64_t nl2 = ptx::f2_pack(-l2, -l2), ndl = ptx::f2_pack(-dl, -dl);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        float p0, p1, d0, d1;
        ptx::f2_unpack(ptx::f2_fma(ptx::f2_pack(__uint_as_float(sv[2 * e]),
                                                __uint_as_float(sv[2 * e + 1])),
                                   c2, nl2),
                       p0, p1);
        p0 = 2 * e <= kmax ? ptx::ex2_ftz(p0) : 0.f;
        p1 = 2 * e + 1 <= kmax ? ptx::ex2_ftz(p1) : 0.f;
        const uint64_t pp = ptx::f2_pack(p0, p1);
        ptx::f2_unpack(ptx::f2_mul(pp, ptx::f2_add(ptx::f2_pack(__uint_as_float(pv[2 * e]),
                                                                __uint_as_float(pv[2 * e + 1])),
                                                   ndl)),
                       d0, d1);
        pw[e] = pk(p0, p1);
        dw[e] = pk(d0, d1);
      }
      // keys 32 q .. 32 q + 31 are 16-byte chunks 4 q .. 4 q + 3 of the row
#pragma unroll
      for (int cl = 0; cl < 4; ++cl) {
        const int sc = ((4 * q + cl) ^ (r & 7)) << 4;
        *reinterpret_cast<uint4*>(prow + sc) =
            make_uint4(pw[4 * cl], pw[4 * cl + 1], pw[4 * cl + 2], pw[4 * cl + 3]);
        *reinterpret_cast<uint4*>(drow + sc) =
            make_uint4(dw[4 * cl], dw[4 * cl + 1], dw[4 * cl + 2], dw[4 * cl + 3]);
      }
      ptx::fence_proxy_async_smem();  // generic writes before the MMAs read them
      ptx::tc_fence_before();
      ptx::mbar_arrive(&sh->pd_full[s]);
      ++n;
    }
    // ---- epilogue: lane = d; dV[key][d] = dV^T[d][key], dK likewise (times scale)
    // (a key block that no query block selects gets zeros)
    const bool have = ok && n > 0 && warp_wkv(&sh->done, 0, abort);
    if (have || (ok && n == 0)) {
      const int dd = r;
      {
        uint32_t vv[32], kv[32];
        if (have) {
          ptx::tc_fence_after();
          ptx::tmem_ld32(tmem + lane_off + 256 + q * 32, vv);
          ptx::tmem_ld32(tmem + lane_off + 320 + q * 32, kv);
          ptx::tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) vv[e] = kv[e] = 0u;
        }
        if (sink) {
          float* pk = sink_part + ((size_t)rg * nbg + bg) * 2 * B * 128;
          float* pv = pk + (size_t)B * 128;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int key = q * 32 + e;  // row of block 0
            pv[key * 128 + dd] = __uint_as_float(vv[e]);
            pk[key * 128 + dd] = __uint_as_float(kv[e]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int key = j * B + q * 32 + e;
            if (key < N) {
              const int64_t o = ((int64_t)bg * N + key) * 128 + dd;
              dV[o] = __float2bfloat16_rn(__uint_as_float(vv[e]));
              dK[o] = __float2bfloat16_rn(__uint_as_float(kv[e]) * scale);
            }
          }
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_bwd_dkv_tc(const void* Q, const void* K, const void* V, const void* dO,
                              const float* lse, const float* delta, int batch, int Hq, int Hkv,
                              int N, float scale, void* dK, void* dV, float* sink_part,
                              int sink_qr, int sink_nsplit, const uint32_t* hitmask, int nwin,
                              cudaStream_t st) {
  CUtensorMap mq, mg, mk, mv;
  if (!make_bf16_map(&mq, Q, 128, N, batch * Hq, 64) ||
      !make_bf16_map(&mg, dO, 128, N, batch * Hq, 64) ||
      !make_bf16_map(&mk, K, 128, N, batch * Hkv, 64) ||
      !make_bf16_map(&mv, V, 128, N, batch * Hkv, 64))
    return cudaErrorInvalidValue;
  const int nq = (N + 63) / 64;
  const long long ctas = (long long)batch * Hkv * (sink_nsplit + nq - 1);
  if (ctas <= 0) return cudaSuccess;
  const size_t smem = 1024 + 2 * (size_t)kBlk + 4 * (size_t)kTile + 4 * (size_t)kPd + sizeof(SharedKv);
  cudaError_t e = cudaFuncSetAttribute(bwd_dkv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  bwd_dkv_tc_kernel<<<(unsigned)ctas, kThreadsKv, smem, st>>>(
      mq, mg, mk, mv, lse, delta, batch, Hq, Hkv, N, nq, scale, (__nv_bfloat16*)dK,
      (__nv_bfloat16*)dV, sink_part, sink_qr, sink_nsplit, hitmask, nwin);
  return cudaGetLastError();
}

}  // namespace ssa
