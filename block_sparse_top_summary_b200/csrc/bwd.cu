// Backward pass of stage 2 (block-sparse softmax attention) with the selection
// held fixed: the hard top-k passes no gradient to routing (DashAttention page,
// "Declaração do Problema" 2) and keys outside the selected blocks get zero
// gradient (SSA page, "1. Definição do Problema" 2; AdaSplash-2 page,
// "4. Resultados Experimentais": the backward skips the zero blocks).
//
// With P = softmax(scale Q K_sel^T) (causal on the diagonal block), O = P V and
// the upstream gradient dO:
//   delta_t = dO_t . O_t                        (bwd_delta_kernel)
//   dS      = P * (dO V^T - delta)
//   dQ      = scale dS K_sel                    (bwd_dq_kernel)
//   dV     += P^T dO,  dK += scale dS^T Q        (bwd_dkv_kernel)
// P is rebuilt from the forward's log-sum-exp: P = exp(scale q.k - lse).
//
// Both contraction kernels run bf16 mma.sync m16n8k16 tiles with fp32
// accumulation.  Each warp owns 16 rows of the CTA's block: query rows in the
// dQ pass, key rows in the dK/dV pass.  Tiles of B rows x d sit in shared
// memory with the 16-byte chunks of a row XOR-swizzled by (row & 7), so every
// ldmatrix is conflict-free.  The fp32 accumulators of one contraction are
// rounded to bf16 and reused as the A fragments of the next (P and dS).
//
// dQ: one CTA per (b, query head, query block i); it walks the selected blocks
// of i in index order.  dK/dV: one CTA per (b, KV head, key block j), issued
// key block first so the sink column (selected by every query block) starts
// in the first wave; it finds the query blocks whose selection holds j by a
// binary search of their ascending index rows, in ascending order, and sums
// their rows over the G query heads of the group.  No atomics: every output
// element is written once, in a fixed summation order.
//
// Tiles move with 16-byte cp.async copies, all of a thread's copies in flight
// at once, into two buffers: the next step's tiles (the next selected block's
// K and V in the dQ pass, the next (query block, head)'s Q, dO, lse and delta
// in the dK/dV pass) load while the current step's contractions run.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace ssa {

namespace {

// Keys (dQ) or queries (dK/dV) per contraction chunk: the S and dP
// accumulators of a chunk stay in registers beside the d-wide outputs.
template <int D>
constexpr int chunk_of() {
  return D == 128 ? 32 : 64;
}
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// c += a . b on one m16n8k16 tile (bf16 in, fp32 accumulate).
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// A fragment of k-step p from the fp32 accumulators of n-tiles 2p and 2p + 1.
__device__ __forceinline__ void acc_to_a(const float (&c0)[4], const float (&c1)[4],
                                         uint32_t (&a)[4]) {
  a[0] = pack_bf16(c0[0], c0[1]);
  a[1] = pack_bf16(c0[2], c0[3]);
  a[2] = pack_bf16(c1[0], c1[1]);
  a[3] = pack_bf16(c1[2], c1[3]);
}

// Byte offset of 16-byte chunk c of row r in a swizzled tile of rows of D bf16.
template <int D>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)(r * (D * 2) + ((c ^ (r & 7)) << 4));
}

// Rows [row0, row0 + rows) of a [N, D] bf16 matrix into a swizzled tile; rows
// at or past N read as zeros.
template <int D>
__device__ __forceinline__ void load_tile(unsigned char* dst, const __nv_bfloat16* src, int row0,
                                          int rows, int N) {
  constexpr int CPR = D / 8;
  for (int e = threadIdx.x; e < rows * CPR; e += blockDim.x) {
    const int r = e / CPR, c = e - r * CPR;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (row0 + r < N) v = __ldg(reinterpret_cast<const uint4*>(src + (size_t)(row0 + r) * D) + c);
    *reinterpret_cast<uint4*>(dst + swz<D>(r, c)) = v;
  }
}

// Asynchronous 16-byte (4-byte) copies global -> shared; a source size of 0
// writes zeros and reads nothing (the address is still a valid one).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int NPEND>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(NPEND) : "memory");
}

// load_tile with asynchronous copies: every thread's copies are in flight at
// once; complete them with cp_async_commit / cp_async_wait and a barrier.
template <int D>
__device__ __forceinline__ void load_tile_async(uint32_t dst, const __nv_bfloat16* src, int row0,
                                                int rows, int N) {
  constexpr int CPR = D / 8;
  for (int e = threadIdx.x; e < rows * CPR; e += blockDim.x) {
    const int r = e / CPR, c = e - r * CPR;
    const bool ok = row0 + r < N;
    const __nv_bfloat16* p = ok ? src + (size_t)(row0 + r) * D + c * 8 : src;
    cp_async16(dst + swz<D>(r, c), p, ok ? 16u : 0u);
  }
}

}  // namespace

// delta[row] = dO[row] . O[row]; one warp per row, 8 rows per CTA.
template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const __nv_bfloat16* __restrict__ O,
                                                        const __nv_bfloat16* __restrict__ dO,
                                                        float* __restrict__ delta, long long rows) {
  constexpr int E = D / 32;
  const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const __nv_bfloat16* o = O + r * D + lane * E;
  const __nv_bfloat16* g = dO + r * D + lane * E;
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) s = fmaf(__bfloat162float(o[e]), __bfloat162float(g[e]), s);
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
  if (lane == 0) delta[r] = s;
}

// dQ for one (b, query head h, query block i); B / 16 warps.
template <int D>
__global__ void __launch_bounds__(256, 1) bwd_dq_kernel(
    const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
    const __nv_bfloat16* __restrict__ V, const __nv_bfloat16* __restrict__ dO,
    const float* __restrict__ lse, const float* __restrict__ delta,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt, int Hq, int Hkv, int N,
    int B, int nq, int max_sel, float scale, __nv_bfloat16* __restrict__ dQ) {
  constexpr int CH = chunk_of<D>();
  constexpr int NT = CH / 8;  // S column tiles per chunk
  constexpr int KS = D / 16;      // k steps over d
  constexpr int ON = D / 8;       // dQ column tiles
  extern __shared__ __align__(128) unsigned char smem_bwd[];
  const int tile = B * D * 2;
  // Q, dO, then K and V twice: the next selected block's tiles load while
  // the current one is in use
  const uint32_t aQ = ptx::smem_u32(smem_bwd), aG = aQ + tile;
  auto k_at = [&](int buf) { return aQ + (uint32_t)((2 + 2 * buf) * tile); };
  auto v_at = [&](int buf) { return aQ + (uint32_t)((3 + 2 * buf) * tile); };

  const int i = blockIdx.x % nq;
  const int bh = blockIdx.x / nq;  // b * Hq + h
  const int h = bh % Hq, b = bh / Hq;
  const int G = Hq / Hkv, g = h / G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gr = lane >> 2, tq = lane & 3, lm = lane >> 3, lr = lane & 7;
  const int q0 = i * B;
  const size_t hoff = (size_t)bh * N * D;
  const size_t goff = ((size_t)b * Hkv + g) * N * D;

  load_tile_async<D>(aQ, Q + hoff, q0, B, N);
  load_tile_async<D>(aG, dO + hoff, q0, B, N);

  // this lane's two query rows: warp * 16 + gr and + 8
  const int ra = q0 + warp * 16 + gr, rb = ra + 8;
  const float c2 = scale * kLog2e;
  const float la = ra < N ? lse[(size_t)bh * N + ra] * kLog2e : INFINITY;
  const float lb = rb < N ? lse[(size_t)bh * N + rb] * kLog2e : INFINITY;
  const float da = ra < N ? delta[(size_t)bh * N + ra] : 0.f;
  const float db = rb < N ? delta[(size_t)bh * N + rb] : 0.f;

  float acc[ON][4];
#pragma unroll
  for (int n = 0; n < ON; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;

  const size_t urow = ((size_t)b * Hkv + g) * nq + i;
  const int n_sel = min(max(cnt[urow], 0), max_sel);
  const int32_t* sel = idx + urow * max_sel;
  // entries outside [0, i] are skipped (the same for every thread)
  auto next_valid = [&](int s) {
    while (s < n_sel && (sel[s] < 0 || sel[s] > i)) ++s;
    return s;
  };
  int s = next_valid(0);
  if (s < n_sel) {
    load_tile_async<D>(k_at(0), K + goff, sel[s] * B, B, N);
    load_tile_async<D>(v_at(0), V + goff, sel[s] * B, B, N);
  }
  cp_async_commit();  // group: Q, dO and the first K / V
  for (int it = 0; s < n_sel; ++it) {
    const int j = sel[s];
    const int buf = it & 1;
    const int s2 = next_valid(s + 1);
    __syncthreads();  // the other buffer's tiles (previous block) are consumed
    if (s2 < n_sel) {
      load_tile_async<D>(k_at(buf ^ 1), K + goff, sel[s2] * B, B, N);
      load_tile_async<D>(v_at(buf ^ 1), V + goff, sel[s2] * B, B, N);
    }
    cp_async_commit();
    cp_async_wait<1>();  // everything but the newest group has landed
    __syncthreads();
    s = s2;
    const uint32_t aK = k_at(buf), aV = v_at(buf);
    for (int kc = 0; kc < B; kc += CH) {
      const int nk = min(CH, B - kc);  // a multiple of 16
      float sc[NT][4], dp[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[n][e] = dp[n][e] = 0.f;
      // S = Q K^T and dP = dO V^T over this warp's 16 rows and the chunk's keys
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t aq[4], ag[4];
        const int ar = warp * 16 + (lm & 1) * 8 + lr;
        ldsm4(aQ + swz<D>(ar, 2 * ks + (lm >> 1)), aq);
        ldsm4(aG + swz<D>(ar, 2 * ks + (lm >> 1)), ag);
#pragma unroll
        for (int p = 0; p < NT / 2; ++p) {
          if (16 * p < nk) {
            const int kr = kc + 16 * p + (lm >> 1) * 8 + lr;
            uint32_t kb[4], vb[4];
            ldsm4(aK + swz<D>(kr, 2 * ks + (lm & 1)), kb);
            ldsm4(aV + swz<D>(kr, 2 * ks + (lm & 1)), vb);
            mma16816(sc[2 * p], aq, kb[0], kb[1]);
            mma16816(sc[2 * p + 1], aq, kb[2], kb[3]);
            mma16816(dp[2 * p], ag, vb[0], vb[1]);
            mma16816(dp[2 * p + 1], ag, vb[2], vb[3]);
          }
        }
      }
      // dS = P * (dP - delta), P rebuilt from the log-sum-exp; masked keys give 0
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kl = kc + n * 8 + 2 * tq + (e & 1);  // key within block j
          const int key = j * B + kl;
          const int row = e < 2 ? ra : rb;
          const float l2 = e < 2 ? la : lb;
          const float dl = e < 2 ? da : db;
          const float p = (kl < B && key <= row) ? exp2f(fmaf(sc[n][e], c2, -l2)) : 0.f;
          sc[n][e] = p * (dp[n][e] - dl);
        }
      // dQ += dS K
#pragma unroll
      for (int p = 0; p < NT / 2; ++p) {
        if (16 * p < nk) {
          uint32_t a[4];
          acc_to_a(sc[2 * p], sc[2 * p + 1], a);
          const int kr = kc + 16 * p + (lm & 1) * 8 + lr;
#pragma unroll
          for (int qd = 0; qd < ON / 2; ++qd) {
            uint32_t kb[4];
            ldsm4_t(aK + swz<D>(kr, 2 * qd + (lm >> 1)), kb);
            mma16816(acc[2 * qd], a, kb[0], kb[1]);
            mma16816(acc[2 * qd + 1], a, kb[2], kb[3]);
          }
        }
      }
    }
  }
  cp_async_wait<0>();  // no copy outlives the CTA
  // dQ = scale * acc, rows past N skipped
#pragma unroll
  for (int n = 0; n < ON; ++n) {
    const int col = n * 8 + 2 * tq;
    if (ra < N)
      *reinterpret_cast<__nv_bfloat162*>(dQ + hoff + (size_t)ra * D + col) =
          __floats2bfloat162_rn(acc[n][0] * scale, acc[n][1] * scale);
    if (rb < N)
      *reinterpret_cast<__nv_bfloat162*>(dQ + hoff + (size_t)rb * D + col) =
          __floats2bfloat162_rn(acc[n][2] * scale, acc[n][3] * scale);
  }
}

// dK and dV for one (b, KV head g, key block j); B / 16 warps.
template <int D>
__global__ void __launch_bounds__(256, 1) bwd_dkv_kernel(
    const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
    const __nv_bfloat16* __restrict__ V, const __nv_bfloat16* __restrict__ dO,
    const float* __restrict__ lse, const float* __restrict__ delta,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt, int batch, int Hq, int Hkv,
    int N, int B, int nq, int max_sel, float scale, __nv_bfloat16* __restrict__ dK,
    __nv_bfloat16* __restrict__ dV, float* __restrict__ sink_part, int sink_qr, int sink_nsplit) {
  constexpr int CH = chunk_of<D>();
  constexpr int NT = CH / 8;  // query column tiles per chunk
  constexpr int KS = D / 16;
  constexpr int ON = D / 8;
  extern __shared__ __align__(128) unsigned char smem_bwd[];
  const int tile = B * D * 2;
  // K, V, then Q and dO twice (the next step's tiles load while the current
  // ones are in use), then lse and delta twice ([2][B] each, natural log)
  const uint32_t aK = ptx::smem_u32(smem_bwd), aV = aK + tile;
  auto q_at = [&](int buf) { return aK + (uint32_t)((2 + 2 * buf) * tile); };
  auto g_at = [&](int buf) { return aK + (uint32_t)((3 + 2 * buf) * tile); };
  float* s_lse = reinterpret_cast<float*>(smem_bwd + 6 * tile);
  float* s_del = s_lse + 2 * B;
  __shared__ int s_list[256];
  __shared__ int s_wcnt[8];

  const int nbg = batch * Hkv;
  // CTAs [0, nbg * sink_nsplit) take the sink column (key block 0, which every
  // query block selects) in ranges of sink_qr query blocks and write fp32
  // partial sums; the others take one key block j >= 1 each over every query
  // block i >= j.  The sink ranges come first, so they start in the first wave.
  const int nsink = nbg * sink_nsplit;
  const bool sink = (int)blockIdx.x < nsink;
  int j, bg, i_lo, i_hi;
  if (sink) {
    const int rg = blockIdx.x / nbg;
    j = 0;
    bg = blockIdx.x - rg * nbg;
    i_lo = rg * sink_qr;
    i_hi = min(nq, i_lo + sink_qr);
  } else {
    const int u = blockIdx.x - nsink;
    j = 1 + u / nbg;
    bg = u - (j - 1) * nbg;
    i_lo = j;
    i_hi = nq;
  }
  const int b = bg / Hkv, g = bg - b * Hkv;
  const int G = Hq / Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int gr = lane >> 2, tq = lane & 3, lm = lane >> 3, lr = lane & 7;
  const size_t goff = (size_t)bg * N * D;
  const float c2 = scale * kLog2e;

  load_tile_async<D>(aK, K + goff, j * B, B, N);
  load_tile_async<D>(aV, V + goff, j * B, B, N);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  // step stp of a range: hit stp / G, head stp % G, into buffer buf
  auto issue = [&](int stp, int buf) {
    const int i = s_list[stp / G];
    const int bh = b * Hq + g * G + stp % G;
    load_tile_async<D>(q_at(buf), Q + (size_t)bh * N * D, i * B, B, N);
    load_tile_async<D>(g_at(buf), dO + (size_t)bh * N * D, i * B, B, N);
    for (int r = threadIdx.x; r < B; r += blockDim.x) {
      const int t = i * B + r;
      const bool ok = t < N;
      cp_async4(ptx::smem_u32(s_lse + buf * B + r), ok ? lse + (size_t)bh * N + t : lse,
                ok ? 4u : 0u);
      cp_async4(ptx::smem_u32(s_del + buf * B + r), ok ? delta + (size_t)bh * N + t : delta,
                ok ? 4u : 0u);
    }
  };

  float dk[ON][4], dv[ON][4];
#pragma unroll
  for (int n = 0; n < ON; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.f;

  // this lane's two key positions
  const int ka = j * B + warp * 16 + gr, kb_ = ka + 8;
  const int32_t* idx_bg = idx + (size_t)bg * nq * max_sel;
  const int32_t* cnt_bg = cnt + (size_t)bg * nq;

  for (int base = i_lo; base < i_hi; base += blockDim.x) {
    // ---- the query blocks in [base, base + blockDim.x) whose selection holds j
    const int qi = base + threadIdx.x;
    bool hit = false;
    if (qi < i_hi) {
      const int32_t* row = idx_bg + (size_t)qi * max_sel;
      int lo = 0, hi = min(max(cnt_bg[qi], 0), max_sel);  // ascending entries in [lo, hi)
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const int v = row[mid];
        if (v == j) {
          hit = true;
          break;
        }
        if (v < j) lo = mid + 1;
        else hi = mid;
      }
    }
    const unsigned bal = __ballot_sync(0xffffffffu, hit);
    if (lane == 0) s_wcnt[warp] = __popc(bal);
    __syncthreads();
    int off = 0, n_hit = 0;
    for (int w = 0; w < nwarps; ++w) {
      const int c = s_wcnt[w];
      if (w < warp) off += c;
      n_hit += c;
    }
    if (hit) s_list[off + __popc(bal & ((1u << lane) - 1u))] = qi;
    __syncthreads();

    const int nst = n_hit * G;
    if (nst > 0) issue(0, 0);
    cp_async_commit();
    for (int stp = 0; stp < nst; ++stp) {
      const int buf = stp & 1;
      __syncthreads();  // the other buffer (previous step) is consumed
      if (stp + 1 < nst) issue(stp + 1, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();  // this step's group has landed
      __syncthreads();
      {
        const int i = s_list[stp / G];
        const uint32_t aQ = q_at(buf), aG = g_at(buf);
        const float* lse_b = s_lse + buf * B;
        const float* del_b = s_del + buf * B;
        for (int qc = 0; qc < B; qc += CH) {
          const int nqc = min(CH, B - qc);  // a multiple of 16
          float st[NT][4], dpt[NT][4];  // S^T and dP^T: this warp's 16 keys x the chunk's queries
#pragma unroll
          for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) st[n][e] = dpt[n][e] = 0.f;
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            uint32_t ak[4], av[4];
            const int ar = warp * 16 + (lm & 1) * 8 + lr;
            ldsm4(aK + swz<D>(ar, 2 * ks + (lm >> 1)), ak);
            ldsm4(aV + swz<D>(ar, 2 * ks + (lm >> 1)), av);
#pragma unroll
            for (int p = 0; p < NT / 2; ++p) {
              if (16 * p < nqc) {
                const int qr = qc + 16 * p + (lm >> 1) * 8 + lr;
                uint32_t qb[4], gb[4];
                ldsm4(aQ + swz<D>(qr, 2 * ks + (lm & 1)), qb);
                ldsm4(aG + swz<D>(qr, 2 * ks + (lm & 1)), gb);
                mma16816(st[2 * p], ak, qb[0], qb[1]);
                mma16816(st[2 * p + 1], ak, qb[2], qb[3]);
                mma16816(dpt[2 * p], av, gb[0], gb[1]);
                mma16816(dpt[2 * p + 1], av, gb[2], gb[3]);
              }
            }
          }
          // P^T and dS^T = P^T * (dP^T - delta); a key after the query, or a
          // query row past N (log-sum-exp +inf), gives 0
#pragma unroll
          for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int ql = qc + n * 8 + 2 * tq + (e & 1);  // query within block i
              const int key = e < 2 ? ka : kb_;
              float p = 0.f, ds = 0.f;
              if (ql < B && key <= i * B + ql && i * B + ql < N) {
                p = exp2f(fmaf(st[n][e], c2, -lse_b[ql] * kLog2e));
                ds = p * (dpt[n][e] - del_b[ql]);
              }
              st[n][e] = p;
              dpt[n][e] = ds;
            }
          // dV += P^T dO and dK += dS^T Q
#pragma unroll
          for (int p = 0; p < NT / 2; ++p) {
            if (16 * p < nqc) {
              uint32_t pa[4], sa[4];
              acc_to_a(st[2 * p], st[2 * p + 1], pa);
              acc_to_a(dpt[2 * p], dpt[2 * p + 1], sa);
              const int qr = qc + 16 * p + (lm & 1) * 8 + lr;
#pragma unroll
              for (int qd = 0; qd < ON / 2; ++qd) {
                uint32_t gb[4], qb[4];
                ldsm4_t(aG + swz<D>(qr, 2 * qd + (lm >> 1)), gb);
                ldsm4_t(aQ + swz<D>(qr, 2 * qd + (lm >> 1)), qb);
                mma16816(dv[2 * qd], pa, gb[0], gb[1]);
                mma16816(dv[2 * qd + 1], pa, gb[2], gb[3]);
                mma16816(dk[2 * qd], sa, qb[0], qb[1]);
                mma16816(dk[2 * qd + 1], sa, qb[2], qb[3]);
              }
            }
          }
        }
      }
    }
    __syncthreads();  // s_wcnt and s_list are rewritten by the next range
  }
  cp_async_wait<0>();  // no copy outlives the CTA
  if (sink) {
    // fp32 partial sums of this range: [range][bg][dK, dV][B][D], unscaled
    float* pk = sink_part + ((size_t)(blockIdx.x / nbg) * nbg + bg) * 2 * B * D;
    float* pv = pk + (size_t)B * D;
    const int ra = warp * 16 + gr, rb = ra + 8;
#pragma unroll
    for (int n = 0; n < ON; ++n) {
      const int col = n * 8 + 2 * tq;
      *reinterpret_cast<float2*>(pk + (size_t)ra * D + col) = make_float2(dk[n][0], dk[n][1]);
      *reinterpret_cast<float2*>(pv + (size_t)ra * D + col) = make_float2(dv[n][0], dv[n][1]);
      *reinterpret_cast<float2*>(pk + (size_t)rb * D + col) = make_float2(dk[n][2], dk[n][3]);
      *reinterpret_cast<float2*>(pv + (size_t)rb * D + col) = make_float2(dv[n][2], dv[n][3]);
    }
    return;
  }
  // dK = scale * dk, dV = dv; key rows past N skipped
#pragma unroll
  for (int n = 0; n < ON; ++n) {
    const int col = n * 8 + 2 * tq;
    if (ka < N) {
      *reinterpret_cast<__nv_bfloat162*>(dK + goff + (size_t)ka * D + col) =
          __floats2bfloat162_rn(dk[n][0] * scale, dk[n][1] * scale);
      *reinterpret_cast<__nv_bfloat162*>(dV + goff + (size_t)ka * D + col) =
          __floats2bfloat162_rn(dv[n][0], dv[n][1]);
    }
    if (kb_ < N) {
      *reinterpret_cast<__nv_bfloat162*>(dK + goff + (size_t)kb_ * D + col) =
          __floats2bfloat162_rn(dk[n][2] * scale, dk[n][3] * scale);
      *reinterpret_cast<__nv_bfloat162*>(dV + goff + (size_t)kb_ * D + col) =
          __floats2bfloat162_rn(dv[n][2], dv[n][3]);
    }
  }
}

// dK and dV of the sink block: the ranges' partial sums added in range order
// (a fixed order: the result does not depend on scheduling), dK scaled.
template <int D>
__global__ void __launch_bounds__(256) bwd_sink_reduce_kernel(
    const float* __restrict__ sink_part, int nbg, int nsplit, int B, int N, float scale,
    __nv_bfloat16* __restrict__ dK, __nv_bfloat16* __restrict__ dV) {
  const int bg = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;  // element of the B x D tile
  if (e >= B * D) return;
  const int r = e / D;
  float k = 0.f, v = 0.f;
  for (int rg = 0; rg < nsplit; ++rg) {
    const float* p = sink_part + ((size_t)rg * nbg + bg) * 2 * B * D;
    k += p[e];
    v += p[(size_t)B * D + e];
  }
  if (r < N) {
    dK[(size_t)bg * N * D + e] = __float2bfloat16_rn(k * scale);
    dV[(size_t)bg * N * D + e] = __float2bfloat16_rn(v);
  }
}

// The selection transposed: for every (bg, i) and entry j <= i of its row,
// bit i of key block j's mask.  OR is order-free, so the masks do not depend
// on scheduling.  mask is zeroed beforehand.
__global__ void __launch_bounds__(256) bwd_hitmask_kernel(const int32_t* __restrict__ idx,
                                                          const int32_t* __restrict__ cnt,
                                                          int nbg, int nq, int max_sel, int nwin,
                                                          uint32_t* __restrict__ mask) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (long long)nbg * nq) return;
  const int bg = (int)(t / nq), i = (int)(t - (long long)bg * nq);
  const int ns = min(max(cnt[t], 0), max_sel);
  const int32_t* row = idx + t * max_sel;
  for (int e = 0; e < ns; ++e) {
    const int j = row[e];
    if (j >= 0 && j <= i)
      atomicOr(&mask[((long long)bg * nq + j) * nwin + (i >> 5)], 1u << (i & 31));
  }
}

size_t attn_bwd_smem_bytes(int d, int B) {
  return (size_t)6 * B * d * 2 + (size_t)4 * B * sizeof(float);
}

BwdPlan plan_bwd(int batch, int Hq, int Hkv, int N, int d, int B) {
  BwdPlan p{};
  const int nq = (N + B - 1) / B;
  const int G = Hq / Hkv;
  p.sink_qr = 256 / G > 16 ? 256 / G : 16;  // about 256 (query block, head) steps per range
  p.sink_nsplit = (nq + p.sink_qr - 1) / p.sink_qr;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  p.off_delta = 0;
  p.off_part = up((size_t)batch * Hq * N * sizeof(float));
  p.off_mask = up(p.off_part +
                  (size_t)batch * Hkv * p.sink_nsplit * 2 * (size_t)B * d * sizeof(float));
  p.nwin = (attn_tc_supported(SSA_BF16, Hq, Hkv, d, B) && B == 64) ? (nq + 31) / 32 : 0;
  p.bytes = up(p.off_mask + (size_t)batch * Hkv * nq * p.nwin * sizeof(uint32_t));
  return p;
}

template <int D>
static cudaError_t launch_bwd_t(const BwdPlan& pl, const void* Q, const void* K, const void* V,
                                const void* O, const void* dO, const float* lse,
                                const int32_t* idx, const int32_t* cnt, int batch, int Hq,
                                int Hkv, int N, int B, int max_sel, float scale, void* dQ,
                                void* dK, void* dV, void* ws, cudaStream_t st) {
  using bf = __nv_bfloat16;
  float* delta = reinterpret_cast<float*>(static_cast<char*>(ws) + pl.off_delta);
  float* part = reinterpret_cast<float*>(static_cast<char*>(ws) + pl.off_part);
  const int nq = (N + B - 1) / B;
  const int nbg = batch * Hkv;
  const long long rows = (long long)batch * Hq * N;
  const unsigned threads = (unsigned)(2 * B);  // B / 16 warps
  const size_t smem = attn_bwd_smem_bytes(D, B);
  bwd_delta_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>((const bf*)O, (const bf*)dO,
                                                                   delta, rows);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const bool tc = attn_tc_supported(SSA_BF16, Hq, Hkv, D, B);
  if (tc) {
    e = launch_bwd_dq_tc(Q, K, V, dO, lse, delta, idx, cnt, batch, Hq, Hkv, N, B, max_sel, scale,
                         dQ, st);
  } else {
    e = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    bwd_dq_kernel<D><<<(unsigned)((long long)batch * Hq * nq), threads, smem, st>>>(
        (const bf*)Q, (const bf*)K, (const bf*)V, (const bf*)dO, lse, delta, idx, cnt, Hq, Hkv,
        N, B, nq, max_sel, scale, (bf*)dQ);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  if (tc && B == 64 && pl.nwin > 0) {
    uint32_t* mask = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + pl.off_mask);
    const size_t mbytes = (size_t)nbg * nq * pl.nwin * sizeof(uint32_t);
    e = cudaMemsetAsync(mask, 0, mbytes, st);
    if (e != cudaSuccess) return e;
    const long long rows_bg = (long long)nbg * nq;
    bwd_hitmask_kernel<<<(unsigned)((rows_bg + 255) / 256), 256, 0, st>>>(idx, cnt, nbg, nq,
                                                                          max_sel, pl.nwin, mask);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = launch_bwd_dkv_tc(Q, K, V, dO, lse, delta, batch, Hq, Hkv, N, scale, dK, dV, part,
                          pl.sink_qr, pl.sink_nsplit, mask, pl.nwin, st);
  } else {
    e = cudaFuncSetAttribute(bwd_dkv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    const long long ctas = (long long)nbg * pl.sink_nsplit + (long long)nbg * (nq - 1);
    bwd_dkv_kernel<D><<<(unsigned)ctas, threads, smem, st>>>(
        (const bf*)Q, (const bf*)K, (const bf*)V, (const bf*)dO, lse, delta, idx, cnt, batch, Hq,
        Hkv, N, B, nq, max_sel, scale, (bf*)dK, (bf*)dV, part, pl.sink_qr, pl.sink_nsplit);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  const dim3 rgrid((unsigned)((B * D + 255) / 256), (unsigned)nbg);
  bwd_sink_reduce_kernel<D><<<rgrid, 256, 0, st>>>(part, nbg, pl.sink_nsplit, B, N, scale,
                                                   (bf*)dK, (bf*)dV);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd(const BwdPlan& pl, const void* Q, const void* K, const void* V,
                            const void* O, const void* dO, const float* lse, const int32_t* idx,
                            const int32_t* cnt, int batch, int Hq, int Hkv, int N, int d, int B,
                            int max_sel, float scale, void* dQ, void* dK, void* dV, void* ws,
                            cudaStream_t st) {
  if (d == 128)
    return launch_bwd_t<128>(pl, Q, K, V, O, dO, lse, idx, cnt, batch, Hq, Hkv, N, B, max_sel,
                             scale, dQ, dK, dV, ws, st);
  return launch_bwd_t<64>(pl, Q, K, V, O, dO, lse, idx, cnt, batch, Hq, Hkv, N, B, max_sel, scale,
                          dQ, dK, dV, ws, st);
}

}  // namespace ssa
