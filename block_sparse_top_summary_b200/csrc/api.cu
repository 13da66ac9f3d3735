// C ABI entry points: host-side argument checks, then the kernel launches.
#include <cuda_runtime.h>

#include "kernels.h"
#include "ssa.h"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool dtype_ok(ssa_dtype dt) { return dt == SSA_F32 || dt == SSA_BF16; }

// Shape checks shared by every entry point.  Returns SSA_OK or the error.
ssa_status check_dims(int d, int B, ssa_dtype dt) {
  if (!dtype_ok(dt)) return SSA_ERR_INVALID_ARG;
  if (B <= 0 || d <= 0) return SSA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SSA_ERR_UNSUPPORTED;
  if (B % 16 != 0 || B > 128) return SSA_ERR_UNSUPPORTED;
  return SSA_OK;
}

ssa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SSA_OK : SSA_ERR_CUDA; }

// Result word of ssa_check_device_error (one per device).
__device__ int g_error_taken = 0;

constexpr int kMaxErrorWords = 4;
struct ErrorWords {
  int* w[kMaxErrorWords];
  int n;
};

// Takes every error word (atomic exchange with 0) and stores the first
// non-zero one, in the order given, into g_error_taken.
__global__ void take_error_words_kernel(ErrorWords words) {
  int first = 0;
  for (int k = 0; k < words.n; ++k) {
    const int v = atomicExch(words.w[k], 0);
    if (first == 0) first = v;
  }
  g_error_taken = first;
}

}  // namespace

extern "C" {

const char* ssa_status_string(int status) {
  switch (status) {
    case SSA_OK: return "SSA_OK";
    case SSA_ERR_INVALID_ARG: return "SSA_ERR_INVALID_ARG";
    case SSA_ERR_UNSUPPORTED: return "SSA_ERR_UNSUPPORTED";
    case SSA_ERR_CUDA: return "SSA_ERR_CUDA";
    case SSA_ERR_TIMEOUT: return "SSA_ERR_TIMEOUT";
    default: return "SSA_ERR_UNKNOWN";
  }
}

int ssa_version(void) { return 204; }

ssa_status ssa_block_summary(const void* K, ssa_dtype dtype, int batch, int Hkv, int N, int d,
                             int B, float* S, ssa_stream stream) {
  ssa_status st = check_dims(d, B, dtype);
  if (st != SSA_OK) return st;
  if (batch <= 0 || Hkv <= 0 || N <= 0) return SSA_ERR_INVALID_ARG;
  if (N / B == 0) return SSA_OK;
  if (K == nullptr || S == nullptr) return SSA_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(S)) return SSA_ERR_INVALID_ARG;
  return from_cuda(ssa::launch_block_summary(K, dtype, batch, Hkv, N, d, B, S,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

ssa_status ssa_route(const void* Q, ssa_dtype dtype, const float* S, int batch, int Hq, int Hkv,
                     int N, int d, int B, int topk, int max_sel, int32_t* idx, int32_t* cnt,
                     float* scores, ssa_stream stream) {
  ssa_status st = check_dims(d, B, dtype);
  if (st != SSA_OK) return st;
  if (batch <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || topk < 0) return SSA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SSA_ERR_INVALID_ARG;
  const int nq = (N + B - 1) / B;
  if (nq > ssa::kRouteMaxBlocks) return SSA_ERR_UNSUPPORTED;
  const int cand_max = nq > 2 ? nq - 2 : 0;
  const int need = (topk < cand_max ? topk : cand_max) + 2;
  if (max_sel < need) return SSA_ERR_INVALID_ARG;
  if (Q == nullptr || idx == nullptr || cnt == nullptr) return SSA_ERR_INVALID_ARG;
  if (N / B > 0 && S == nullptr) return SSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(S)) return SSA_ERR_INVALID_ARG;
  if (scores != nullptr && !aligned16(scores)) return SSA_ERR_INVALID_ARG;
  return from_cuda(ssa::launch_route(Q, dtype, S, batch, Hq, Hkv, N, d, B, topk, max_sel, idx, cnt,
                                     scores, reinterpret_cast<cudaStream_t>(stream)));
}

ssa_status ssa_sparse_attn_fwd(const void* Q, const void* K, const void* V, ssa_dtype dtype,
                               const int32_t* idx, const int32_t* cnt, int batch, int Hq, int Hkv,
                               int N, int d, int B, int max_sel, float scale, void* O, float* lse,
                               ssa_stream stream) {
  ssa_status st = check_dims(d, B, dtype);
  if (st != SSA_OK) return st;
  if (batch <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || max_sel < 1) return SSA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SSA_ERR_INVALID_ARG;
  if (!(scale > 0.f)) return SSA_ERR_INVALID_ARG;
  if (Q == nullptr || K == nullptr || V == nullptr || idx == nullptr || cnt == nullptr ||
      O == nullptr)
    return SSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return SSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (ssa::attn_tc_supported(dtype, Hq, Hkv, d, B))
    return from_cuda(
        ssa::launch_attn_tc(Q, K, V, idx, cnt, nullptr, batch, Hq, Hkv, N, B, max_sel, scale, O,
                            lse, s));
  return from_cuda(ssa::launch_attn_simt(Q, K, V, dtype, idx, cnt, nullptr, batch, Hq, Hkv, N, d,
                                         B, max_sel, scale, O, lse, s));
}

ssa_status ssa_learned_summary(const void* K, ssa_dtype dtype, const float* qbar, int batch,
                               int Hkv, int N, int d, int B, float* S, ssa_stream stream) {
  ssa_status st = check_dims(d, B, dtype);
  if (st != SSA_OK) return st;
  if (batch <= 0 || Hkv <= 0 || N <= 0) return SSA_ERR_INVALID_ARG;
  if (N / B == 0) return SSA_OK;
  if (K == nullptr || qbar == nullptr || S == nullptr) return SSA_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(S)) return SSA_ERR_INVALID_ARG;
  return from_cuda(ssa::launch_learned_summary(K, dtype, qbar, batch, Hkv, N, d, B, S,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

ssa_status ssa_route_entmax(const void* Q, ssa_dtype dtype, const float* S, int batch, int Hq,
                            int Hkv, int N, int d, int B, float alpha, float gamma, float sigma,
                            int max_sel, int32_t* idx, int32_t* cnt, float* bias, float* w,
                            ssa_stream stream) {
  ssa_status st = check_dims(d, B, dtype);
  if (st != SSA_OK) return st;
  if (batch <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || Hq % Hkv != 0) return SSA_ERR_INVALID_ARG;
  if (!(alpha > 1.f) || !(alpha <= 8.f) || !(gamma > 0.f) || !(sigma >= 0.f))
    return SSA_ERR_INVALID_ARG;
  const int nq = (N + B - 1) / B, nfull = N / B;
  const int most = (nq - 1 < nfull ? nq - 1 : nfull) + 1;  // every candidate + the diagonal
  if (max_sel < most) return SSA_ERR_INVALID_ARG;
  if ((size_t)4 * ((size_t)d + 2 * (size_t)nq) > 200 * 1024) return SSA_ERR_UNSUPPORTED;
  if (Q == nullptr || idx == nullptr || cnt == nullptr || bias == nullptr ||
      (nfull > 0 && S == nullptr))
    return SSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(S)) return SSA_ERR_INVALID_ARG;
  return from_cuda(ssa::launch_entmax_route(Q, dtype, S, batch, Hq, Hkv, N, d, B, alpha, gamma,
                                            sigma, max_sel, idx, cnt, bias, w,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

ssa_status ssa_sparse_attn_fwd_prior(const void* Q, const void* K, const void* V,
                                     ssa_dtype dtype, const int32_t* idx, const int32_t* cnt,
                                     const float* bias, int batch, int Hq, int Hkv, int N, int d,
                                     int B, int max_sel, float scale, void* O, float* lse,
                                     ssa_stream stream) {
  ssa_status st = check_dims(d, B, dtype);
  if (st != SSA_OK) return st;
  if (batch <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || max_sel < 1) return SSA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0 || !(scale > 0.f)) return SSA_ERR_INVALID_ARG;
  if (Q == nullptr || K == nullptr || V == nullptr || idx == nullptr || cnt == nullptr ||
      bias == nullptr || O == nullptr)
    return SSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return SSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (ssa::attn_tc_supported(dtype, Hq, Hkv, d, B))
    return from_cuda(ssa::launch_attn_tc(Q, K, V, idx, cnt, bias, batch, Hq, Hkv, N, B, max_sel,
                                         scale, O, lse, s));
  return from_cuda(ssa::launch_attn_simt(Q, K, V, dtype, idx, cnt, bias, batch, Hq, Hkv, N, d, B,
                                         max_sel, scale, O, lse, s));
}

ssa_status ssa_sparse_attn_bwd_workspace_size(int batch, int Hq, int Hkv, int N, int d, int B,
                                              size_t* bytes) {
  if (bytes == nullptr) return SSA_ERR_INVALID_ARG;
  ssa_status st = check_dims(d, B, SSA_BF16);
  if (st != SSA_OK) return st;
  if (batch <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || Hq % Hkv != 0) return SSA_ERR_INVALID_ARG;
  *bytes = ssa::plan_bwd(batch, Hq, Hkv, N, d, B).bytes;
  return SSA_OK;
}

ssa_status ssa_sparse_attn_bwd(const void* Q, const void* K, const void* V, const void* O,
                               const void* dO, const float* lse, ssa_dtype dtype,
                               const int32_t* idx, const int32_t* cnt, int batch, int Hq, int Hkv,
                               int N, int d, int B, int max_sel, float scale, void* dQ, void* dK,
                               void* dV, void* workspace, size_t ws_bytes, ssa_stream stream) {
  ssa_status st = check_dims(d, B, dtype);
  if (st != SSA_OK) return st;
  if (dtype != SSA_BF16) return SSA_ERR_UNSUPPORTED;
  if (batch <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || max_sel < 1) return SSA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SSA_ERR_INVALID_ARG;
  if (!(scale > 0.f)) return SSA_ERR_INVALID_ARG;
  if (Q == nullptr || K == nullptr || V == nullptr || O == nullptr || dO == nullptr ||
      lse == nullptr || idx == nullptr || cnt == nullptr || dQ == nullptr || dK == nullptr ||
      dV == nullptr || workspace == nullptr)
    return SSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(dO) ||
      !aligned16(dQ) || !aligned16(dK) || !aligned16(dV))
    return SSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SSA_ERR_INVALID_ARG;
  const long long nq = ((long long)N + B - 1) / B;
  if ((long long)batch * Hq * nq > 0x7fffffffLL || (long long)batch * Hq * N / 8 > 0x7fffffffLL)
    return SSA_ERR_UNSUPPORTED;
  const ssa::BwdPlan pl = ssa::plan_bwd(batch, Hq, Hkv, N, d, B);
  if (ws_bytes < pl.bytes) return SSA_ERR_INVALID_ARG;
  return from_cuda(ssa::launch_attn_bwd(pl, Q, K, V, O, dO, lse, idx, cnt, batch, Hq, Hkv, N, d,
                                        B, max_sel, scale, dQ, dK, dV, workspace,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

int ssa_sparse_attn_uses_tensor_cores(ssa_dtype dtype, int Hq, int Hkv, int d, int B) {
  if (!dtype_ok(dtype) || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return 0;
  return ssa::attn_tc_supported(dtype, Hq, Hkv, d, B) ? 1 : 0;
}

ssa_status ssa_decode_workspace_size(int batch, int Hq, int Hkv, int Lmax, int d, int B, int topk,
                                     size_t* bytes) {
  if (bytes == nullptr) return SSA_ERR_INVALID_ARG;
  ssa_status st = check_dims(d, B, SSA_BF16);
  if (st != SSA_OK) return st;
  if (batch <= 0 || Hq <= 0 || Hkv <= 0 || Lmax <= 0 || topk < 0) return SSA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SSA_ERR_INVALID_ARG;
  *bytes = ssa::plan_decode(batch, Hq, Hkv, d, B, topk, Lmax).bytes;
  return SSA_OK;
}

ssa_status ssa_decode(const void* q, const void* Kc, const void* Vc, ssa_dtype dtype,
                      const float* S, const int32_t* seqlens, int batch, int Hq, int Hkv, int Lmax,
                      int d, int B, int topk, float scale, void* O, int32_t* idx, void* workspace,
                      size_t ws_bytes, ssa_stream stream) {
  ssa_status st = check_dims(d, B, dtype);
  if (st != SSA_OK) return st;
  if (batch <= 0 || Hq <= 0 || Hkv <= 0 || Lmax <= 0 || topk < 0) return SSA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SSA_ERR_INVALID_ARG;
  if (Hq / Hkv > 8) return SSA_ERR_UNSUPPORTED;
  if (Lmax / B > 16384) return SSA_ERR_UNSUPPORTED;
  if (!(scale > 0.f)) return SSA_ERR_INVALID_ARG;
  if (q == nullptr || Kc == nullptr || Vc == nullptr || seqlens == nullptr || O == nullptr ||
      workspace == nullptr)
    return SSA_ERR_INVALID_ARG;
  if (Lmax / B > 0 && S == nullptr) return SSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(Kc) || !aligned16(Vc) || !aligned16(S) || !aligned16(O))
    return SSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SSA_ERR_INVALID_ARG;
  const ssa::DecodePlan p = ssa::plan_decode(batch, Hq, Hkv, d, B, topk, Lmax);
  if (ws_bytes < p.bytes) return SSA_ERR_INVALID_ARG;
  return from_cuda(ssa::launch_decode(p, q, Kc, Vc, dtype, S, seqlens, batch, Hq, Hkv, Lmax, d, B,
                                      scale, O, idx, workspace,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

ssa_status ssa_decode_paged(const void* q, const void* Kp, const void* Vp, ssa_dtype dtype,
                            const float* S, const int32_t* page_table, int max_blocks,
                            int num_pages, const int32_t* seqlens, int batch, int Hq, int Hkv,
                            int d, int B, int topk, float scale, void* O, int32_t* idx,
                            void* workspace, size_t ws_bytes, ssa_stream stream) {
  ssa_status st = check_dims(d, B, dtype);
  if (st != SSA_OK) return st;
  if (batch <= 0 || Hq <= 0 || Hkv <= 0 || max_blocks <= 0 || num_pages <= 0 || topk < 0)
    return SSA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SSA_ERR_INVALID_ARG;
  if (Hq / Hkv > 8) return SSA_ERR_UNSUPPORTED;
  if (max_blocks > 16384) return SSA_ERR_UNSUPPORTED;
  if ((long long)max_blocks * B > 0x7fffffffLL || (long long)num_pages * Hkv > 0x7fffffffLL)
    return SSA_ERR_UNSUPPORTED;
  if (!(scale > 0.f)) return SSA_ERR_INVALID_ARG;
  if (q == nullptr || Kp == nullptr || Vp == nullptr || S == nullptr || page_table == nullptr ||
      seqlens == nullptr || O == nullptr || workspace == nullptr)
    return SSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(Kp) || !aligned16(Vp) || !aligned16(S) || !aligned16(O))
    return SSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SSA_ERR_INVALID_ARG;
  const int Lmax = max_blocks * B;
  const ssa::DecodePlan p = ssa::plan_decode(batch, Hq, Hkv, d, B, topk, Lmax);
  if (ws_bytes < p.bytes) return SSA_ERR_INVALID_ARG;
  ssa::CacheMap pm;
  pm.table = page_table;
  pm.max_blocks = max_blocks;
  pm.num_pages = num_pages;
  return from_cuda(ssa::launch_decode(p, q, Kp, Vp, dtype, S, seqlens, batch, Hq, Hkv, Lmax, d, B,
                                      scale, O, idx, workspace,
                                      reinterpret_cast<cudaStream_t>(stream), pm));
}

ssa_status ssa_decode_append_paged(void* Kp, void* Vp, ssa_dtype dtype, float* S,
                                   const int32_t* page_table, int max_blocks, int num_pages,
                                   int32_t* seqlens, const void* k_new, const void* v_new,
                                   int batch, int Hkv, int d, int B, ssa_stream stream) {
  ssa_status st = check_dims(d, B, dtype);
  if (st != SSA_OK) return st;
  if (batch <= 0 || Hkv <= 0 || max_blocks <= 0 || num_pages <= 0) return SSA_ERR_INVALID_ARG;
  if ((long long)max_blocks * B > 0x7fffffffLL) return SSA_ERR_UNSUPPORTED;
  if (Kp == nullptr || Vp == nullptr || S == nullptr || page_table == nullptr ||
      seqlens == nullptr || k_new == nullptr || v_new == nullptr)
    return SSA_ERR_INVALID_ARG;
  if (!aligned16(Kp) || !aligned16(Vp) || !aligned16(S) || !aligned16(k_new) ||
      !aligned16(v_new))
    return SSA_ERR_INVALID_ARG;
  ssa::CacheMap pm;
  pm.table = page_table;
  pm.max_blocks = max_blocks;
  pm.num_pages = num_pages;
  return from_cuda(ssa::launch_decode_append(Kp, Vp, dtype, S, seqlens, k_new, v_new, batch, Hkv,
                                             max_blocks * B, d, B,
                                             reinterpret_cast<cudaStream_t>(stream), pm));
}

ssa_status ssa_route_hierarchical(const void* Q, ssa_dtype dtype, const float* S, int batch,
                                  int Hq, int Hkv, int N, int d, int B, int M, int k_seg,
                                  int k_blk, int max_sel, int32_t* idx, int32_t* cnt,
                                  ssa_stream stream) {
  ssa_status st = check_dims(d, B, dtype);
  if (st != SSA_OK) return st;
  if (batch <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || Hq % Hkv != 0) return SSA_ERR_INVALID_ARG;
  if (M < 1 || k_seg < 0 || k_blk < 0) return SSA_ERR_INVALID_ARG;
  if (k_seg > 64) return SSA_ERR_UNSUPPORTED;
  const int nq = (N + B - 1) / B;
  if (max_sel < (k_blk < nq ? k_blk : nq) + 2) return SSA_ERR_INVALID_ARG;
  if ((size_t)4 * ((size_t)d + nq + nq / M + 1) > 200 * 1024) return SSA_ERR_UNSUPPORTED;
  if (Q == nullptr || idx == nullptr || cnt == nullptr || (N / B > 0 && S == nullptr))
    return SSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(S)) return SSA_ERR_INVALID_ARG;
  return from_cuda(ssa::launch_hier_route(Q, dtype, S, batch, Hq, Hkv, N, d, B, M, k_seg, k_blk,
                                          max_sel, idx, cnt,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

ssa_status ssa_decode_per_head_workspace_size(int batch, int Hq, int Hkv, int Lmax, int d, int B,
                                              int topk, size_t* bytes) {
  if (bytes == nullptr) return SSA_ERR_INVALID_ARG;
  ssa_status st = check_dims(d, B, SSA_BF16);
  if (st != SSA_OK) return st;
  if (batch <= 0 || Hq <= 0 || Hkv <= 0 || Lmax <= 0 || topk < 0) return SSA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SSA_ERR_INVALID_ARG;
  // the larger of the two layouts ssa_decode_per_head may use (it depends on the dtype)
  const size_t a = ssa::plan_decode(batch, Hq, Hq, d, B, topk, Lmax).bytes;
  const size_t u = ssa::plan_decode_union(batch, Hq, Hkv, d, B, topk, Lmax).bytes;
  *bytes = a > u ? a : u;
  return SSA_OK;
}

ssa_status ssa_decode_per_head(const void* q, const void* Kc, const void* Vc, ssa_dtype dtype,
                               const float* S, const int32_t* seqlens, int batch, int Hq, int Hkv,
                               int Lmax, int d, int B, int topk, float scale, void* O,
                               int32_t* idx, void* workspace, size_t ws_bytes,
                               ssa_stream stream) {
  ssa_status st = check_dims(d, B, dtype);
  if (st != SSA_OK) return st;
  if (batch <= 0 || Hq <= 0 || Hkv <= 0 || Lmax <= 0 || topk < 0) return SSA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SSA_ERR_INVALID_ARG;
  if (Lmax / B > 16384) return SSA_ERR_UNSUPPORTED;
  if (!(scale > 0.f)) return SSA_ERR_INVALID_ARG;
  if (q == nullptr || Kc == nullptr || Vc == nullptr || seqlens == nullptr || O == nullptr ||
      workspace == nullptr)
    return SSA_ERR_INVALID_ARG;
  if (Lmax / B > 0 && S == nullptr) return SSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(Kc) || !aligned16(Vc) || !aligned16(S) || !aligned16(O))
    return SSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SSA_ERR_INVALID_ARG;
  const size_t need_a = ssa::plan_decode(batch, Hq, Hq, d, B, topk, Lmax).bytes;
  const size_t need_u = ssa::plan_decode_union(batch, Hq, Hkv, d, B, topk, Lmax).bytes;
  if (ws_bytes < (need_a > need_u ? need_a : need_u)) return SSA_ERR_INVALID_ARG;
  if (dtype == SSA_BF16 && Hq / Hkv <= 8) {
    // One selection per query head; the split pass streams each KV head's
    // union of its heads' blocks once, the heads that did not choose a block
    // masked out of it.
    const ssa::DecodePlan p = ssa::plan_decode_union(batch, Hq, Hkv, d, B, topk, Lmax);
    return from_cuda(ssa::launch_decode(p, q, Kc, Vc, dtype, S, seqlens, batch, Hq, Hkv, Lmax, d,
                                        B, scale, O, idx, workspace,
                                        reinterpret_cast<cudaStream_t>(stream), ssa::CacheMap{}));
  }
  // Every query head is its own unit: the grouped path with one query head
  // per unit, each unit reading the cache head h / (Hq / Hkv).
  const ssa::DecodePlan p = ssa::plan_decode(batch, Hq, Hq, d, B, topk, Lmax);
  ssa::CacheMap cm;
  cm.kv_div = Hq / Hkv;
  return from_cuda(ssa::launch_decode(p, q, Kc, Vc, dtype, S, seqlens, batch, Hq, Hq, Lmax, d, B,
                                      scale, O, idx, workspace,
                                      reinterpret_cast<cudaStream_t>(stream), cm));
}

ssa_status ssa_decode_append(void* Kc, void* Vc, ssa_dtype dtype, float* S, int32_t* seqlens,
                             const void* k_new, const void* v_new, int batch, int Hkv, int Lmax,
                             int d, int B, ssa_stream stream) {
  ssa_status st = check_dims(d, B, dtype);
  if (st != SSA_OK) return st;
  if (batch <= 0 || Hkv <= 0 || Lmax <= 0) return SSA_ERR_INVALID_ARG;
  if (Kc == nullptr || Vc == nullptr || seqlens == nullptr || k_new == nullptr ||
      v_new == nullptr)
    return SSA_ERR_INVALID_ARG;
  if (Lmax / B > 0 && S == nullptr) return SSA_ERR_INVALID_ARG;
  if (!aligned16(Kc) || !aligned16(Vc) || !aligned16(S) || !aligned16(k_new) || !aligned16(v_new))
    return SSA_ERR_INVALID_ARG;
  return from_cuda(ssa::launch_decode_append(Kc, Vc, dtype, S, seqlens, k_new, v_new, batch, Hkv,
                                             Lmax, d, B, reinterpret_cast<cudaStream_t>(stream)));
}

ssa_status ssa_device_error(int* code) {
  if (code == nullptr) return SSA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return SSA_ERR_CUDA;
  int a = ssa::read_and_reset_attn_tc_error();
  int b = ssa::read_and_reset_decode_error();
  int c = ssa::read_and_reset_bwd_tc_error();
  *code = a != 0 ? a : (b != 0 ? b : c);
  return SSA_OK;
}

ssa_status ssa_check_device_error(ssa_stream stream, int* code) {
  if (code == nullptr) return SSA_ERR_INVALID_ARG;
  ErrorWords words{};
  if (ssa::attn_tc_error_word(&words.w[0]) != cudaSuccess) return SSA_ERR_CUDA;
  if (ssa::decode_error_word(&words.w[1]) != cudaSuccess) return SSA_ERR_CUDA;
  if (ssa::bwd_tc_error_word(&words.w[2]) != cudaSuccess) return SSA_ERR_CUDA;
  words.n = 3;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  take_error_words_kernel<<<1, 1, 0, s>>>(words);
  if (cudaGetLastError() != cudaSuccess) return SSA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_error_taken, sizeof(int), 0, cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return SSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SSA_ERR_CUDA;
  *code = v;
  return SSA_OK;
}

}  // extern "C"
