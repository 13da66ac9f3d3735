// Host-side launchers of the library's kernels (internal; the public ABI is ssa.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "ssa.h"

namespace ssa {

cudaError_t launch_block_summary(const void* K, ssa_dtype dt, int batch, int Hkv, int N, int d,
                                 int B, float* S, cudaStream_t st);

// Largest number of query blocks ssa_route handles (its score rows live in
// shared memory).
constexpr int kRouteMaxBlocks = 16384;

cudaError_t launch_route(const void* Q, ssa_dtype dt, const float* S, int batch, int Hq, int Hkv,
                         int N, int d, int B, int topk, int max_sel, int32_t* idx, int32_t* cnt,
                         float* scores, cudaStream_t st);

// True when the tensor-core prefill kernel covers this shape.
bool attn_tc_supported(ssa_dtype dt, int Hq, int Hkv, int d, int B);

// bias: NULL, or the routing prior of each selection entry (natural log) added
// to the scaled logits of that block's keys.
cudaError_t launch_attn_tc(const void* Q, const void* K, const void* V, const int32_t* idx,
                           const int32_t* cnt, const float* bias, int batch, int Hq, int Hkv,
                           int N, int B, int max_sel, float scale, void* O, float* lse,
                           cudaStream_t st);

cudaError_t launch_attn_simt(const void* Q, const void* K, const void* V, ssa_dtype dt,
                             const int32_t* idx, const int32_t* cnt, const float* bias, int batch,
                             int Hq, int Hkv, int N, int d, int B, int max_sel, float scale,
                             void* O, float* lse, cudaStream_t st);

// DashAttention's adaptive stages (learned summary, alpha-entmax routing).
cudaError_t launch_learned_summary(const void* K, ssa_dtype dt, const float* qbar, int batch,
                                   int Hkv, int N, int d, int B, float* S, cudaStream_t st);
cudaError_t launch_entmax_route(const void* Q, ssa_dtype dt, const float* S, int batch, int Hq,
                                int Hkv, int N, int d, int B, float alpha, float gamma,
                                float sigma, int max_sel, int32_t* idx, int32_t* cnt,
                                float* bias, float* w, cudaStream_t st);

// Backward pass of stage 2: delta, dQ, dK, dV.  The workspace holds delta
// ([batch, Hq, N] fp32), the sink column's partial sums
// ([sink_nsplit][batch * Hkv][2][B][d] fp32) and, for the tensor-core dK / dV
// pass, the selection transposed as bit masks: word w of (bg, key block j)
// has bit t set when query block 32 w + t selects j ([batch * Hkv][nq][nwin]
// uint32, nwin = ceil(nq / 32); nwin = 0 when that pass is not used).
struct BwdPlan {
  int sink_qr;      // query blocks per sink range
  int sink_nsplit;  // sink ranges per (batch, KV head)
  int nwin;         // mask words per key block (0: no mask)
  size_t off_delta, off_part, off_mask, bytes;
};
BwdPlan plan_bwd(int batch, int Hq, int Hkv, int N, int d, int B);
size_t attn_bwd_smem_bytes(int d, int B);
// Tensor-core (tcgen05) forms of the two contraction passes, for the shapes of
// attn_tc_supported (dK / dV: B = 64 only); the sink ranges as in the
// mma.sync form.
cudaError_t launch_bwd_dq_tc(const void* Q, const void* K, const void* V, const void* dO,
                             const float* lse, const float* delta, const int32_t* idx,
                             const int32_t* cnt, int batch, int Hq, int Hkv, int N, int B,
                             int max_sel, float scale, void* dQ, cudaStream_t st);
cudaError_t launch_bwd_dkv_tc(const void* Q, const void* K, const void* V, const void* dO,
                              const float* lse, const float* delta, int batch, int Hq, int Hkv,
                              int N, float scale, void* dK, void* dV, float* sink_part,
                              int sink_qr, int sink_nsplit, const uint32_t* hitmask, int nwin,
                              cudaStream_t st);
cudaError_t launch_attn_bwd(const BwdPlan& pl, const void* Q, const void* K, const void* V,
                            const void* O, const void* dO, const float* lse, const int32_t* idx,
                            const int32_t* cnt, int batch, int Hq, int Hkv, int N, int d, int B,
                            int max_sel, float scale, void* dQ, void* dK, void* dV, void* ws,
                            cudaStream_t st);

// How the decode kernels address the KV cache.
// - Paged: page pool [num_pages, Hc, B, d]; table[b * max_blocks + j] is the
//   page of sequence b's logical block j (-1: none).  table == nullptr means
//   the contiguous cache [batch, Hc, Lmax, d].
// - kv_div: the kernels' head units are cache heads (kv_div = 1) or query
//   heads routed one by one (kv_div = Hq / Hkv): unit head u of sequence b
//   reads cache head u / kv_div, and Hc = (unit heads) / kv_div.
struct CacheMap {
  const int32_t* table = nullptr;
  int max_blocks = 0;
  int num_pages = 0;
  int kv_div = 1;
};

// Decode: scratch layout and launch.
struct DecodePlan {
  int G;          // query heads per KV head
  int nblk_max;   // ceil(Lmax / B)
  int kk;         // effective top-k: min(topk, nblk_max)
  int width;      // idx row width: kk + 2
  int parts_max;  // partial records per (sequence, KV head) the scratch holds
  int head_width; // 0: one selection per KV head; else one per query head, of this width,
                  // and the split pass streams their union (bf16, G <= 8)
  size_t off_idx, off_cnt, off_part, off_ctr, bytes;
};

DecodePlan plan_decode(int batch, int Hq, int Hkv, int d, int B, int topk, int Lmax);
// One selection per query head; the KV head's scratch row holds the union of
// its G heads' blocks, each entry j | (head mask << 24).
DecodePlan plan_decode_union(int batch, int Hq, int Hkv, int d, int B, int topk, int Lmax);

cudaError_t launch_decode(const DecodePlan& p, const void* q, const void* Kc, const void* Vc,
                          ssa_dtype dt, const float* S, const int32_t* seqlens, int batch, int Hq,
                          int Hkv, int Lmax, int d, int B, float scale, void* O, int32_t* idx_out,
                          void* ws, cudaStream_t st, CacheMap pm = CacheMap{});

cudaError_t launch_decode_append(void* Kc, void* Vc, ssa_dtype dt, float* S, int32_t* seqlens,
                                 const void* k_new, const void* v_new, int batch, int Hkv,
                                 int Lmax, int d, int B, cudaStream_t st, CacheMap pm = CacheMap{});

// Two-level routing: segments of M complete blocks, then blocks.
cudaError_t launch_hier_route(const void* Q, ssa_dtype dt, const float* S, int batch, int Hq,
                              int Hkv, int N, int d, int B, int M, int k_seg, int k_blk,
                              int max_sel, int32_t* idx, int32_t* cnt, cudaStream_t st);

// Device error words (one per translation unit that has bounded waits):
// read and reset; returns the first non-zero code or 0.
int read_and_reset_attn_tc_error();
int read_and_reset_decode_error();
// Device addresses of the same words (current device), for stream-ordered reads.
cudaError_t attn_tc_error_word(int** word);
cudaError_t decode_error_word(int** word);
int read_and_reset_bwd_tc_error();
cudaError_t bwd_tc_error_word(int** word);

}  // namespace ssa
