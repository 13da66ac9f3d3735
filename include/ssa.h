/*
 * ssa.h - C ABI of the block-sparse attention library with top-k summary routing.
 *
 * The method (DashAttention page, "Metodologia", stages 0-2; GSA page,
 * "Componentes Principais" 2-3; SSA page, "2. Metodologia", sparse stream):
 * keys are cut into contiguous blocks of B rows and each block is summarised
 * by its mean key; each query block scores the summaries of the complete key
 * blocks before it and keeps the top-k; the sink block 0 and the causal
 * diagonal block are always added; exact softmax attention then runs over the
 * keys of the selected blocks only.  Decode runs the same stages for one
 * query token per sequence against a KV cache.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Layout BHND: Q is [batch, Hq, N, d], K and V are [batch, Hkv, N, d], all
 *   contiguous with d innermost.  Query head h uses KV head h / (Hq / Hkv)
 *   (grouped-query attention, GQA).
 * - Every pointer argument is a DEVICE pointer, 16-byte aligned, owned by the
 *   caller.  The library allocates and frees nothing and keeps no state between
 *   calls other than a device-side error word (see ssa_device_error) and the
 *   fixed scratch array of ssa_decode_noalloc.
 * - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *   stream) and nothing synchronises with the host.
 * - Argument checks run on the host before any launch; a failed check returns
 *   an error code and launches nothing.  A launch failure returns SSA_ERR_CUDA.
 * - Supported: d in {64, 128}; B a multiple of 16 in [16, 128]; Hq % Hkv == 0;
 *   dtype SSA_F32 or SSA_BF16 (all of Q, K, V, O share it).
 * - Block counts: nq = ceil(N / B) query blocks; nfull = floor(N / B) complete
 *   key blocks.  A trailing partial block has no summary and is only ever
 *   attended as a diagonal block.
 */
#ifndef SSA_H
#define SSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SSA_OK = 0,
  SSA_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer */
  SSA_ERR_UNSUPPORTED = 2, /* valid but not implemented (d, B, dtype, sizes) */
  SSA_ERR_CUDA = 3,        /* a CUDA launch or runtime call failed */
  SSA_ERR_TIMEOUT = 4      /* a bounded device-side wait expired (see ssa_device_error) */
} ssa_status;

typedef enum { SSA_F32 = 0, SSA_BF16 = 1 } ssa_dtype;

/* Opaque CUDA stream handle; binary-compatible with cudaStream_t. */
typedef struct CUstream_st* ssa_stream;

/* Human-readable name of a status code.  Never NULL. */
const char* ssa_status_string(int status);

/* Library ABI version (major * 100 + minor).  1.01 added ssa_decode_append,
 * 1.02 ssa_sparse_attn_bwd; 2.00 added the `scores` output of ssa_route (an
 * incompatible signature change) and ssa_check_device_error; 2.01 the paged
 * cache (ssa_decode_paged, ssa_decode_append_paged); 2.02 DashAttention's
 * adaptive stages (ssa_learned_summary, ssa_route_entmax,
 * ssa_sparse_attn_fwd_prior); 2.03 the routing variants (ssa_route_hierarchical,
 * ssa_decode_per_head, ssa_decode_per_head_workspace_size); 2.04 the backward
 * takes a sized workspace (ssa_sparse_attn_bwd_workspace_size) in place of
 * its delta scratch. */
int ssa_version(void);

/*
 * Stage 0, block summary (DashAttention page, "Estágio 0": with the learned
 * summary query at zero the block summary is the uniform mean; GSA page,
 * "Componentes Principais" 2: MoBA's mean pooling).
 *
 *   S[b, g, j, :] = (1 / B) * sum_{t = jB}^{jB + B - 1} K[b, g, t, :]   for j < nfull
 *
 * K: [batch, Hkv, N, d] of `dtype`.  S: [batch, Hkv, nfull, d] fp32 (written).
 * N < B is valid and writes nothing.
 */
ssa_status ssa_block_summary(const void* K, ssa_dtype dtype, int batch, int Hkv, int N, int d,
                             int B, float* S, ssa_stream stream);

/*
 * Stage 1, routing (DashAttention page, "Estágio 1": each query scores the
 * block summaries; GQA heads sharing a KV head share one support; The Sparse
 * Frontier page, RQ2: block-wise selection in prefill; GSA page,
 * "Componentes Principais" 3: top-k of the blocks).
 *
 * For every (b, KV head g, query block i):
 *   qbar = mean of Q over the rows of block i and the heads of group g;
 *   s_j  = qbar . S[b, g, j, :] / sqrt(d) for candidates j = 1 .. i-1;
 *   R    = the min(topk, i-1) candidates of highest s_j, equal scores going to
 *          the lower block index;
 *   selection = {0} U R U {i}, written ascending.
 * Scores are computed in fp32 from the fp32 summaries.
 *
 * Q: [batch, Hq, N, d] of `dtype`.  S: [batch, Hkv, nfull, d] fp32.
 * idx: [batch, Hkv, nq, max_sel] int32 (written; entries past cnt are -1).
 * cnt: [batch, Hkv, nq] int32 (written).
 * scores: NULL, or [batch, Hkv, nq, nfull] fp32 (written): scores[b, g, i, j]
 *    is the fp32 score s_j that the selection ranked, for the candidates
 *    j = 1 .. i-1, and -inf for every other j (the sink, the diagonal block
 *    and later blocks).  16-byte aligned.
 * topk >= 0; any topk >= nq selects every candidate.
 * max_sel must be >= min(topk, max(nq - 2, 0)) + 2.
 * SSA_ERR_UNSUPPORTED if nq > 16384 (the score rows of a tile of query
 * blocks are held in shared memory: tiles of 8 query blocks up to about 6800
 * blocks, then of 4 and of 2).
 */
ssa_status ssa_route(const void* Q, ssa_dtype dtype, const float* S, int batch, int Hq, int Hkv,
                     int N, int d, int B, int topk, int max_sel, int32_t* idx, int32_t* cnt,
                     float* scores, ssa_stream stream);

/*
 * Stage 2, exact softmax attention over the selected blocks (SSA page,
 * "2. Metodologia", sparse stream; DashAttention page, "Estágio 2", attention
 * restricted to the routed blocks plus the diagonal branch).
 *
 * For query row t of head h (block i = t / B, group g = h / (Hq / Hkv)) the
 * keys are the rows of the blocks idx[b, g, i, 0 .. cnt-1] at key positions
 * <= t (the causal mask binds only on the diagonal block):
 *   O[b, h, t, :] = softmax(scale * q_t . K_sel^T) V_sel
 *   lse[b, h, t]  = log(sum exp(scale * q_t . K_sel^T))   (natural log)
 * Accumulation is fp32; O is rounded to `dtype` (round to nearest even).
 *
 * idx/cnt as written by ssa_route (entries ascending, each in [0, i], the
 * diagonal i included).  lse may be NULL.  scale > 0 (normally 1/sqrt(d)).
 * bf16 with d = 128, B in {64, 128} and (Hq/Hkv)*B a multiple of 256 runs on
 * the tensor cores (TMA + tcgen05 + TMEM); every other shape runs a SIMT kernel.
 * A bounded device-side wait that expires sets the device error word
 * (SSA_ERR_TIMEOUT, see ssa_device_error) instead of hanging.
 */
ssa_status ssa_sparse_attn_fwd(const void* Q, const void* K, const void* V, ssa_dtype dtype,
                               const int32_t* idx, const int32_t* cnt, int batch, int Hq, int Hkv,
                               int N, int d, int B, int max_sel, float scale, void* O, float* lse,
                               ssa_stream stream);

/*
 * DashAttention's adaptive stages (DashAttention page, "Metodologia").  The
 * page names alpha-entmax without a formula; it is taken as the standard map
 *   entmax_alpha(x)_j = [(alpha - 1) x_j - tau]_+ ^ (1 / (alpha - 1)),
 * tau chosen so that the entries sum to 1 (alpha = 2 is sparsemax).
 */

/*
 * Stage 0 with a learned summary query ("Estágio 0": a local attention inside
 * each block, pooled by one learned query):
 *   S[b, g, j, :] = sum_t softmax_t(scale * qbar[g] . K[b, g, t]) K[b, g, t, :]
 * over the B keys t of each complete block j, scale = 1/sqrt(d).  qbar = 0
 * gives the mean of ssa_block_summary.
 * K: [batch, Hkv, N, d] of `dtype`; qbar: [Hkv, d] fp32 (one learned query per
 * KV head); S: [batch, Hkv, nfull, d] fp32 (written).  One warp per block.
 */
ssa_status ssa_learned_summary(const void* K, ssa_dtype dtype, const float* qbar, int batch,
                               int Hkv, int N, int d, int B, float* S, ssa_stream stream);

/*
 * Stage 1 with alpha-entmax routing ("Estágio 1": each query head scores the
 * summaries, alpha-entmax turns the scores into sparse routing
 * probabilities, and the heads of a GQA group average their probabilities so
 * that they share one support).  For every (b, KV head g, query block i):
 *   for each query head h of group g: qbar_h = mean of head h's rows of block
 *     i; z_j = gamma * qbar_h . S[b, g, j] / sqrt(d) for the candidates
 *     j = 0 .. min(i, nfull) - 1 (the complete blocks before i);
 *     p_h = entmax_alpha(z) (tau by 40 bisection steps in fp32 on
 *     [max - 1, max] of (alpha - 1) z);
 *   w = mean over the group's heads of p_h.
 * Written per row: idx = the support {j : w_j > 0} ascending, then the
 * diagonal block i; bias = sigma * ln(w_j) for each support entry and 0 for
 * the diagonal (the prior of stage 2); cnt = the number of entries; entries
 * past cnt are -1 (idx) and 0 (bias).  w: NULL, or [batch, Hkv, nq, nfull]
 * fp32 (written; 0 off the candidates).
 * idx, bias: [batch, Hkv, nq, max_sel] with max_sel >= min(nq - 1, nfull) + 1.
 * 1 < alpha <= 8, gamma > 0, sigma >= 0.  One CTA per (b, g, i); its
 * candidate rows live in shared memory, so nq is limited to about 25000.
 */
ssa_status ssa_route_entmax(const void* Q, ssa_dtype dtype, const float* S, int batch, int Hq,
                            int Hkv, int N, int d, int B, float alpha, float gamma, float sigma,
                            int max_sel, int32_t* idx, int32_t* cnt, float* bias, float* w,
                            ssa_stream stream);

/*
 * Stage 2 with the prior-induced softmax ("Estágio 2": the routing
 * probabilities act as a prior g ~ w^sigma on the routed keys; the maximiser
 * of z.p - KL(p || g) is p ~ g exp(z), so a routed key's logit gains
 * sigma * ln w_j; the diagonal branch has no prior; every other key is
 * masked).  As ssa_sparse_attn_fwd, with bias[b, g, i, e] added to the scaled
 * logits of every key of block idx[b, g, i, e] (the causal mask still binds
 * on the diagonal):
 *   O[b, h, t] = softmax(scale * q_t . K_sel^T + bias_sel) V_sel.
 * idx, cnt, bias as written by ssa_route_entmax (bias [batch, Hkv, nq,
 * max_sel] fp32).  The shapes of ssa_sparse_attn_fwd's tensor-core path (bf16,
 * d = 128, B in {64, 128}, (Hq/Hkv)*B a multiple of 256) run on that kernel,
 * with the offset joining each block's scaled logits; others run the FFMA
 * kernel.
 */
ssa_status ssa_sparse_attn_fwd_prior(const void* Q, const void* K, const void* V,
                                     ssa_dtype dtype, const int32_t* idx, const int32_t* cnt,
                                     const float* bias, int batch, int Hq, int Hkv, int N, int d,
                                     int B, int max_sel, float scale, void* O, float* lse,
                                     ssa_stream stream);

/*
 * Two-level routing (Gist Sparse Attention page, "Componentes Principais" 4,
 * H-GSA: a coarse level over groups of blocks narrows the fine level).
 * A segment is M consecutive complete blocks (segment m holds blocks mM ..
 * mM + M - 1); its score is the mean of its blocks' scores, which equals
 * qbar . (mean of their summaries) / sqrt(d).  For every (b, KV head g, query
 * block i), with qbar and the block scores s_j of ssa_route:
 *   - a segment is closed when all its blocks lie before i ((m + 1) M <= i);
 *     the closed segments holding a candidate compete, and the top k_seg of
 *     them are kept (equal scores: lower segment index);
 *   - the pool is the candidates 1 .. i-1 inside a kept segment or inside no
 *     closed segment (the segment still open at i goes straight to the block
 *     level, as the diagonal block goes straight to attention);
 *   - R = the top min(k_blk, pool size) of the pool by s_j (ties: lower
 *     index); selection = {0} U R U {i}, ascending, -1 padded.
 * M = 1 with k_seg >= nq is the flat ssa_route.  idx, cnt as for ssa_route,
 * with max_sel >= min(k_blk, nq) + 2.  k_seg <= 64.  Query blocks are taken
 * in tiles of 8 per CTA with the pooling and scoring of ssa_route (the same
 * fp32 scores, bitwise), while the tile's score rows fit in shared memory
 * (about 6000 complete blocks with large M); beyond that one CTA per query
 * block, whose sums run in another order.
 */
ssa_status ssa_route_hierarchical(const void* Q, ssa_dtype dtype, const float* S, int batch,
                                  int Hq, int Hkv, int N, int d, int B, int M, int k_seg,
                                  int k_blk, int max_sel, int32_t* idx, int32_t* cnt,
                                  ssa_stream stream);

/*
 * Backward pass of stage 2 with the selection held fixed (DashAttention page,
 * "Declaração do Problema" 2: hard top-k passes no gradient to the routing;
 * SSA page, "1. Definição do Problema" 2: keys outside the selected blocks get
 * zero gradient; AdaSplash-2 page, "4. Resultados Experimentais": the backward
 * skips the zero blocks).
 *
 * With P the softmax of ssa_sparse_attn_fwd (rebuilt as exp(scale q.k - lse))
 * and dO the gradient of the loss with respect to O:
 *   delta[b, h, t] = dO[b, h, t, :] . O[b, h, t, :]
 *   dS             = P * (dO V_sel^T - delta)
 *   dQ             = scale * dS K_sel
 *   dK[b, g]      += scale * dS^T Q,   dV[b, g] += P^T dO
 * dK and dV sum over the query heads of group g and over every query block
 * whose selection holds the key's block; keys no query sees get 0.  Every
 * output element is written exactly once, in a fixed summation order (no
 * atomics), so the result is deterministic.
 *
 * Q, O, dO, dQ: [batch, Hq, N, d]; K, V, dK, dV: [batch, Hkv, N, d]; all bf16
 * (SSA_ERR_UNSUPPORTED for SSA_F32).  lse: [batch, Hq, N] fp32 as written by
 * ssa_sparse_attn_fwd; idx/cnt: as written by ssa_route (ascending entries).
 * workspace: caller-owned device scratch of at least
 * ssa_sparse_attn_bwd_workspace_size(...) bytes, 256-byte aligned, contents on
 * entry ignored.  It holds delta and the partial sums of the sink block
 * (block 0, which every query block selects): its dK and dV are summed over
 * ranges of query blocks by separate CTAs, and the ranges are added in a
 * fixed order; for d = 128, B = 64 and (Hq / Hkv) * B a multiple of 256 it
 * also holds the selection transposed as per-key-block bit masks.  Calls that
 * share a workspace must not overlap on the device.  The contractions run on
 * tensor cores (tcgen05 with TMEM accumulators for the forward's tensor-core
 * shapes, mma.sync tiles otherwise; bf16 in, fp32 accumulate); P and dS are
 * rounded to bf16 as operands, outputs to bf16.
 */
ssa_status ssa_sparse_attn_bwd(const void* Q, const void* K, const void* V, const void* O,
                               const void* dO, const float* lse, ssa_dtype dtype,
                               const int32_t* idx, const int32_t* cnt, int batch, int Hq, int Hkv,
                               int N, int d, int B, int max_sel, float scale, void* dQ, void* dK,
                               void* dV, void* workspace, size_t ws_bytes, ssa_stream stream);

/* Scratch size, in bytes, that ssa_sparse_attn_bwd needs for these sizes. */
ssa_status ssa_sparse_attn_bwd_workspace_size(int batch, int Hq, int Hkv, int N, int d, int B,
                                              size_t* bytes);

/*
 * 1 if ssa_sparse_attn_fwd runs this shape on the tensor cores, else 0 (the
 * SIMT kernel).  Pure host query.
 */
int ssa_sparse_attn_uses_tensor_cores(ssa_dtype dtype, int Hq, int Hkv, int d, int B);

/*
 * Scratch size, in bytes, that ssa_decode needs for these sizes.
 */
ssa_status ssa_decode_workspace_size(int batch, int Hq, int Hkv, int Lmax, int d, int B,
                                     int topk, size_t* bytes);

/*
 * One decode step (DashAttention page, "Contribuições Principais" 4:
 * incremental decoding with the same stages; The Sparse Frontier page, RQ2:
 * decode keeps the whole KV cache and loads only the selected blocks).
 *
 * Sequence b holds L = seqlens[b] tokens in its cache, the current token
 * included, so the query sits at position L-1 and its diagonal block is
 * last = (L-1) / B (possibly partial; its keys at positions >= L are masked).
 *   qbar = mean over the group's heads of q;  s_j = qbar . S[b, g, j] / sqrt(d)
 *   for the complete blocks j = 1 .. last-1; selection = {0} U top-k U {last}.
 * The selected blocks are split across CTAs (split-KV) and the partial
 * results are merged with a log-sum-exp combine.
 *
 * q: [batch, Hq, d]; Kc, Vc: [batch, Hkv, Lmax, d] of `dtype`;
 * S: [batch, Hkv, Lmax / B, d] fp32 block summaries of the cache (only the
 *    complete blocks before `last` are read);
 * seqlens: [batch] int32, 1 <= seqlens[b] <= Lmax (read on the device; a value
 *    out of range makes that sequence write zeros);
 * O: [batch, Hq, d] of `dtype` (written);
 * idx: NULL or [batch, Hkv, min(topk, ceil(Lmax / B)) + 2] int32 (written,
 *    ascending, -1 padded);
 * workspace: >= ssa_decode_workspace_size(...) bytes of device memory, 256-byte
 *    aligned, contents on entry ignored.  Calls that share a workspace must
 *    not overlap on the device.
 */
ssa_status ssa_decode(const void* q, const void* Kc, const void* Vc, ssa_dtype dtype,
                      const float* S, const int32_t* seqlens, int batch, int Hq, int Hkv, int Lmax,
                      int d, int B, int topk, float scale, void* O, int32_t* idx, void* workspace,
                      size_t ws_bytes, ssa_stream stream);

/*
 * Decode with per-query-head routing (The Sparse Frontier page, RQ2: in
 * decode each query can afford its own selection -- Quest selects pages per
 * query -- while the whole cache stays resident).  As ssa_decode, except that
 * every query head h routes on its own query instead of the group mean:
 *   s_j = q[b, h] . S[b, h / G, j] / sqrt(d), j = 1 .. last-1;
 *   selection_h = {0} U top-k U {last};
 * and attends only its own selection, reading the cache head h / G.
 * idx: NULL or [batch, Hq, min(topk, ceil(Lmax / B)) + 2] int32 (written).
 * workspace: ssa_decode_per_head_workspace_size(...) bytes, 256-byte aligned.
 * Any G = Hq / Hkv.  For bf16 with G <= 8 the cache blocks of a KV head are
 * streamed once for the union of its heads' selections, each head masked out
 * of the blocks it did not choose; otherwise every query head is a unit of
 * its own.
 */
ssa_status ssa_decode_per_head_workspace_size(int batch, int Hq, int Hkv, int Lmax, int d, int B,
                                              int topk, size_t* bytes);

ssa_status ssa_decode_per_head(const void* q, const void* Kc, const void* Vc, ssa_dtype dtype,
                               const float* S, const int32_t* seqlens, int batch, int Hq, int Hkv,
                               int Lmax, int d, int B, int topk, float scale, void* O,
                               int32_t* idx, void* workspace, size_t ws_bytes,
                               ssa_stream stream);

/*
 * Append one token per sequence to the decode KV cache and keep its block
 * summaries current (DashAttention page, "Contribuições Principais" 4,
 * incremental decoding; "Estágio 0": a block's summary is the mean of its B
 * keys, formed once the block is complete).
 *
 * For sequence b holding L = seqlens[b] tokens with 0 <= L < Lmax:
 *   Kc[b, g, L, :] = k_new[b, g, :],  Vc[b, g, L, :] = v_new[b, g, :]  (all g)
 *   if (L + 1) % B == 0:  S[b, g, (L+1)/B - 1, :] = mean over that block's B
 *                         keys (fp32 sum, then / B)
 *   seqlens[b] = L + 1.
 * A sequence with L outside [0, Lmax) is left unchanged (its cache is full or
 * its length invalid).  After the call, ssa_decode with the same seqlens
 * attends the new token as the current one.
 *
 * Kc, Vc: [batch, Hkv, Lmax, d] of `dtype` (modified in place);
 * S: [batch, Hkv, Lmax / B, d] fp32 (modified in place; may be NULL only if
 *    Lmax < B);
 * seqlens: [batch] int32 (read and raised in place, on the device);
 * k_new, v_new: [batch, Hkv, d] of `dtype`.
 * All device pointers, 16-byte aligned.  Supported: d in {64, 128}; B a
 * multiple of 16 in [16, 128].  Calls on one cache must not overlap on the
 * device.
 */
ssa_status ssa_decode_append(void* Kc, void* Vc, ssa_dtype dtype, float* S, int32_t* seqlens,
                             const void* k_new, const void* v_new, int batch, int Hkv, int Lmax,
                             int d, int B, ssa_stream stream);

/*
 * Decode and append over a paged KV cache (The Sparse Frontier page, RQ2:
 * decode keeps the whole cache and loads only the selected blocks;
 * DashAttention page, "Contribuições Principais" 4: incremental decoding).
 * The same computation as ssa_decode / ssa_decode_append on the cache the
 * page table describes, with no copy into a contiguous cache.
 *
 * Layout: a page holds one block of B tokens for every KV head of one
 * sequence, so the page pools are Kp, Vp: [num_pages, Hkv, B, d] of `dtype`.
 * page_table: [batch, max_blocks] int32; page_table[b, j] is the page of
 * logical block j of sequence b, or -1 for none.  Sequences may share pages
 * (a common prefix).  The cache of sequence b has room for Lmax = max_blocks *
 * B tokens.  S: [batch, Hkv, max_blocks, d] fp32 block summaries, per sequence
 * in logical block order.
 *
 * ssa_decode_paged: arguments and results as ssa_decode with Lmax =
 * max_blocks * B (seqlens, O, idx, workspace of ssa_decode_workspace_size for
 * that Lmax).  Every block that holds tokens of a sequence (j <= (L-1) / B)
 * must have a page; a selected block without one is skipped (it adds no
 * keys).  Rows of a page past the sequence's length are never read as keys.
 *
 * ssa_decode_append_paged: as ssa_decode_append; the new rows go to row L % B
 * of page page_table[b, L / B], and a block completed by the append gets its
 * summary in S[b, :, L / B].  A sequence whose next block has no page is left
 * unchanged (its length is not raised).
 * Both: device pointers, 16-byte aligned (the workspace 256-byte aligned).
 */
ssa_status ssa_decode_paged(const void* q, const void* Kp, const void* Vp, ssa_dtype dtype,
                            const float* S, const int32_t* page_table, int max_blocks,
                            int num_pages, const int32_t* seqlens, int batch, int Hq, int Hkv,
                            int d, int B, int topk, float scale, void* O, int32_t* idx,
                            void* workspace, size_t ws_bytes, ssa_stream stream);

ssa_status ssa_decode_append_paged(void* Kp, void* Vp, ssa_dtype dtype, float* S,
                                   const int32_t* page_table, int max_blocks, int num_pages,
                                   int32_t* seqlens, const void* k_new, const void* v_new,
                                   int batch, int Hkv, int d, int B, ssa_stream stream);

/*
 * Largest scratch area ssa_decode_noalloc can use (40 MiB).
 */
#define SSA_DECODE_NOALLOC_MAX_BYTES ((size_t)40 << 20)

/*
 * ssa_decode without a caller-supplied workspace.  The pages have no
 * counterpart: this is a library convenience.
 *
 * For callers that cannot allocate device memory at call time: code whose
 * device memory is owned by another allocator it cannot reach, fixed-budget
 * plug-in hosts, and serving loops where cudaMalloc (which may synchronise the
 * device) is not allowed.  Arguments and results are those of ssa_decode
 * minus `workspace` / `ws_bytes`; the scratch lives in one fixed device array
 * of SSA_DECODE_NOALLOC_MAX_BYTES inside the library, which every GPU that
 * loads the library holds until the process exits.
 * - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * - The first call on each device looks up that device's address of the array
 *   (with the device current), so make that first call before any stream
 *   capture; later calls only read the cached address.  The cached address
 *   belongs to the device's primary context as it was at that first call: after
 *   cudaDeviceReset on that device it is stale, so do not call this entry point
 *   on a device that was reset after its first call.
 * - All calls share the one array and it keeps the previous call's contents;
 *   everything that must start at zero is cleared by the call itself.  Calls
 *   that overlap on the GPU (other streams, other host threads) race on it:
 *   order them.
 * - SSA_ERR_UNSUPPORTED if ssa_decode_workspace_size for these sizes exceeds
 *   SSA_DECODE_NOALLOC_MAX_BYTES (checked on the host; nothing is launched).
 */
ssa_status ssa_decode_noalloc(const void* q, const void* Kc, const void* Vc, ssa_dtype dtype,
                              const float* S, const int32_t* seqlens, int batch, int Hq, int Hkv,
                              int Lmax, int d, int B, int topk, float scale, void* O,
                              int32_t* idx, ssa_stream stream);

/*
 * Device error word: 0, or the ssa_status of the first bounded device-side
 * wait that expired since the last reset.  Synchronises the device, then
 * writes the word to *code and resets it to 0.
 */
ssa_status ssa_device_error(int* code);

/*
 * The device error word, read in stream order: enqueues on `stream` a
 * one-thread kernel that takes the word (atomic exchange with 0), copies it
 * back, and waits for `stream` only (cudaStreamSynchronize; other streams
 * keep running).  *code is 0, or the ssa_status of the first bounded wait that
 * expired in work that finished before that kernel ran, on any stream of the
 * current device.  The copy goes through one result word of the library per
 * device: calls from several host threads at once must be serialised.  Not
 * for use during stream capture (it synchronises).
 */
ssa_status ssa_check_device_error(ssa_stream stream, int* code);

#ifdef __cplusplus
}
#endif

#endif /* SSA_H */
