"""Plain fp64 CPU oracle for block-sparse attention with top-k summary routing.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module:
only the tests, the package smoke check and the benchmark's CPU-baseline leg
call it.  It shares no code with the CUDA library and imports nothing from it.

What it computes, in the order the pages give the pipeline (DashAttention page,
"Metodologia": three stages; GSA page, "Componentes Principais" 2-3):

* stage 0, block summary: the context is cut into contiguous blocks of size B
  and each key block is pooled to one vector.  The pooling is the uniform mean
  (DashAttention page, "Estágio 0": the learned summary query starts at zero,
  which makes it uniform mean pooling; GSA page, "Componentes Principais" 2:
  MoBA's mean pooling);
* stage 1, routing: each query block scores the summaries of the complete key
  blocks strictly before it and keeps the top-k (DashAttention page,
  "Declaração do Problema" and "Estágio 1"; GSA page, "Componentes Principais"
  3).  Routing is per query block in prefill (The Sparse Frontier page, RQ2:
  block-wise selection is the prefill choice).  Query heads that share a KV
  head share one selection (DashAttention page, "Estágio 1", GQA handling):
  their scores are averaged.  The sink block 0 and the diagonal block are
  always added (DashAttention page, "Estágio 2", diagonal branch);
* stage 2: exact softmax attention over the keys of the selected blocks only,
  causally masked (SSA page, "2. Metodologia", sparse stream; DashAttention
  page, "Estágio 2");
* decode: the same stages for one query token at the end of a KV cache
  (DashAttention page, "Contribuições Principais" 4; The Sparse Frontier page,
  RQ2, decode keeps the whole cache and loads selected pages);
* incremental decoding keeps the cache and its summaries current: each new
  token's key and value are appended, and a block's summary is formed once
  the block is complete (DashAttention page, "Contribuições Principais" 4 and
  "Estágio 0");
* training: the backward pass of stage 2.  The hard top-k selection passes
  no gradient to the routing or the summaries (DashAttention page,
  "Declaração do Problema" 2), and keys outside the selected blocks get zero
  gradient (SSA page, "1. Definição do Problema" 2; AdaSplash-2 page,
  "4. Resultados Experimentais": the backward skips zero-gradient blocks).
  So the gradients are those of stage 2 with the selection held fixed.

Every array is float64.  bf16 and fp32 inputs upcast to float64 exactly.
Where the pages leave a step open, the reading taken is stated at the function.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "block_summary",
    "pool_query_blocks",
    "summary_scores",
    "select_topk",
    "route",
    "sparse_attention",
    "attention_probs",
    "decode_route",
    "decode",
    "decode_append",
    "sparse_attention_backward",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def block_summary(K, B: int) -> np.ndarray:
    """Mean of K over each complete block of B keys.

    K: ``[batch, Hkv, N, d]``.  Returns ``S``: ``[batch, Hkv, N // B, d]``.
    A trailing partial block has no summary: it can only ever be a diagonal
    block, which is always selected and never scored (DashAttention page,
    "Estágio 0": a block's summary exists once the block is complete).
    """
    K = _f64(K)
    b, h, N, d = K.shape
    nfull = N // B
    return K[:, :, : nfull * B, :].reshape(b, h, nfull, B, d).mean(axis=3)


def pool_query_blocks(Q, B: int, Hkv: int) -> np.ndarray:
    """Mean of Q over the rows of each query block and the heads of each GQA group.

    Q: ``[batch, Hq, N, d]``; query head h belongs to KV head ``h // (Hq // Hkv)``.
    Returns ``[batch, Hkv, ceil(N / B), d]``.  A trailing partial query block
    is averaged over the rows it has.
    """
    Q = _f64(Q)
    b, Hq, N, d = Q.shape
    G = Hq // Hkv
    nq = -(-N // B)
    out = np.empty((b, Hkv, nq, d))
    for i in range(nq):
        rows = Q[:, :, i * B : min(N, (i + 1) * B), :]  # [b, Hq, r, d]
        grp = rows.reshape(b, Hkv, G, rows.shape[2], d)
        out[:, :, i, :] = grp.mean(axis=(2, 3))
    return out


def summary_scores(qbar, S) -> np.ndarray:
    """Score of every (query block, key block) pair: ``qbar_i . S_j / sqrt(d)``.

    By linearity this equals the mean, over the block's query rows and the
    group's heads, of ``q . S_j / sqrt(d)``.  Returns ``[batch, Hkv, nq, nfull]``.
    """
    qbar = _f64(qbar)
    S = _f64(S)
    d = S.shape[-1]
    return np.einsum("bgid,bgjd->bgij", qbar, S) / math.sqrt(d)


def select_topk(scores, cand, k: int) -> np.ndarray:
    """The ``min(k, len(cand))`` candidates of highest score.

    Order: higher score first; equal scores go to the lower block index.
    Returns the chosen block indices (unsorted order of rank).
    """
    scores = _f64(scores)
    cand = np.asarray(cand, dtype=np.int64)
    if k <= 0 or cand.size == 0:
        return np.empty(0, dtype=np.int64)
    order = np.lexsort((cand, -scores))  # primary key: -score, then index
    return cand[order[: min(k, cand.size)]]


def route(Q, S, B: int, topk: int, Hkv: int):
    """Per (batch, KV head, query block) block selection.

    Candidates for query block i are the complete blocks ``1 .. i-1``; the sink
    block 0 and the diagonal block i are always added and are not counted in
    ``topk``.  Returns ``(idx, cnt, scores)``: ``idx`` int64 ``[b, Hkv, nq, topk + 2]``
    ascending, padded with -1 (``topk`` clipped to ``nq`` for the width);
    ``cnt`` ``[b, Hkv, nq]``; ``scores`` ``[b, Hkv, nq, nfull]`` (all pairs, the
    non-candidates included, for near-tie accounting).
    """
    Q = _f64(Q)
    N = Q.shape[2]
    nq = -(-N // B)
    qbar = pool_query_blocks(Q, B, Hkv)
    sc = summary_scores(qbar, S)
    b = Q.shape[0]
    kk = min(topk, nq)
    width = kk + 2
    idx = np.full((b, Hkv, nq, width), -1, dtype=np.int64)
    cnt = np.zeros((b, Hkv, nq), dtype=np.int64)
    for bi in range(b):
        for g in range(Hkv):
            for i in range(nq):
                cand = np.arange(1, max(i, 1))  # 1 .. i-1
                chosen = select_topk(sc[bi, g, i, cand], cand, kk)
                sel = sorted({0, i} | set(int(c) for c in chosen))
                idx[bi, g, i, : len(sel)] = sel
                cnt[bi, g, i] = len(sel)
    return idx, cnt, sc


def _selected_keys(sel, B: int, N: int) -> np.ndarray:
    pos = [np.arange(j * B, min(N, (j + 1) * B)) for j in sel]
    return np.concatenate(pos) if pos else np.empty(0, dtype=np.int64)


def sparse_attention(Q, K, V, idx, cnt, B: int, scale: float | None = None,
                     units=None):
    """Exact softmax attention of each query row over its selected blocks.

    For query row t (block ``i = t // B``) of head h, the keys are the rows of
    the blocks ``idx[b, h // G, i, :cnt]`` with key position ``<= t``.  Returns
    ``(O, LSE)``: ``O`` ``[b, Hq, N, d]``, ``LSE`` ``[b, Hq, N]`` (natural log of
    the softmax denominator of the scaled logits).  ``units``, if given, is an
    iterable of ``(b, g, i)`` to compute; other rows are left as NaN.
    """
    Q = _f64(Q)
    K = _f64(K)
    V = _f64(V)
    b, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    nq = -(-N // B)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.full((b, Hq, N, d), np.nan)
    LSE = np.full((b, Hq, N), np.nan)
    if units is None:
        units = [(bi, g, i) for bi in range(b) for g in range(Hkv) for i in range(nq)]
    for bi, g, i in units:
        sel = [int(j) for j in idx[bi, g, i, : cnt[bi, g, i]]]
        kpos = _selected_keys(sel, B, N)
        t0, t1 = i * B, min(N, (i + 1) * B)
        qpos = np.arange(t0, t1)
        q = Q[bi, g * G : (g + 1) * G, t0:t1, :]  # [G, r, d]
        logits = np.einsum("hrd,kd->hrk", q, K[bi, g][kpos]) * scale
        mask = kpos[None, None, :] > qpos[None, :, None]
        logits = np.where(mask, -np.inf, logits)
        m = logits.max(axis=-1, keepdims=True)
        e = np.exp(logits - m)
        den = e.sum(axis=-1, keepdims=True)
        p = e / den
        O[bi, g * G : (g + 1) * G, t0:t1, :] = np.einsum("hrk,kd->hrd", p, V[bi, g][kpos])
        LSE[bi, g * G : (g + 1) * G, t0:t1] = (m + np.log(den))[..., 0]
    return O, LSE


def sparse_attention_backward(Q, K, V, idx, cnt, dO, B: int, scale: float | None = None):
    """Gradients of :func:`sparse_attention`'s ``O`` with the selection fixed.

    Given the upstream gradient ``dO`` ``[b, Hq, N, d]``, returns
    ``(dQ, dK, dV)`` with the shapes of Q, K and V.  Per unit (b, g, i), P is
    the unit's softmax over its selected, causally visible keys, and with
    ``O = P V``:

    * ``dV[keys] += P^T dO``;
    * ``dS = P * (dO V^T - rowsum(dO * O))``, the softmax Jacobian applied to
      ``dP = dO V^T``;
    * ``dQ = scale * dS K[keys]`` and ``dK[keys] += scale * dS^T Q``.

    dK and dV sum over the G query heads that share the KV head and over the
    query blocks that selected the key.  Keys that no unit selected, and
    positions after every query that sees them, get exactly 0.
    """
    Q = _f64(Q)
    K = _f64(K)
    V = _f64(V)
    dO = _f64(dO)
    b, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    nq = -(-N // B)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    for bi in range(b):
        for g in range(Hkv):
            for i in range(nq):
                sel = [int(j) for j in idx[bi, g, i, : cnt[bi, g, i]]]
                kpos = _selected_keys(sel, B, N)
                t0, t1 = i * B, min(N, (i + 1) * B)
                qpos = np.arange(t0, t1)
                q = Q[bi, g * G : (g + 1) * G, t0:t1, :]    # [G, r, d]
                do = dO[bi, g * G : (g + 1) * G, t0:t1, :]  # [G, r, d]
                k = K[bi, g][kpos]                          # [n, d]
                v = V[bi, g][kpos]
                logits = np.einsum("hrd,kd->hrk", q, k) * scale
                logits = np.where(kpos[None, None, :] > qpos[None, :, None], -np.inf, logits)
                e = np.exp(logits - logits.max(axis=-1, keepdims=True))
                p = e / e.sum(axis=-1, keepdims=True)       # [G, r, n]
                o = np.einsum("hrk,kd->hrd", p, v)
                dp = np.einsum("hrd,kd->hrk", do, v)
                ds = p * (dp - np.einsum("hrd,hrd->hr", do, o)[..., None])
                dQ[bi, g * G : (g + 1) * G, t0:t1, :] = scale * np.einsum("hrk,kd->hrd", ds, k)
                dK[bi, g, kpos] += scale * np.einsum("hrk,hrd->kd", ds, q)
                dV[bi, g, kpos] += np.einsum("hrk,hrd->kd", p, do)
    return dQ, dK, dV


def attention_probs(Q, K, idx, cnt, B: int, scale: float | None = None) -> np.ndarray:
    """The full attention matrix ``P`` ``[b, Hq, N, N]`` of the block-sparse path.

    ``P[b, h, t, s]`` is the softmax weight of key s for query t; keys outside
    the selected blocks or after t get exactly 0.  Small inputs only.
    """
    Q = _f64(Q)
    K = _f64(K)
    b, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    nq = -(-N // B)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    P = np.zeros((b, Hq, N, N))
    for bi in range(b):
        for h in range(Hq):
            g = h // G
            for i in range(nq):
                sel = [int(j) for j in idx[bi, g, i, : cnt[bi, g, i]]]
                kpos = _selected_keys(sel, B, N)
                for t in range(i * B, min(N, (i + 1) * B)):
                    ks = kpos[kpos <= t]
                    z = (K[bi, g][ks] @ Q[bi, h, t]) * scale
                    w = np.exp(z - z.max())
                    P[bi, h, t, ks] = w / w.sum()
    return P


def decode_route(q, S, seqlens, B: int, topk: int):
    """Block selection for one query token per sequence.

    The cache of sequence b holds ``L = seqlens[b]`` tokens, the current one
    included, so the query sits at position ``L - 1`` and its diagonal block
    is ``last = (L - 1) // B`` (possibly partial).  Candidates are the complete
    blocks ``1 .. last-1``, scored by the group-mean query against their
    summaries; sink 0 and ``last`` are always added.
    q: ``[b, Hq, d]``; S: ``[b, Hkv, nblk, d]``.  Returns ``(idx, cnt, scores)``
    with ``idx`` ``[b, Hkv, topk + 2]`` ascending, -1 padded.
    """
    q = _f64(q)
    S = _f64(S)
    b, Hq, d = q.shape
    Hkv = S.shape[1]
    G = Hq // Hkv
    qbar = q.reshape(b, Hkv, G, d).mean(axis=2)
    sc = np.einsum("bgd,bgjd->bgj", qbar, S) / math.sqrt(d)
    width = topk + 2
    idx = np.full((b, Hkv, width), -1, dtype=np.int64)
    cnt = np.zeros((b, Hkv), dtype=np.int64)
    for bi in range(b):
        last = (int(seqlens[bi]) - 1) // B
        for g in range(Hkv):
            cand = np.arange(1, max(last, 1))
            chosen = select_topk(sc[bi, g, cand], cand, topk)
            sel = sorted({0, last} | set(int(c) for c in chosen))
            idx[bi, g, : len(sel)] = sel
            cnt[bi, g] = len(sel)
    return idx, cnt, sc


def decode(q, Kc, Vc, seqlens, B: int, topk: int, scale: float | None = None,
           S=None, idx=None, cnt=None, batches=None):
    """One decode step: route over block summaries, then attend the selected blocks.

    ``S`` defaults to the fp64 mean of the cache's complete blocks.  ``idx`` /
    ``cnt`` may be given to attend a fixed selection.  Returns
    ``(O, LSE, idx, cnt)`` with ``O`` ``[b, Hq, d]``.  ``batches`` restricts the
    attention to some sequences (others NaN); routing still covers all.
    """
    q = _f64(q)
    b, Hq, d = q.shape
    Hkv = Kc.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if idx is None:
        if S is None:
            S = np.stack([block_summary(_f64(Kc[bi : bi + 1]), B)[0] for bi in range(b)])
        idx, cnt, _ = decode_route(q, S, seqlens, B, topk)
    O = np.full((b, Hq, d), np.nan)
    LSE = np.full((b, Hq), np.nan)
    for bi in (range(b) if batches is None else batches):
        L = int(seqlens[bi])
        Kb = _f64(Kc[bi])
        Vb = _f64(Vc[bi])
        for g in range(Hkv):
            sel = [int(j) for j in idx[bi, g, : cnt[bi, g]]]
            kpos = _selected_keys(sel, B, L)  # keys at positions < L only
            z = np.einsum("hd,kd->hk", q[bi, g * G : (g + 1) * G], Kb[g][kpos]) * scale
            m = z.max(axis=-1, keepdims=True)
            e = np.exp(z - m)
            den = e.sum(axis=-1, keepdims=True)
            O[bi, g * G : (g + 1) * G] = (e / den) @ Vb[g][kpos]
            LSE[bi, g * G : (g + 1) * G] = (m + np.log(den))[:, 0]
    return O, LSE, idx, cnt


def decode_append(Kc, Vc, S, seqlens, k_new, v_new, B: int):
    """Append one token per sequence to a KV cache and keep its summaries current.

    ``Kc``, ``Vc``: ``[b, Hkv, Lmax, d]``; ``S``: ``[b, Hkv, Lmax // B, d]``;
    ``seqlens``: ``[b]`` tokens held; ``k_new``, ``v_new``: ``[b, Hkv, d]``.
    For a sequence holding L tokens, 0 <= L < Lmax, the new row goes to
    position L and the sequence then holds L + 1 tokens; when L + 1 is a
    multiple of B, block (L + 1) / B - 1 has just become complete and its
    summary is the mean of its B keys (the stage-0 summary, formed once a
    block is complete: DashAttention page, "Estágio 0" and "Contribuições
    Principais" 4).  A sequence with L outside [0, Lmax) is left unchanged.
    Returns new ``(Kc, Vc, S, seqlens)`` (float64 copies, seqlens int64).
    """
    Kc = _f64(Kc).copy()
    Vc = _f64(Vc).copy()
    S = _f64(S).copy()
    seqlens = np.asarray(seqlens, dtype=np.int64).copy()
    k_new = _f64(k_new)
    v_new = _f64(v_new)
    Lmax = Kc.shape[2]
    for bi in range(Kc.shape[0]):
        L = int(seqlens[bi])
        if not 0 <= L < Lmax:
            continue
        Kc[bi, :, L] = k_new[bi]
        Vc[bi, :, L] = v_new[bi]
        seqlens[bi] = L + 1
        if (L + 1) % B == 0:
            j = (L + 1) // B - 1
            S[bi, :, j] = Kc[bi, :, j * B : (j + 1) * B].mean(axis=1)
    return Kc, Vc, S, seqlens
