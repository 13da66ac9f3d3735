"""Plain fp64 CPU oracle of two routing variants: per-head decode routing and
two-level (hierarchical) routing.

TEST INFRASTRUCTURE ONLY, like the rest of this package: nothing on the
product path may import it.

* Per-head decode routing.  In decode a single query token is routed per
  step, so fine selection is cheap, and a method that keeps the whole KV cache
  but loads only the pages the query selects generalises best (The Sparse
  Frontier page, RQ2, decode flexibility and Quest's token-to-page selection).
  The page gives no scoring rule beyond that, so the reading here keeps the
  block summaries of the main path and drops only the GQA pooling: every
  query head scores the summaries with its own query and keeps its own top-k,
  plus the sink block 0 and the last (diagonal) block.
* Two-level routing (GSA page, "Componentes Principais" 4, H-GSA: meta-level
  summaries of groups of block summaries; select the best segments first,
  then the best blocks inside them, then attend their raw tokens).  A segment
  is M consecutive complete blocks; its meta-summary is the mean of their
  summaries, which is the mean of all the segment's keys.

Readings where the pages leave a step open (two-level routing):

* a segment takes part in the meta-level choice only when all its blocks lie
  before the query block; the candidate blocks of the other segments (the
  recent ones, next to the diagonal) go straight to the block level, as the
  diagonal block goes straight to attention in the flat path;
* the meta level keeps the top k_seg segments by q̄·Ŝ_m/√d among those that
  hold at least one candidate block; the block level keeps the top k_blk of
  the candidate blocks inside the kept and the recent segments, by the same
  score as the flat path; ties go to the lower index at both levels; the sink
  block 0 and the diagonal block are added as in the flat path.
"""
from __future__ import annotations

import math

import numpy as np

from .ssa_oracle import pool_query_blocks, select_topk, summary_scores

__all__ = ["decode_route_per_head", "decode_per_head", "segment_summaries",
           "hierarchical_route"]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def decode_route_per_head(q, S, seqlens, B: int, topk: int):
    """Per query head: the decode selection of each head on its own query.

    Same candidates and forced blocks as the grouped decode routing (complete
    blocks ``1 .. last-1``; sink 0 and ``last = (L-1) // B``), scored by
    ``q_h · S[b, h // G, j] / sqrt(d)``.  Returns ``(idx, cnt)``: ``idx``
    ``[b, Hq, topk + 2]`` ascending, -1 padded; sequences with an invalid
    length get ``cnt = 0``.
    """
    q = _f64(q)
    S = _f64(S)
    b, Hq, d = q.shape
    Hkv = S.shape[1]
    G = Hq // Hkv
    width = topk + 2
    idx = np.full((b, Hq, width), -1, dtype=np.int64)
    cnt = np.zeros((b, Hq), dtype=np.int64)
    for bi in range(b):
        L = int(seqlens[bi])
        if L <= 0:
            continue
        last = (L - 1) // B
        cand = np.arange(1, max(last, 1))
        for h in range(Hq):
            sc = (S[bi, h // G, cand] @ q[bi, h]) / math.sqrt(d) if cand.size else np.empty(0)
            sel = sorted(set([0, last]) | set(select_topk(sc, cand, topk).tolist()))
            idx[bi, h, : len(sel)] = sel
            cnt[bi, h] = len(sel)
    return idx, cnt


def decode_per_head(q, Kc, Vc, seqlens, idx, cnt, B: int, scale: float | None = None):
    """Decode attention with a block list per query head.

    Head h of sequence b attends the keys of blocks ``idx[b, h, :cnt]`` at
    positions ``< L``.  Returns ``O`` ``[b, Hq, d]`` (zeros where ``cnt = 0``).
    """
    q = _f64(q)
    Kc = _f64(Kc)
    Vc = _f64(Vc)
    b, Hq, d = q.shape
    G = Hq // Kc.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.zeros((b, Hq, d))
    for bi in range(b):
        L = int(seqlens[bi])
        for h in range(Hq):
            if cnt[bi, h] == 0:
                continue
            pos = np.concatenate([np.arange(j * B, min(L, (j + 1) * B))
                                  for j in idx[bi, h, : cnt[bi, h]]])
            k = Kc[bi, h // G][pos]
            z = (k @ q[bi, h]) * scale
            e = np.exp(z - z.max())
            O[bi, h] = (e / e.sum()) @ Vc[bi, h // G][pos]
    return O


def segment_summaries(S, M: int) -> np.ndarray:
    """Meta-summaries: the mean of each run of M consecutive block summaries
    (complete runs only).  ``S`` ``[b, Hkv, nfull, d]`` → ``[b, Hkv, nfull // M, d]``."""
    S = _f64(S)
    b, Hkv, nf, d = S.shape
    ns = nf // M
    return S[:, :, : ns * M].reshape(b, Hkv, ns, M, d).mean(axis=3)


def hierarchical_route(Q, S, B: int, M: int, k_seg: int, k_blk: int, Hkv: int):
    """Two-level block selection per (batch, KV head, query block).

    Returns ``(idx, cnt)`` with ``idx`` ``[b, Hkv, nq, k_blk + 2]`` ascending,
    -1 padded (the layout of the flat routing).
    """
    Q = _f64(Q)
    S = _f64(S)
    N = Q.shape[2]
    nq = -(-N // B)
    qbar = pool_query_blocks(Q, B, Hkv)
    sc_blk = summary_scores(qbar, S)                       # [b, Hkv, nq, nfull]
    Sm = segment_summaries(S, M)
    sc_seg = summary_scores(qbar, Sm) if Sm.shape[2] else None
    b = Q.shape[0]
    width = min(k_blk, nq) + 2
    idx = np.full((b, Hkv, nq, width), -1, dtype=np.int64)
    cnt = np.zeros((b, Hkv, nq), dtype=np.int64)
    for bi in range(b):
        for g in range(Hkv):
            for i in range(nq):
                cand = np.arange(1, max(i, 1))              # complete blocks 1 .. i-1
                closed = [m for m in range(Sm.shape[2]) if (m + 1) * M <= i]
                eligible = [m for m in closed if np.any((cand >= m * M) & (cand < (m + 1) * M))]
                kept = set()
                if eligible:
                    e = np.asarray(eligible)
                    kept = set(select_topk(sc_seg[bi, g, i, e], e, k_seg).tolist())
                in_closed = np.zeros(cand.shape, dtype=bool)
                in_kept = np.zeros(cand.shape, dtype=bool)
                for m in closed:
                    inside = (cand >= m * M) & (cand < (m + 1) * M)
                    in_closed |= inside
                    if m in kept:
                        in_kept |= inside
                pool = cand[in_kept | ~in_closed]
                R = select_topk(sc_blk[bi, g, i, pool], pool, k_blk) if pool.size else []
                sel = sorted({0, i} | set(np.asarray(R).tolist()))
                idx[bi, g, i, : len(sel)] = sel
                cnt[bi, g, i] = len(sel)
    return idx, cnt
