"""Plain fp64 CPU oracle of decoding over a paged KV cache.

TEST INFRASTRUCTURE ONLY, like the rest of this package: nothing on the
product path may import it.

Decode keeps the whole cache and loads only the blocks a query selects (The
Sparse Frontier page, RQ2: Quest retains the full KV cache and loads pages
selectively), and incremental decoding appends tokens and forms a block's
summary once the block is complete (DashAttention page, "Contribuições
Principais" 4 and "Estágio 0").  Here the cache lives in pages instead of one
contiguous array per sequence.

Layout (a reading; the pages fix none): a page holds one block of B tokens for
every KV head of one sequence, so the page pool is ``[num_pages, Hkv, B, d]``;
``page_table[b, j]`` is the page of logical block j of sequence b (-1 where
none is mapped).  Block summaries stay per sequence in logical order,
``[batch, Hkv, max_blocks, d]``.  Every function is the contiguous one applied
to the cache the page table describes.
"""
from __future__ import annotations

import numpy as np

from .ssa_oracle import decode

__all__ = ["gather_pages", "decode_paged", "decode_append_paged"]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def gather_pages(P, page_table) -> np.ndarray:
    """The contiguous cache ``[batch, Hkv, max_blocks * B, d]`` a page table
    describes; unmapped blocks read as zeros."""
    P = _f64(P)
    pt = np.asarray(page_table)
    _, Hkv, B, d = P.shape
    b, nb = pt.shape
    out = np.zeros((b, Hkv, nb * B, d))
    for bi in range(b):
        for j in range(nb):
            if pt[bi, j] >= 0:
                out[bi, :, j * B : (j + 1) * B] = P[pt[bi, j]]
    return out


def decode_paged(q, Kp, Vp, page_table, seqlens, B: int, topk: int, S=None,
                 scale: float | None = None):
    """One decode step over a paged cache: ``(O, LSE, idx, cnt)`` as ``decode``
    returns them for the gathered cache."""
    return decode(q, gather_pages(Kp, page_table), gather_pages(Vp, page_table), seqlens, B,
                  topk, scale=scale, S=S)


def decode_append_paged(Kp, Vp, S, page_table, seqlens, k_new, v_new, B: int):
    """Append one token per sequence to a paged cache and keep its summaries current.

    For a sequence holding L tokens, the new rows go to row ``L % B`` of page
    ``page_table[b, L // B]``; when L + 1 is a multiple of B, the summary of
    block ``L // B`` becomes the mean of that page's B keys.  A sequence whose
    next block has no page (or L < 0) is left unchanged.  Returns new
    ``(Kp, Vp, S, seqlens)`` (float64 copies, seqlens int64).
    """
    Kp = _f64(Kp).copy()
    Vp = _f64(Vp).copy()
    S = _f64(S).copy()
    seqlens = np.asarray(seqlens, dtype=np.int64).copy()
    pt = np.asarray(page_table)
    k_new = _f64(k_new)
    v_new = _f64(v_new)
    for bi in range(pt.shape[0]):
        L = int(seqlens[bi])
        if L < 0 or L // B >= pt.shape[1] or pt[bi, L // B] < 0:
            continue
        page = pt[bi, L // B]
        Kp[page, :, L % B] = k_new[bi]
        Vp[page, :, L % B] = v_new[bi]
        seqlens[bi] = L + 1
        if (L + 1) % B == 0:
            S[bi, :, L // B] = Kp[page].mean(axis=1)
    return Kp, Vp, S, seqlens
