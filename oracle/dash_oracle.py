"""Plain fp64 CPU oracle of DashAttention's adaptive form of the path.

TEST INFRASTRUCTURE ONLY, like the rest of this package: nothing on the
product path may import it.

The DashAttention page ("Metodologia") replaces each stage of the top-k path:

* stage 0, learned block summary: a learned query q̄ attends, by scaled
  dot-product attention, over the keys of each block; at q̄ = 0 this is the
  uniform mean of the keys ("Estágio 0": initialised at zero it behaves as
  mean pooling);
* stage 1, α-entmax routing: the logits of a query against the block
  summaries, scaled by γ, are mapped by α-entmax, whose support size follows
  from the scores instead of a fixed k; the query heads that share a KV head
  average their probabilities into one shared sparse support ("Estágio 1",
  ŵ = α-entmax(γ z̄) and the GQA handling);
* stage 2, prior-induced softmax: softmax is the maximiser of zᵀp − KL(p‖u)
  over the simplex; with the uniform u replaced by a prior g built from the
  routing probabilities, the maximiser is p ∝ g·exp(z), so log g is added to
  the logits and g = 0 masks a key; the diagonal block keeps a separate
  branch, and σ sets how strongly the prior follows the routing scores
  against a uniform baseline ("Estágio 2").

α-entmax itself (the page names it without a formula) is the standard map
p_i = [(α − 1) z_i − τ]_+^{1/(α−1)}, with the threshold τ fixed by Σ p = 1;
for α = 2 it is sparsemax.  τ is found by bisection.

Readings where the page leaves a step open:

* the summary attention's values are the block's keys (the summary is
  compared with queries, and q̄ = 0 must give the mean key);
* routing is per (query block, query head), with the head's query pooled over
  the block's rows, as in the top-k path; logits are q̄·S_j/√d;
* candidates are the complete blocks before the query block (0 .. i−1); the
  diagonal block i is the separate branch and is always attended, causally;
* the prior is g_j ∝ w_j^σ on the routing support: σ = 0 is uniform over the
  support, σ = 1 follows the routing probabilities; a key of routed block j
  gets the bias σ·log w_j, a diagonal key gets 0, every other key −inf.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = ["entmax", "learned_block_summary", "entmax_route", "prior_sparse_attention"]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def entmax(z, alpha: float, n_iter: int = 200) -> np.ndarray:
    """α-entmax of the last axis of ``z`` (α > 1), by bisection on τ.

    ``p = [(α−1) z − τ]_+ ** (1/(α−1))`` with ``Σ p = 1``.  ``-inf`` entries
    get 0.  With m the largest ``(α−1) z``, τ lies in ``[m − 1, m]``: at
    ``m − 1`` the largest term alone is 1, at ``m`` every term is 0.
    """
    if not alpha > 1.0:
        raise ValueError("alpha must be > 1")
    z = _f64(z)
    x = (alpha - 1.0) * z
    m = x.max(axis=-1, keepdims=True)
    lo, hi = m - 1.0, m
    inv = 1.0 / (alpha - 1.0)

    def mass(t):
        return (np.clip(x - t, 0.0, None) ** inv).sum(axis=-1, keepdims=True)

    for _ in range(n_iter):
        mid = 0.5 * (lo + hi)
        big = mass(mid) >= 1.0
        lo = np.where(big, mid, lo)
        hi = np.where(big, hi, mid)
    p = np.clip(x - lo, 0.0, None) ** inv
    return p / p.sum(axis=-1, keepdims=True)


def learned_block_summary(K, B: int, qbar, scale: float | None = None) -> np.ndarray:
    """Stage 0 with a learned summary query.

    ``S[b, g, j] = Σ_t softmax_t(scale · q̄_g · k_t) k_t`` over the B keys of each
    complete block j.  ``qbar``: ``[Hkv, d]`` (one learned query per KV head)
    or ``[d]`` (shared).  Returns ``[b, Hkv, N // B, d]``.
    """
    K = _f64(K)
    b, Hkv, N, d = K.shape
    nf = N // B
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    qb = np.broadcast_to(_f64(qbar), (Hkv, d))
    S = np.zeros((b, Hkv, nf, d))
    for bi in range(b):
        for g in range(Hkv):
            for j in range(nf):
                k = K[bi, g, j * B : (j + 1) * B]
                z = (k @ qb[g]) * scale
                e = np.exp(z - z.max())
                S[bi, g, j] = (e / e.sum()) @ k
    return S


def entmax_route(Q, S, B: int, Hkv: int, alpha: float, gamma: float,
                 scale: float | None = None) -> np.ndarray:
    """Stage 1: routing probabilities ``w`` ``[b, Hkv, nq, nfull]``.

    For query block i and query head h of group g: ``q̄_h`` is the mean of
    head h's rows in the block, ``z_j = scale · q̄_h · S[b, g, j]`` for the
    candidates ``j < min(i, nfull)``, and ``p_h = α-entmax(γ z)``.  ``w`` is the
    mean of ``p_h`` over the group's heads; it is 0 off the candidates, and a
    block with no candidates (i = 0) has an all-zero row.
    """
    Q = _f64(Q)
    S = _f64(S)
    b, Hq, N, d = Q.shape
    G = Hq // Hkv
    nq = -(-N // B)
    nf = S.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    w = np.zeros((b, Hkv, nq, nf))
    for bi in range(b):
        for g in range(Hkv):
            for i in range(nq):
                nc = min(i, nf)
                if nc == 0:
                    continue
                acc = np.zeros(nc)
                for h in range(g * G, (g + 1) * G):
                    qb = Q[bi, h, i * B : min(N, (i + 1) * B)].mean(axis=0)
                    z = (S[bi, g, :nc] @ qb) * scale
                    acc += entmax(gamma * z, alpha)
                w[bi, g, i, :nc] = acc / G
    return w


def prior_sparse_attention(Q, K, V, w, B: int, sigma: float, scale: float | None = None):
    """Stage 2: attention with the prior-induced softmax.

    Query row t (block i) of head h in group g attends key s with logit
    ``scale · q_t · k_s + bias``: ``bias = σ · log w[b, g, i, s // B]`` when
    that routing probability is positive, 0 on the diagonal block (keys
    ``s <= t``), and the key is masked otherwise.  Returns ``(O, LSE)`` like
    the top-k attention.
    """
    Q = _f64(Q)
    K = _f64(K)
    V = _f64(V)
    w = _f64(w)
    b, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    nq = -(-N // B)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.zeros((b, Hq, N, d))
    LSE = np.zeros((b, Hq, N))
    for bi in range(b):
        for g in range(Hkv):
            for i in range(nq):
                t0, t1 = i * B, min(N, (i + 1) * B)
                routed = [j for j in range(w.shape[3]) if j < i and w[bi, g, i, j] > 0.0]
                kpos = [np.arange(j * B, (j + 1) * B) for j in routed] + [np.arange(t0, t1)]
                kpos = np.concatenate(kpos)
                bias = np.concatenate(
                    [np.full(B, sigma * math.log(w[bi, g, i, j])) for j in routed]
                    + [np.zeros(t1 - t0)])
                qpos = np.arange(t0, t1)
                q = Q[bi, g * G : (g + 1) * G, t0:t1, :]
                logits = np.einsum("hrd,kd->hrk", q, K[bi, g][kpos]) * scale + bias
                logits = np.where(kpos[None, None, :] > qpos[None, :, None], -np.inf, logits)
                m = logits.max(axis=-1, keepdims=True)
                e = np.exp(logits - m)
                den = e.sum(axis=-1, keepdims=True)
                O[bi, g * G : (g + 1) * G, t0:t1] = np.einsum("hrk,kd->hrd", e / den,
                                                              V[bi, g][kpos])
                LSE[bi, g * G : (g + 1) * G, t0:t1] = (m + np.log(den))[..., 0]
    return O, LSE
