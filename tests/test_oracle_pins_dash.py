"""Pins for the oracle of DashAttention's adaptive stages (learned summary,
α-entmax routing, prior-induced softmax), each against something other than
the oracle's own formulas: closed forms of α-entmax at α = 2 and α = 1.5,
torch's scaled_dot_product_attention, and the pinned top-k attention.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O


# ------------------------------------------------------------------ α-entmax
def _sparsemax_sorted(z):
    # Euclidean projection onto the simplex: with z sorted descending, the
    # support is the largest k with 1 + k z_(k) > sum_{j<=k} z_(j)
    zs = np.sort(z)[::-1]
    cs = np.cumsum(zs)
    k = np.arange(1, z.size + 1)
    kk = k[1 + k * zs > cs][-1]
    tau = (cs[kk - 1] - 1.0) / kk
    return np.maximum(z - tau, 0.0)


def _entmax15_sorted(z):
    # α = 1.5: p = (z/2 - τ)_+^2.  On a support of the k largest u = z/2,
    # sum (u - τ)^2 = 1 gives τ_k = mean_k - sqrt(1/k - var_k); the support is
    # the largest k whose k-th value still exceeds τ_k.
    u = np.sort(z / 2.0)[::-1]
    best = None
    for k in range(1, u.size + 1):
        mean = u[:k].mean()
        var = (u[:k] ** 2).mean() - mean ** 2
        rad = 1.0 / k - var
        if rad < 0:
            break
        tau = mean - math.sqrt(rad)
        if u[k - 1] > tau:
            best = tau
    return np.maximum(z / 2.0 - best, 0.0) ** 2


@pytest.mark.parametrize("seed", range(6))
def test_entmax_alpha2_is_sparsemax(seed):
    rng = np.random.default_rng(seed)
    z = rng.standard_normal(17) * (0.3 + seed)
    np.testing.assert_allclose(O.entmax(z, 2.0), _sparsemax_sorted(z), rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", range(6))
def test_entmax_alpha15_matches_sort_based_closed_form(seed):
    rng = np.random.default_rng(100 + seed)
    z = rng.standard_normal(23) * (0.5 + seed)
    np.testing.assert_allclose(O.entmax(z, 1.5), _entmax15_sorted(z), rtol=0, atol=1e-12)


def test_entmax_simplex_threshold_and_invariances():
    rng = np.random.default_rng(7)
    z = rng.standard_normal((5, 31)) * 2.0
    for alpha in (1.25, 1.5, 2.0, 3.0):
        p = O.entmax(z, alpha)
        assert np.all(p >= 0.0)
        np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-12)
        # order preserved, and support = the entries above one threshold
        for r in range(z.shape[0]):
            o = np.argsort(-z[r])
            assert np.all(np.diff(p[r, o]) <= 1e-15)
            on = p[r] > 0
            assert z[r, on].min() > z[r, ~on].max() if (~on).any() else True
        np.testing.assert_allclose(O.entmax(z + 3.7, alpha), p, rtol=0, atol=1e-12)
        perm = rng.permutation(z.shape[1])
        np.testing.assert_allclose(O.entmax(z[:, perm], alpha), p[:, perm], rtol=0, atol=1e-12)
    # a sharper input gives a smaller support (α = 2)
    s1 = (O.entmax(z, 2.0) > 0).sum(-1)
    s4 = (O.entmax(4.0 * z, 2.0) > 0).sum(-1)
    assert np.all(s4 <= s1) and np.any(s4 < s1)


def test_entmax_masked_entries_get_zero():
    z = np.array([0.3, -np.inf, 1.2, -np.inf, 0.9])
    p = O.entmax(z, 1.5)
    assert p[1] == 0.0 and p[3] == 0.0
    np.testing.assert_allclose(p[[0, 2, 4]], _entmax15_sorted(z[[0, 2, 4]]), rtol=0, atol=1e-12)


# ------------------------------------------------------ stage 0: learned summary
def test_learned_summary_zero_query_is_the_block_mean():
    rng = np.random.default_rng(8)
    K = rng.standard_normal((2, 3, 8 * 5 + 3, 16))
    S0 = O.learned_block_summary(K, 8, np.zeros((3, 16)))
    np.testing.assert_allclose(S0, O.block_summary(K, 8), rtol=0, atol=1e-12)


def test_learned_summary_equals_sdpa_over_the_block():
    rng = np.random.default_rng(9)
    b, Hkv, B, nb, d = 1, 2, 16, 4, 32
    K = rng.standard_normal((b, Hkv, B * nb, d))
    qbar = rng.standard_normal((Hkv, d)) * 3.0
    S = O.learned_block_summary(K, B, qbar)
    for g in range(Hkv):
        for j in range(nb):
            k = torch.from_numpy(K[0, g, j * B : (j + 1) * B])[None, None]
            q = torch.from_numpy(qbar[g])[None, None, None]
            ref = torch.nn.functional.scaled_dot_product_attention(q, k, k)[0, 0, 0].numpy()
            np.testing.assert_allclose(S[0, g, j], ref, rtol=0, atol=1e-12)


def test_learned_summary_sharp_query_picks_its_key():
    rng = np.random.default_rng(10)
    K = rng.standard_normal((1, 1, 16, 8))
    K[0, 0, 5] *= 4.0
    S = O.learned_block_summary(K, 16, K[0, 0, 5] * 50.0)
    np.testing.assert_allclose(S[0, 0, 0], K[0, 0, 5], rtol=0, atol=1e-9)


# ------------------------------------------------------- stage 1: entmax routing
def _route_case(seed, Hq=4, Hkv=2, N=8 * 9 + 5, d=16, B=8):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((1, Hq, N, d))
    K = rng.standard_normal((1, Hkv, N, d))
    return Q, K, O.block_summary(K, B), B, Hkv


def test_entmax_route_rows_are_distributions_on_the_candidates():
    Q, K, S, B, Hkv = _route_case(11)
    w = O.entmax_route(Q, S, B, Hkv, alpha=1.5, gamma=4.0)
    nq, nf = w.shape[2], w.shape[3]
    assert np.all(w[:, :, 0] == 0.0)
    for i in range(1, nq):
        np.testing.assert_allclose(w[0, :, i].sum(-1), 1.0, rtol=0, atol=1e-12)
        assert np.all(w[0, :, i, min(i, nf):] == 0.0)


def test_entmax_route_is_the_group_mean_of_per_head_entmax():
    # recompute one (group, block) by hand: per-head pooled query, logits,
    # α = 2 sparsemax by the sort-based closed form, mean over the heads
    Q, K, S, B, Hkv = _route_case(12)
    gamma, g, i = 3.0, 1, 7
    G = Q.shape[1] // Hkv
    w = O.entmax_route(Q, S, B, Hkv, alpha=2.0, gamma=gamma)
    d = Q.shape[-1]
    ref = np.zeros(i)
    for h in range(g * G, (g + 1) * G):
        qb = Q[0, h, i * B : (i + 1) * B].mean(0)
        ref += _sparsemax_sorted(gamma * (S[0, g, :i] @ qb) / math.sqrt(d))
    np.testing.assert_allclose(w[0, g, i, :i], ref / G, rtol=0, atol=1e-12)


def test_entmax_route_one_dominant_block_takes_all():
    Q, K, S, B, Hkv = _route_case(13, Hq=2, Hkv=2)
    S = S.copy()
    i, j = 6, 2
    S[0, 0, j] = Q[0, 0, i * B : (i + 1) * B].mean(0) * 40.0
    w = O.entmax_route(Q, S, B, Hkv, alpha=2.0, gamma=1.0)
    assert w[0, 0, i, j] == 1.0 and np.count_nonzero(w[0, 0, i]) == 1


# ----------------------------------------------- stage 2: prior-induced softmax
def test_prior_attention_without_prior_is_topk_attention_on_the_support():
    Q, K, S, B, Hkv = _route_case(14)
    V = np.random.default_rng(15).standard_normal(K.shape)
    w = O.entmax_route(Q, S, B, Hkv, alpha=1.5, gamma=6.0)
    out, lse = O.prior_sparse_attention(Q, K, V, w, B, sigma=0.0)
    nq = w.shape[2]
    width = nq + 1
    idx = np.full((1, Hkv, nq, width), -1)
    cnt = np.zeros((1, Hkv, nq), dtype=np.int64)
    for g in range(Hkv):
        for i in range(nq):
            sel = sorted([j for j in range(w.shape[3]) if w[0, g, i, j] > 0] + [i])
            idx[0, g, i, : len(sel)] = sel
            cnt[0, g, i] = len(sel)
    ref, rlse = O.sparse_attention(Q, K, V, idx, cnt, B)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rlse, rtol=0, atol=1e-12)


def test_prior_attention_equals_sdpa_with_the_log_prior_as_additive_mask():
    Q, K, S, B, Hkv = _route_case(16)
    V = np.random.default_rng(17).standard_normal(K.shape)
    sigma = 0.7
    w = O.entmax_route(Q, S, B, Hkv, alpha=1.5, gamma=6.0)
    out, _ = O.prior_sparse_attention(Q, K, V, w, B, sigma=sigma)
    N = Q.shape[2]
    G = Q.shape[1] // Hkv
    mask = np.full((1, Q.shape[1], N, N), -np.inf)
    for h in range(Q.shape[1]):
        g = h // G
        for t in range(N):
            i = t // B
            for s in range(t + 1):
                j = s // B
                if j == i:
                    mask[0, h, t, s] = 0.0
                elif j < w.shape[3] and w[0, g, i, j] > 0:
                    mask[0, h, t, s] = sigma * math.log(w[0, g, i, j])
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q), torch.from_numpy(np.repeat(K, G, 1)),
        torch.from_numpy(np.repeat(V, G, 1)), attn_mask=torch.from_numpy(mask)).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
