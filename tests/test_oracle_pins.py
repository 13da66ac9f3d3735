"""Pins for the fp64 oracle: closed forms, brute force and library special cases.

Each test checks the oracle against something other than its own formulas, so
that a dropped term, a wrong index, a wrong head grouping or a transposed
operand fails at least one of them.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle as O
from workloads import planted_decode, planted_prefill, to_f64

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ---------------------------------------------------------------- stage 0: summary
def test_summary_constant_blocks_exact():
    rng = np.random.default_rng(1)
    b, h, B, nb, d = 2, 3, 8, 5, 4
    c = rng.integers(-50, 50, size=(b, h, nb, d)).astype(np.float64)
    K = np.repeat(c, B, axis=2)  # row t of block j carries c[..., j, :]
    S = O.block_summary(K, B)
    assert S.shape == (b, h, nb, d)
    assert np.array_equal(S, c)


def test_summary_arithmetic_progression_closed_form():
    # K[t] = a + r * t  =>  mean over block j = a + r * (j*B + (B-1)/2)
    B, nb, d = 16, 6, 3
    t = np.arange(nb * B, dtype=np.float64)
    a = np.array([0.5, -2.0, 3.25])
    r = np.array([1.0, 0.25, -0.5])
    K = (a[None, :] + t[:, None] * r[None, :])[None, None]
    S = O.block_summary(K, B)[0, 0]
    for j in range(nb):
        np.testing.assert_allclose(S[j], a + r * (j * B + (B - 1) / 2), rtol=0, atol=1e-12)


def test_summary_partial_tail_has_no_summary():
    K = np.ones((1, 1, 3 * 8 + 5, 2))
    assert O.block_summary(K, 8).shape == (1, 1, 3, 2)


# ---------------------------------------------------------------- stage 1: routing
def test_pool_gqa_grouping_closed_form():
    # Hq=4, Hkv=2: heads {0,1} -> KV head 0, {2,3} -> KV head 1.
    B, N, d = 4, 10, 2  # ragged: blocks of 4, 4, 2 rows
    Q = np.zeros((1, 4, N, d))
    for h in range(4):
        Q[0, h, :, 0] = h + 1
        Q[0, h, :, 1] = np.arange(N)  # row index
    qb = O.pool_query_blocks(Q, B, 2)
    assert qb.shape == (1, 2, 3, d)
    np.testing.assert_array_equal(qb[0, :, :, 0], [[1.5] * 3, [3.5] * 3])
    # row means per block: (0..3)->1.5, (4..7)->5.5, (8,9)->8.5 (partial block)
    np.testing.assert_array_equal(qb[0, 0, :, 1], [1.5, 5.5, 8.5])


def test_scores_equal_mean_of_per_row_per_head_dots():
    # The workload statement scores a (query block, KV head) pair as the mean over
    # the block's rows and the group's heads of q . kbar / sqrt(d); the oracle
    # pools first.  Recompute the pages' form row by row.
    rng = np.random.default_rng(2)
    b, Hq, Hkv, N, d, B = 1, 6, 2, 40, 5, 8
    Q = rng.standard_normal((b, Hq, N, d))
    K = rng.standard_normal((b, Hkv, N, d))
    S = O.block_summary(K, B)
    sc = O.summary_scores(O.pool_query_blocks(Q, B, Hkv), S)
    G = Hq // Hkv
    for g in range(Hkv):
        for i in range(N // B):
            for j in range(N // B):
                vals = [float(Q[0, h, t] @ S[0, g, j]) / math.sqrt(d)
                        for h in range(g * G, (g + 1) * G) for t in range(i * B, (i + 1) * B)]
                assert abs(sc[0, g, i, j] - sum(vals) / len(vals)) < 1e-12


def _brute_topk(scores, cand, k):
    """All subsets of size min(k, n): the max-sum ones, then the lexicographically
    smallest sorted index tuple (exact for integer scores)."""
    n = len(cand)
    m = min(k, n)
    best = None
    for sub in itertools.combinations(range(n), m):
        s = sum(scores[p] for p in sub)
        key = (-s, tuple(sorted(cand[p] for p in sub)))
        if best is None or key < best:
            best = key
    return sorted(best[1]) if best else []


@pytest.mark.parametrize("seed", range(40))
def test_select_topk_matches_brute_force_with_ties(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(0, 9))
    cand = np.sort(rng.choice(np.arange(1, 30), size=n, replace=False))
    scores = rng.integers(-3, 4, size=n).astype(np.float64)  # many exact ties
    k = int(rng.integers(0, 11))
    got = sorted(int(x) for x in O.select_topk(scores, cand, k))
    assert got == [int(x) for x in _brute_topk(scores, cand, k)]


def test_route_structure_and_threshold_property():
    rng = np.random.default_rng(3)
    b, Hq, Hkv, N, d, B, k = 2, 4, 2, 8 * 16 + 5, 8, 16, 3
    Q = rng.standard_normal((b, Hq, N, d))
    K = rng.standard_normal((b, Hkv, N, d))
    S = O.block_summary(K, B)
    idx, cnt, sc = O.route(Q, S, B, k, Hkv)
    nq = -(-N // B)
    assert idx.shape == (b, Hkv, nq, k + 2)
    for bi, g, i in itertools.product(range(b), range(Hkv), range(nq)):
        sel = list(idx[bi, g, i, : cnt[bi, g, i]])
        assert sel == sorted(set(sel))
        assert np.all(idx[bi, g, i, cnt[bi, g, i]:] == -1)
        assert sel[0] == 0 and sel[-1] == i
        assert cnt[bi, g, i] == (1 if i == 0 else 2 + min(k, max(i - 1, 0)))
        routed = [j for j in sel if j not in (0, i)]
        rest = [j for j in range(1, i) if j not in routed]
        if routed and rest:  # every routed block outscores every dropped candidate
            assert min(sc[bi, g, i, routed]) > max(sc[bi, g, i, rest])


def test_route_exact_ties_go_to_lower_index():
    # Blocks 2, 5 and 7 are identical and aligned with every query, so their
    # scores tie exactly at the top; with k = 2 blocks 2 and 5 must win.
    rng = np.random.default_rng(4)
    B, d, nb = 8, 16, 10
    K = rng.standard_normal((1, 1, nb * B, d)) * 0.1
    u = rng.standard_normal(d)
    blk = rng.standard_normal((B, d)) * 0.1 + u
    for j in (2, 5, 7):
        K[0, 0, j * B : (j + 1) * B] = blk
    Q = np.broadcast_to(u, (1, 1, nb * B, d)).copy()
    S = O.block_summary(K, B)
    assert S[0, 0, 2].tobytes() == S[0, 0, 5].tobytes() == S[0, 0, 7].tobytes()
    idx, cnt, _ = O.route(Q, S, B, 2, 1)
    assert list(idx[0, 0, 9, : cnt[0, 0, 9]]) == [0, 2, 5, 9]
    assert list(idx[0, 0, 8, : cnt[0, 0, 8]]) == [0, 2, 5, 8]
    assert list(idx[0, 0, 6, : cnt[0, 0, 6]])[:3] == [0, 2, 5]


def test_route_planted_clusters_are_found():
    Q, K, V = planted_prefill(1, 4, 1, 64 * 40, 64, 64, clusters=4, seed=7, dtype="f32")
    Qf, Kf = to_f64(Q), to_f64(K)
    S = O.block_summary(Kf, 64)
    idx, cnt, sc = O.route(Qf, S, 64, 40, 1)  # k >= candidates: pin structure only
    # With k large every candidate is taken; with k = #same-cluster blocks, the
    # routed set must be exactly the same-cluster blocks (scores ~1.4 vs ~0).
    qb = O.pool_query_blocks(Qf, 64, 1)[0, 0]
    Sb = S[0, 0]
    hits = 0
    for i in range(20, 40):
        same = [j for j in range(1, i) if qb[i] @ Sb[j] / 8 > 0.7]
        if not same:
            continue
        idx2, cnt2, _ = O.route(Qf[:, :, : (i + 1) * 64], S[:, :, :i + 1], 64, len(same), 1)
        routed = [j for j in idx2[0, 0, i, : cnt2[0, 0, i]] if j not in (0, i)]
        assert routed == same
        hits += 1
    assert hits >= 10


# ------------------------------------------------------ stage 2: attention
def _dense_sdpa(Q, K, V):
    G = Q.shape[1] // K.shape[1]
    q = torch.from_numpy(Q)
    k = torch.from_numpy(K).repeat_interleave(G, dim=1)
    v = torch.from_numpy(V).repeat_interleave(G, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True).numpy()


@pytest.mark.parametrize("N,B", [(256, 32), (16 * 7 + 9, 16)])
def test_all_blocks_selected_equals_dense_causal_sdpa(N, B):
    rng = np.random.default_rng(5)
    b, Hq, Hkv, d = 2, 4, 2, 16
    Q, K, V = (rng.standard_normal((b, h, N, d)) for h in (Hq, Hkv, Hkv))
    S = O.block_summary(K, B)
    idx, cnt, _ = O.route(Q, S, B, 10**6, Hkv)
    out, lse = O.sparse_attention(Q, K, V, idx, cnt, B)
    ref = _dense_sdpa(Q, K, V)
    assert np.max(np.abs(out - ref)) / np.max(np.abs(ref)) < 1e-12
    # LSE against torch.logsumexp of the causally masked dense logits
    G = Hq // Hkv
    lg = torch.from_numpy(Q) @ torch.from_numpy(K).repeat_interleave(G, 1).transpose(-1, -2)
    lg = lg / math.sqrt(d)
    lg = lg.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(lg, -1).numpy(), rtol=0, atol=1e-12)


def _tiny_case(seed=6, k=2):
    rng = np.random.default_rng(seed)
    b, Hq, Hkv, N, d, B = 1, 4, 2, 8 * 9 + 3, 8, 8
    Q, K, V = (rng.standard_normal((b, h, N, d)) for h in (Hq, Hkv, Hkv))
    S = O.block_summary(K, B)
    idx, cnt, _ = O.route(Q, S, B, k, Hkv)
    return Q, K, V, idx, cnt, B


def test_probs_rows_sum_to_one_and_zero_outside_selection():
    Q, K, V, idx, cnt, B = _tiny_case()
    P = O.attention_probs(Q, K, idx, cnt, B)
    N = Q.shape[2]
    G = Q.shape[1] // K.shape[1]
    np.testing.assert_allclose(P.sum(-1), 1.0, rtol=0, atol=1e-12)
    for h in range(Q.shape[1]):
        for t in range(N):
            sel = idx[0, h // G, t // B, : cnt[0, h // G, t // B]]
            allowed = np.zeros(N, bool)
            for j in sel:
                allowed[j * B : (j + 1) * B] = True
            allowed[t + 1 :] = False
            assert np.all(P[0, h, t, ~allowed] == 0.0)
            assert np.all(P[0, h, t, allowed] > 0.0)


def test_output_is_probs_times_values():
    Q, K, V, idx, cnt, B = _tiny_case(k=3)
    P = O.attention_probs(Q, K, idx, cnt, B)
    out, _ = O.sparse_attention(Q, K, V, idx, cnt, B)
    G = Q.shape[1] // K.shape[1]
    ref = np.einsum("bhts,bhsd->bhtd", P, np.repeat(V, G, axis=1))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_zero_query_gives_mean_of_allowed_values():
    Q, K, V, idx, cnt, B = _tiny_case(k=2)
    Q = np.zeros_like(Q)
    out, lse = O.sparse_attention(Q, K, V, idx, cnt, B)
    N = Q.shape[2]
    G = Q.shape[1] // K.shape[1]
    for h in range(Q.shape[1]):
        for t in range(N):
            sel = idx[0, h // G, t // B, : cnt[0, h // G, t // B]]
            pos = [s for j in sel for s in range(j * B, min(N, (j + 1) * B)) if s <= t]
            np.testing.assert_allclose(out[0, h, t], V[0, h // G, pos].mean(0), atol=1e-12)
            assert abs(lse[0, h, t] - math.log(len(pos))) < 1e-12


def test_error_bound_linear_in_dropped_mass():
    # o_full - o_sparse = sum_{j not in S} p_j v_j - delta/(1-delta) sum_{j in S} p_j v_j,
    # so |o_full - o_sparse| <= 2 * delta * max_j |v_j|  (SSA page, the error is
    # linear in the dropped attention mass).
    Q, K, V, idx, cnt, B = _tiny_case(seed=8, k=1)
    out, _ = O.sparse_attention(Q, K, V, idx, cnt, B)
    full = _dense_sdpa(Q, K, V)
    N = Q.shape[2]
    G = Q.shape[1] // K.shape[1]
    d = Q.shape[-1]
    vmax = np.linalg.norm(V, axis=-1).max()
    for h in range(Q.shape[1]):
        g = h // G
        z = (Q[0, h] @ K[0, g].T) / math.sqrt(d)
        z = np.where(np.triu(np.ones((N, N), bool), 1), -np.inf, z)
        p = np.exp(z - z.max(-1, keepdims=True))
        p /= p.sum(-1, keepdims=True)
        for t in range(N):
            sel = idx[0, g, t // B, : cnt[0, g, t // B]]
            inside = np.zeros(N, bool)
            for j in sel:
                inside[j * B : (j + 1) * B] = True
            delta = p[t, ~inside].sum()
            err = np.linalg.norm(full[0, h, t] - out[0, h, t])
            assert err <= 2 * delta * vmax + 1e-12


# ------------------------------------------------- stage 2: backward pass
@pytest.mark.parametrize("N,B", [(128, 32), (16 * 5 + 7, 16)])
def test_backward_all_blocks_equals_autograd_of_dense_causal_sdpa(N, B):
    rng = np.random.default_rng(11)
    b, Hq, Hkv, d = 2, 4, 2, 16
    Q, K, V = (rng.standard_normal((b, h, N, d)) for h in (Hq, Hkv, Hkv))
    dO = rng.standard_normal((b, Hq, N, d))
    S = O.block_summary(K, B)
    idx, cnt, _ = O.route(Q, S, B, 10**6, Hkv)
    dQ, dK, dV = O.sparse_attention_backward(Q, K, V, idx, cnt, dO, B)
    q, k, v = (torch.from_numpy(x).requires_grad_() for x in (Q, K, V))
    G = Hq // Hkv
    out = torch.nn.functional.scaled_dot_product_attention(
        q, k.repeat_interleave(G, 1), v.repeat_interleave(G, 1), is_causal=True)
    (out * torch.from_numpy(dO)).sum().backward()
    for mine, ref in ((dQ, q.grad), (dK, k.grad), (dV, v.grad)):
        ref = ref.numpy()
        assert np.max(np.abs(mine - ref)) / np.max(np.abs(ref)) < 1e-12


def _loss(Q, K, V, idx, cnt, dO, B):
    out, _ = O.sparse_attention(Q, K, V, idx, cnt, B)
    return float(np.sum(out * dO))


def test_backward_matches_central_differences_with_fixed_selection():
    Q, K, V, idx, cnt, B = _tiny_case(seed=12, k=2)
    rng = np.random.default_rng(13)
    dO = rng.standard_normal(Q.shape)
    grads = O.sparse_attention_backward(Q, K, V, idx, cnt, dO, B)
    eps = 1e-5
    for which in range(3):
        for _ in range(3):
            u = rng.standard_normal(grads[which].shape)
            xs_p = [Q, K, V]
            xs_m = [Q, K, V]
            xs_p[which] = xs_p[which] + eps * u
            xs_m[which] = xs_m[which] - eps * u
            fd = (_loss(*xs_p, idx, cnt, dO, B) - _loss(*xs_m, idx, cnt, dO, B)) / (2 * eps)
            an = float(np.sum(grads[which] * u))
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(an))


def test_backward_gradient_stays_inside_one_blocks_selection():
    # dO nonzero on query block i only: dQ lives on block i's rows, dK and dV
    # on the keys block i attends (its selected blocks, the diagonal block up
    # to its last row) and are exactly 0 elsewhere.
    Q, K, V, idx, cnt, B = _tiny_case(seed=14, k=2)
    rng = np.random.default_rng(15)
    N = Q.shape[2]
    G = Q.shape[1] // K.shape[1]
    for i in (3, 6, (N - 1) // B):
        dO = np.zeros(Q.shape)
        t0, t1 = i * B, min(N, (i + 1) * B)
        dO[:, :, t0:t1] = rng.standard_normal((Q.shape[0], Q.shape[1], t1 - t0, Q.shape[3]))
        dQ, dK, dV = O.sparse_attention_backward(Q, K, V, idx, cnt, dO, B)
        rows = np.zeros(N, bool)
        rows[t0:t1] = True
        assert np.all(dQ[:, :, ~rows] == 0.0) and np.any(dQ[:, :, rows] != 0.0)
        for g in range(K.shape[1]):
            seen = np.zeros(N, bool)
            for j in idx[0, g, i, : cnt[0, g, i]]:
                seen[j * B : min(N, (j + 1) * B)] = True
            seen[t1:] = False
            assert np.all(dK[0, g, ~seen] == 0.0) and np.all(dV[0, g, ~seen] == 0.0)
            assert np.all(np.any(dV[0, g, seen] != 0.0, axis=-1))
        assert G > 1


def test_backward_key_and_value_gradient_sums():
    # Each softmax row sums to 1, so its Jacobian rows sum to 0: summed over
    # every key, dK vanishes and dV equals the sum of dO over the group.
    Q, K, V, idx, cnt, B = _tiny_case(seed=16, k=3)
    dO = np.random.default_rng(17).standard_normal(Q.shape)
    _, dK, dV = O.sparse_attention_backward(Q, K, V, idx, cnt, dO, B)
    G = Q.shape[1] // K.shape[1]
    for g in range(K.shape[1]):
        np.testing.assert_allclose(dK[0, g].sum(0), 0.0, rtol=0, atol=1e-12)
        np.testing.assert_allclose(dV[0, g].sum(0), dO[0, g * G : (g + 1) * G].sum((0, 1)),
                                   rtol=0, atol=1e-11)


def test_backward_value_shift_leaves_gradients_unchanged():
    # V + c shifts every output row by c and dO . O by dO . c, which cancels
    # in dS, so dQ and dK stay; dV = P^T dO does not read V.
    Q, K, V, idx, cnt, B = _tiny_case(seed=18, k=2)
    dO = np.random.default_rng(19).standard_normal(Q.shape)
    c = np.random.default_rng(20).standard_normal(V.shape[-1]) * 5.0
    a = O.sparse_attention_backward(Q, K, V, idx, cnt, dO, B)
    s = O.sparse_attention_backward(Q, K, V + c, idx, cnt, dO, B)
    for x, y in zip(a, s):
        np.testing.assert_allclose(x, y, rtol=0, atol=1e-11)


# ------------------------------------------------------------------ decode
def test_decode_all_blocks_equals_dense_last_row():
    q, Kc, Vc, L = planted_decode(3, 4, 2, 200, 16, 16, clusters=3, seed=9, dtype="f32",
                                  seqlens=[200, 37, 16])
    qf, Kf, Vf = to_f64(q), to_f64(Kc), to_f64(Vc)
    out, lse, idx, cnt = O.decode(qf, Kf, Vf, L.numpy(), 16, 10**6)
    G = 2
    for bi, Lb in enumerate(L.tolist()):
        k = torch.from_numpy(Kf[bi, :, :Lb]).repeat_interleave(G, 0)
        v = torch.from_numpy(Vf[bi, :, :Lb]).repeat_interleave(G, 0)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qf[bi])[:, None, :], k, v)[:, 0].numpy()
        np.testing.assert_allclose(out[bi], ref, rtol=0, atol=1e-12)
        last = (Lb - 1) // 16
        assert cnt[bi, 0] == min(last + 1, 10**6)


def test_decode_row_equals_prefill_row_with_same_selection():
    # Decode at position L-1 is the last row of prefill over the same L keys
    # when both attend the same blocks.
    rng = np.random.default_rng(10)
    Hq, Hkv, L, d, B, k = 4, 2, 16 * 6 + 5, 8, 16, 2
    Q = rng.standard_normal((1, Hq, L, d))
    K = rng.standard_normal((1, Hkv, L, d))
    V = rng.standard_normal((1, Hkv, L, d))
    q = Q[:, :, L - 1, :]
    od, _, idx_d, cnt_d = O.decode(q, K, V, np.array([L]), B, k)
    nq = -(-L // B)
    idx = np.full((1, Hkv, nq, k + 2), -1)
    cnt = np.zeros((1, Hkv, nq), np.int64)
    idx[0, :, nq - 1] = idx_d[0]
    cnt[0, :, nq - 1] = cnt_d[0]
    op, _ = O.sparse_attention(Q, K, V, idx, cnt, B, units=[(0, g, nq - 1) for g in range(Hkv)])
    np.testing.assert_allclose(od[0], op[0, :, L - 1], rtol=0, atol=1e-12)


def test_decode_route_threshold_property_and_structure():
    q, Kc, Vc, L = planted_decode(2, 8, 2, 64 * 30, 32, 64, clusters=5, seed=11, dtype="f32",
                                  seqlens=[64 * 30, 64 * 17 + 1])
    qf, Kf = to_f64(q), to_f64(Kc)
    S = np.stack([O.block_summary(Kf[b : b + 1], 64)[0] for b in range(2)])
    idx, cnt, sc = O.decode_route(qf, S, L.numpy(), 64, 4)
    for bi in range(2):
        last = (int(L[bi]) - 1) // 64
        for g in range(2):
            sel = list(idx[bi, g, : cnt[bi, g]])
            assert sel[0] == 0 and sel[-1] == last and len(sel) == 6
            routed = sel[1:-1]
            rest = [j for j in range(1, last) if j not in routed]
            assert min(sc[bi, g, routed]) > max(sc[bi, g, rest])


def test_generators_are_seeded():
    a = planted_prefill(1, 4, 2, 300, 16, 64, clusters=3, seed=3)
    b = planted_prefill(1, 4, 2, 300, 16, 64, clusters=3, seed=3)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_decode_scores_equal_mean_over_group_heads_of_dots():
    rng = np.random.default_rng(12)
    b, Hq, Hkv, d, nb = 2, 6, 2, 8, 7
    q = rng.standard_normal((b, Hq, d))
    S = rng.standard_normal((b, Hkv, nb, d))
    _, _, sc = O.decode_route(q, S, np.array([nb * 4, nb * 4]), 4, 2)
    G = Hq // Hkv
    for bi in range(b):
        for g in range(Hkv):
            for j in range(nb):
                vals = [float(q[bi, h] @ S[bi, g, j]) / math.sqrt(d) for h in range(g * G, (g + 1) * G)]
                assert abs(sc[bi, g, j] - sum(vals) / G) < 1e-12


# ---------------------------------------------------------------- decode: appending tokens
def test_append_from_empty_rebuilds_the_cache_and_every_summary():
    # Appending a cache's rows one by one, starting from empty, must give back
    # that cache and the summary of every complete block: nothing more, in the
    # same positions.
    rng = np.random.default_rng(40)
    b, h, Lmax, d, B = 2, 3, 40, 4, 8
    K = rng.integers(-9, 9, size=(b, h, Lmax, d)).astype(np.float64)
    V = rng.integers(-9, 9, size=(b, h, Lmax, d)).astype(np.float64)
    Kc = np.zeros_like(K)
    Vc = np.zeros_like(V)
    S = np.full((b, h, Lmax // B, d), np.nan)
    L = np.zeros(b, dtype=np.int64)
    for t in range(Lmax):
        Kc, Vc, S, L = O.decode_append(Kc, Vc, S, L, K[:, :, t], V[:, :, t], B)
        assert L.tolist() == [t + 1] * b
        done = (t + 1) // B
        assert np.isnan(S[:, :, done:]).all()  # no summary before its block is complete
    assert np.array_equal(Kc, K) and np.array_equal(Vc, V)
    # integer rows: the means are exact, so compare with the closed form directly
    for j in range(Lmax // B):
        assert np.array_equal(S[:, :, j], K[:, :, j * B:(j + 1) * B].sum(axis=2) / B)


def test_append_arithmetic_block_gives_its_midpoint():
    # Rows a + r*delta for r = 0..B-1 of one block: its mean is a + (B-1)/2 * delta.
    b, h, B, d = 1, 2, 16, 3
    a = np.array([1.0, -2.0, 0.5])
    delta = np.array([0.25, 1.0, -0.5])
    Lmax = 2 * B
    Kc = np.zeros((b, h, Lmax, d))
    Vc = np.zeros_like(Kc)
    S = np.zeros((b, h, Lmax // B, d))
    Kc[:, :, B:2 * B - 1] = a + np.arange(B - 1)[:, None] * delta  # rows B .. 2B-2 already there
    L = np.array([2 * B - 1])
    knew = np.broadcast_to(a + (B - 1) * delta, (b, h, d))
    Kc2, Vc2, S2, L2 = O.decode_append(Kc, Vc, S, L, knew, np.ones((b, h, d)), B)
    assert L2.tolist() == [2 * B]
    np.testing.assert_allclose(S2[0, :, 1], np.broadcast_to(a + (B - 1) / 2 * delta, (h, d)),
                               rtol=0, atol=1e-12)
    assert np.array_equal(S2[:, :, 0], S[:, :, 0])  # the other block's summary is untouched
    assert np.array_equal(Vc2[0, :, 2 * B - 1], np.ones((h, d)))


def test_append_leaves_incomplete_blocks_and_invalid_lengths_alone():
    rng = np.random.default_rng(41)
    b, h, Lmax, d, B = 4, 2, 24, 4, 8
    Kc = rng.standard_normal((b, h, Lmax, d))
    Vc = rng.standard_normal((b, h, Lmax, d))
    S = rng.standard_normal((b, h, Lmax // B, d))
    L = np.array([3, Lmax, -1, Lmax - 1])
    kn = rng.standard_normal((b, h, d))
    vn = rng.standard_normal((b, h, d))
    Kc2, Vc2, S2, L2 = O.decode_append(Kc, Vc, S, L, kn, vn, B)
    assert L2.tolist() == [4, Lmax, -1, Lmax]
    # sequence 0: row 3 written, block 0 not complete, its summary unchanged
    assert np.array_equal(Kc2[0, :, 3], kn[0]) and np.array_equal(Vc2[0, :, 3], vn[0])
    assert np.array_equal(S2[0], S[0])
    # sequences 1 and 2: full cache / negative length, nothing changes
    for bi in (1, 2):
        assert np.array_equal(Kc2[bi], Kc[bi]) and np.array_equal(Vc2[bi], Vc[bi])
        assert np.array_equal(S2[bi], S[bi])
    # sequence 3: the last row completes the last block, equal to block_summary of the result
    assert np.array_equal(Kc2[3, :, Lmax - 1], kn[3])
    np.testing.assert_allclose(S2[3, :, -1], O.block_summary(Kc2[3:4], B)[0, :, -1], rtol=0,
                               atol=1e-12)
    assert np.array_equal(S2[3, :, :-1], S[3, :, :-1])
