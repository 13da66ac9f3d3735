"""Pins for the oracle of the routing variants: per-head decode routing and
two-level (segment, then block) routing.  Each reduces, in a special case, to
the pinned flat routing or to torch's attention, or is checked on a planted
input whose answer is known by construction.
"""
import numpy as np
import torch

import oracle as O


def _sets(idx, cnt):
    return [sorted(int(x) for x in idx[u][: cnt[u]]) for u in np.ndindex(cnt.shape)]


# ------------------------------------------------------ per-head decode routing
def _decode_case(seed, Hq, Hkv, Lmax=64 * 10, d=32, B=64, lens=(640, 333, 65)):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((len(lens), Hq, d))
    Kc = rng.standard_normal((len(lens), Hkv, Lmax, d))
    Vc = rng.standard_normal((len(lens), Hkv, Lmax, d))
    S = np.stack([O.block_summary(Kc[b : b + 1], B)[0] for b in range(len(lens))])
    return q, Kc, Vc, S, np.array(lens), B


def test_per_head_routing_without_groups_is_the_decode_routing():
    q, Kc, Vc, S, L, B = _decode_case(30, Hq=3, Hkv=3)
    idx, cnt = O.decode_route_per_head(q, S, L, B, 3)
    gidx, gcnt, _ = O.decode_route(q, S, L, B, 3)
    assert _sets(idx, cnt) == _sets(gidx, gcnt)


def test_per_head_routing_of_identical_heads_is_the_group_selection():
    q, Kc, Vc, S, L, B = _decode_case(31, Hq=8, Hkv=2)
    q = np.repeat(q[:, ::4], 4, axis=1)  # every head of a group carries the same query
    idx, cnt = O.decode_route_per_head(q, S, L, B, 2)
    gidx, gcnt, _ = O.decode_route(q, S, L, B, 2)
    for b in range(q.shape[0]):
        for h in range(8):
            assert sorted(idx[b, h, : cnt[b, h]]) == sorted(gidx[b, h // 4, : gcnt[b, h // 4]])


def test_per_head_routing_heads_differ_and_each_keeps_its_best_block():
    q, Kc, Vc, S, L, B = _decode_case(32, Hq=4, Hkv=1, lens=(640,))
    idx, cnt = O.decode_route_per_head(q, S, L, B, 1)
    last = (L[0] - 1) // B
    for h in range(4):
        sc = S[0, 0, 1:last] @ q[0, h]
        assert 1 + int(np.argmax(sc)) in idx[0, h, : cnt[0, h]]
    assert len({tuple(idx[0, h]) for h in range(4)}) > 1


def test_per_head_decode_with_every_block_is_dense_attention():
    q, Kc, Vc, S, L, B = _decode_case(33, Hq=4, Hkv=2)
    idx, cnt = O.decode_route_per_head(q, S, L, B, 100)
    out = O.decode_per_head(q, Kc, Vc, L, idx, cnt, B)
    for b, Lb in enumerate(L):
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[b][:, None, :]),
            torch.from_numpy(np.repeat(Kc[b, :, :Lb], 2, 0)),
            torch.from_numpy(np.repeat(Vc[b, :, :Lb], 2, 0)))[:, 0].numpy()
        np.testing.assert_allclose(out[b], ref, rtol=0, atol=1e-12)


def test_per_head_decode_of_one_head_groups_is_the_decode():
    q, Kc, Vc, S, L, B = _decode_case(34, Hq=2, Hkv=2)
    idx, cnt = O.decode_route_per_head(q, S, L, B, 2)
    out = O.decode_per_head(q, Kc, Vc, L, idx, cnt, B)
    ref = O.decode(q, Kc, Vc, L, B, 2, idx=idx, cnt=cnt)[0]
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


# -------------------------------------------------------- two-level routing
def _prefill_case(seed, Hq=4, Hkv=2, N=8 * 23 + 3, d=16, B=8):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((1, Hq, N, d))
    K = rng.standard_normal((1, Hkv, N, d))
    return Q, K, O.block_summary(K, B), B, Hkv


def test_segment_summary_is_the_mean_of_the_segment_keys():
    Q, K, S, B, Hkv = _prefill_case(40)
    M = 4
    Sm = O.segment_summaries(S, M)
    np.testing.assert_allclose(Sm, O.block_summary(K, B * M)[:, :, : Sm.shape[2]], rtol=0,
                               atol=1e-12)


def test_two_level_with_every_segment_kept_is_the_flat_routing():
    Q, K, S, B, Hkv = _prefill_case(41)
    idx, cnt = O.hierarchical_route(Q, S, B, M=3, k_seg=100, k_blk=4, Hkv=Hkv)
    fidx, fcnt, _ = O.route(Q, S, B, 4, Hkv)
    assert _sets(idx, cnt) == _sets(fidx, fcnt)


def test_two_level_with_one_block_segments_is_flat_topk_of_the_smaller_k():
    Q, K, S, B, Hkv = _prefill_case(42)
    idx, cnt = O.hierarchical_route(Q, S, B, M=1, k_seg=3, k_blk=5, Hkv=Hkv)
    fidx, fcnt, _ = O.route(Q, S, B, 3, Hkv)
    assert _sets(idx, cnt) == _sets(fidx, fcnt)


def test_two_level_skips_a_strong_block_in_a_losing_segment():
    # block 5 alone scores highest, but its segment (blocks 4..7) loses the
    # meta-level vote to segment 0..3, whose four blocks all score well
    Q, K, S, B, Hkv = _prefill_case(43, Hq=1, Hkv=1)
    d = Q.shape[-1]
    i = 20
    qb = Q[0, 0, i * B : (i + 1) * B].mean(0)
    u = qb / np.linalg.norm(qb)
    S = np.zeros_like(S)
    S[0, 0, 1:4] = 3.0 * u
    S[0, 0, 5] = 5.0 * u
    S[0, 0, [4, 6, 7]] = -3.0 * u
    idx, cnt = O.hierarchical_route(Q, S, B, M=4, k_seg=1, k_blk=2, Hkv=1)
    fidx, fcnt, _ = O.route(Q, S, B, 2, 1)
    sel = sorted(idx[0, 0, i, : cnt[0, 0, i]])
    assert 5 in fidx[0, 0, i, : fcnt[0, 0, i]]
    assert 5 not in sel and sel[0] == 0 and sel[-1] == i
    # at i = 20 every segment up to blocks 16..19 is closed, so with k_seg = 1
    # only blocks 1..3 compete at the block level; two of them are kept
    assert len([j for j in sel if 1 <= j <= 3]) == 2


def test_two_level_recent_blocks_always_reach_the_block_level():
    # query block 13 with M = 4: segments 0..2 are closed (blocks 0..11), block
    # 12 sits in the open segment and competes at the block level unfiltered
    Q, K, S, B, Hkv = _prefill_case(44, Hq=1, Hkv=1)
    i = 13
    qb = Q[0, 0, i * B : (i + 1) * B].mean(0)
    u = qb / np.linalg.norm(qb)
    S = np.zeros_like(S)
    S[0, 0, 12] = 4.0 * u   # the open segment's block
    S[0, 0, 2] = 3.0 * u    # segment 0
    S[0, 0, 9] = 2.0 * u    # segment 2
    idx, cnt = O.hierarchical_route(Q, S, B, M=4, k_seg=1, k_blk=2, Hkv=1)
    sel = sorted(idx[0, 0, i, : cnt[0, 0, i]])
    assert sel == [0, 2, 12, 13]
