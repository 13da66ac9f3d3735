"""The benchmark's work accounting against an independent count.

``bench.attn_flops`` counts 4 d FLOPs per unmasked (query, key) pair of the
selected blocks from the routing counts alone.  The oracle's attention matrix
P has a positive entry exactly for every such pair, so counting them is an
independent check, including the ragged last block and GQA groups.
"""
import numpy as np
import pytest

import bench
import oracle as O


@pytest.mark.parametrize("N,B,topk,Hq,Hkv", [(8 * 9 + 3, 8, 2, 4, 2), (16 * 6, 16, 1, 2, 1),
                                            (8 * 7 + 5, 8, 100, 3, 1)])
def test_attn_flops_counts_every_attended_pair(N, B, topk, Hq, Hkv):
    rng = np.random.default_rng(N + topk)
    d = 8
    Q = rng.standard_normal((1, Hq, N, d))
    K = rng.standard_normal((1, Hkv, N, d))
    idx, cnt, _ = O.route(Q, O.block_summary(K, B), B, topk, Hkv)
    P = O.attention_probs(Q, K, idx, cnt, B)
    pairs = int(np.count_nonzero(P > 0))
    G = Hq // Hkv
    flops = sum(bench.attn_flops(cnt[0, g], N, B, G, d) for g in range(Hkv))
    assert flops == pairs * 4 * d


def test_decode_bytes_counts_the_rows_each_selection_reads():
    # K and V rows = cache positions t < L whose block is selected; summaries =
    # the complete candidate blocks 1 .. last-1 (fp32); plus q and O
    rng = np.random.default_rng(5)
    batch, Hq, Hkv, Lmax, d, B, topk = 3, 4, 2, 8 * 10, 8, 8, 3
    q = rng.standard_normal((batch, Hq, d))
    Kc = rng.standard_normal((batch, Hkv, Lmax, d))
    L = np.array([80, 43, 1])
    S = np.stack([O.block_summary(Kc[b : b + 1], B)[0] for b in range(batch)])
    idx, cnt, _ = O.decode_route(q, S, L, B, topk)
    esize = 2
    expect = 0.0
    for b in range(batch):
        last = (L[b] - 1) // B
        for g in range(Hkv):
            sel = set(int(j) for j in idx[b, g, : cnt[b, g]])
            rows = sum(1 for t in range(L[b]) if t // B in sel)
            expect += 2 * rows * d * esize + len(range(1, max(last, 1))) * d * 4
    expect += 2 * batch * Hq * d * esize
    assert bench.decode_bytes(idx, L, B, d, Hq // Hkv, esize) == expect


def test_per_head_decode_bytes_counts_the_union_of_a_groups_rows():
    # the K/V rows of the blocks any head of a KV head's group selects (once),
    # that KV head's candidate summaries (once), and every head's q and O
    rng = np.random.default_rng(6)
    batch, Hq, Hkv, Lmax, d, B, topk = 2, 4, 2, 8 * 9, 8, 8, 2
    G = Hq // Hkv
    L = np.array([72, 30])
    idx = np.full((batch, Hq, topk + 2), -1)
    for b in range(batch):
        last = (L[b] - 1) // B
        for h in range(Hq):
            cand = rng.choice(np.arange(1, max(last, 2)), size=min(topk, max(last - 1, 0)),
                              replace=False) if last > 1 else np.array([], dtype=int)
            sel = sorted({0, last} | set(int(c) for c in cand))
            idx[b, h, :len(sel)] = sel
    esize = 2
    expect = 0.0
    for b in range(batch):
        last = (L[b] - 1) // B
        for g in range(Hkv):
            sel = set(int(j) for h in range(g * G, (g + 1) * G) for j in idx[b, h] if j >= 0)
            rows = sum(1 for t in range(L[b]) if t // B in sel)
            expect += 2 * rows * d * esize + len(range(1, max(last, 1))) * d * 4
    expect += 2 * batch * Hq * d * esize
    assert bench.per_head_decode_bytes(idx, L, B, d, G, esize) == expect
    # one head per group: the grouped count
    assert bench.per_head_decode_bytes(idx[:, ::2], L, B, d, 1, esize) == \
        bench.decode_bytes(idx[:, ::2], L, B, d, 1, esize)
