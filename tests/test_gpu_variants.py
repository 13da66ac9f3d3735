"""GPU-vs-oracle parity of the routing variants: per-query-head decode
routing and two-level (segment, then block) routing, through the C ABI.

Selections must equal the oracle's except near-ties (fp64 score gap below
1e-4 relative), which are counted.  For the two-level routing a near-tie may
sit at either level: between the last kept segment and the best segment left
out, or between the differing blocks.  Outputs are compared with the oracle on
the GPU's own selection.
"""
import numpy as np
import pytest
import torch

import oracle as O
from parity import (BF16_MAX_ABS, BF16_REL_L2, F32_MAX_ABS, NEAR_TIE_REL, compare_selection,
                    out_errors)
from workloads import planted_decode, planted_prefill, to_f64

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]
DEV = "cuda"


@pytest.fixture(scope="module")
def ssa():
    import block_sparse_top_summary_b200 as m
    m.load_library()
    return m


def _check(dtype, got, ref):
    ma, rel = out_errors(got, ref)
    if dtype == "f32":
        assert ma <= F32_MAX_ABS, (ma, rel)
    else:
        assert ma <= BF16_MAX_ABS and rel <= BF16_REL_L2, (ma, rel)


# ---------------------------------------------------------------- per-head decode
# bf16 with G <= 8 streams the union of a group's selections with head masks;
# fp32 and G = 16 take one unit per query head
@pytest.mark.parametrize("dtype,d,B,G", [("bf16", 128, 64, 4), ("f32", 64, 32, 2),
                                         ("bf16", 128, 64, 1), ("bf16", 64, 16, 8),
                                         ("bf16", 128, 128, 16), ("bf16", 128, 32, 2)])
def test_per_head_decode_parity(ssa, dtype, d, B, G):
    batch, Hkv, Lmax, topk = 3, 2, B * 12, 3
    q, Kc, Vc, L = planted_decode(batch, Hkv * G, Hkv, Lmax, d, B, 3, seed=80, dtype=dtype,
                                  seqlens=[Lmax, B * 7 + 5, 9])
    qd, Kd, Vd, Ld = q.to(DEV), Kc.to(DEV), Vc.to(DEV), L.to(DEV)
    S = ssa.ssa_block_summary(Kd, B)
    out, idx = ssa.ssa_decode_per_head(qd, Kd, Vd, S, Ld, B, topk)
    torch.cuda.synchronize()
    assert ssa.ssa_device_error() == 0
    gi = idx.cpu().numpy()
    gc = (gi >= 0).sum(-1)
    oi, oc = O.decode_route_per_head(to_f64(q), to_f64(S), L.numpy(), B, topk)
    Sf = to_f64(S)
    qf = to_f64(q)

    def scores(row):
        b, h = row
        return {j: float(Sf[b, h // G, j] @ qf[b, h]) / np.sqrt(d) for j in range(Sf.shape[2])}

    rows, near, bad = compare_selection(gi, gc, oi, oc, scores)
    assert not bad, bad[:3]
    ref = O.decode_per_head(qf, to_f64(Kc), to_f64(Vc), L.numpy(), gi, gc, B)
    _check(dtype, to_f64(out), ref)
    if G == 1:  # one head per group: bitwise the grouped decode
        Og, ig = ssa.ssa_decode(qd, Kd, Vd, S, Ld, B, topk)
        assert torch.equal(Og, out) and torch.equal(ig, idx)


def test_per_head_decode_heads_of_a_group_pick_differently(ssa):
    # four heads of one group with four different planted directions: each
    # head's own best block is in its selection, and the selections differ
    B, d, topk, nb = 64, 128, 1, 16
    gen = torch.Generator().manual_seed(81)
    Kc = torch.randn(1, 1, nb * B, d, generator=gen) * 0.1
    dirs = torch.randn(4, d, generator=gen)
    dirs = dirs / dirs.norm(dim=1, keepdim=True) * 8.0
    for h, j in enumerate((3, 6, 9, 12)):
        Kc[0, 0, j * B:(j + 1) * B] += dirs[h]
    q = dirs[None].clone()
    Kc = Kc.to(torch.bfloat16)
    Vc = torch.randn(1, 1, nb * B, d, generator=gen).to(torch.bfloat16)
    L = torch.tensor([nb * B], dtype=torch.int32)
    Kd = Kc.to(DEV)
    S = ssa.ssa_block_summary(Kd, B)
    _, idx = ssa.ssa_decode_per_head(q.to(torch.bfloat16).to(DEV), Kd, Vc.to(DEV), S, L.to(DEV),
                                     B, topk)
    got = [idx[0, h, :3].tolist() for h in range(4)]
    assert got == [[0, 3, 15], [0, 6, 15], [0, 9, 15], [0, 12, 15]]


# ---------------------------------------------------------------- two-level routing
def _hier_near_tie(qbar, S, i, M, k_seg, gpu, ora):
    """True when the differing selections of row i come from a near-tie at the
    segment level or at the block level (fp64 scores, 1e-4 relative)."""
    d = S.shape[-1]
    sc = (S @ qbar) / np.sqrt(d)
    Sm = O.segment_summaries(S[None, None], M)[0, 0]
    seg = (Sm @ qbar) / np.sqrt(d)

    def close(a, b):
        den = max(abs(a), abs(b))
        return den == 0 or abs(a - b) / den < NEAR_TIE_REL

    closed = [m for m in range(Sm.shape[0]) if (m + 1) * M <= i]
    elig = [m for m in closed if any(1 <= j < i for j in range(m * M, (m + 1) * M))]
    if len(elig) > k_seg:
        order = sorted(elig, key=lambda m: (-seg[m], m))
        if close(seg[order[k_seg - 1]], seg[order[k_seg]]):
            return True
    only_g = set(gpu) - set(ora)
    only_o = set(ora) - set(gpu)
    return len(only_g) == len(only_o) and all(
        any(close(sc[x], sc[y]) for y in only_o) for x in only_g)


@pytest.mark.parametrize("N,B,M,k_seg,k_blk,dtype", [
    (64 * 40 + 9, 64, 4, 3, 6, "bf16"),
    (32 * 70, 32, 8, 2, 5, "f32"),
    (64 * 33, 64, 2, 5, 4, "bf16"),
    (128 * 24, 128, 3, 1, 2, "bf16"),
])
def test_hierarchical_route_parity(ssa, N, B, M, k_seg, k_blk, dtype):
    d, Hq, Hkv = 128, 8, 2
    Q, K, _ = planted_prefill(1, Hq, Hkv, N, d, B, 6, seed=90, dtype=dtype)
    S = ssa.ssa_block_summary(K.to(DEV), B)
    idx, cnt = ssa.ssa_route_hierarchical(Q.to(DEV), S, B, M, k_seg, k_blk, Hkv)
    torch.cuda.synchronize()
    oi, oc = O.hierarchical_route(to_f64(Q), to_f64(S), B, M, k_seg, k_blk, Hkv)
    gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
    qbar = O.pool_query_blocks(to_f64(Q), B, Hkv)
    Sf = to_f64(S)
    near = 0
    for g in range(Hkv):
        for i in range(gc.shape[2]):
            a = gi[0, g, i, :gc[0, g, i]].tolist()
            b = oi[0, g, i, :oc[0, g, i]].tolist()
            assert a == sorted(a) and all(x == -1 for x in gi[0, g, i, gc[0, g, i]:])
            if a != b:
                assert _hier_near_tie(qbar[0, g, i], Sf[0, g], i, M, k_seg, a, b), (g, i, a, b)
                near += 1
    assert near <= max(1, gc.size // 50)


def test_hierarchical_route_with_one_block_segments_is_the_flat_route(ssa):
    # M = 1 and every segment kept: the pool is every candidate, so the
    # selection is ssa_route's; both kernels pool and score with the same
    # code, so the selections are bitwise equal
    B, N, topk = 64, 64 * 50 + 7, 5
    Q, K, _ = planted_prefill(2, 8, 4, N, 128, B, 6, seed=91, dtype="bf16")
    Qd = Q.to(DEV)
    S = ssa.ssa_block_summary(K.to(DEV), B)
    hi, hc = ssa.ssa_route_hierarchical(Qd, S, B, 1, 64, topk, 4)
    fi, fc = ssa.ssa_route(Qd, S, B, topk, 4)
    assert torch.equal(hc, fc) and torch.equal(hi, fi)
