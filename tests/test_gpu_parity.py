"""GPU-vs-oracle parity on small inputs (several tiles, ragged tails, edge cases).

Every GPU call goes through the C ABI (ctypes binding).  Selections must match
the oracle exactly except near-ties (fp64 score gap < 1e-4 relative), which
are counted; outputs are compared with the oracle recomputed on the GPU's own
selection, at max-abs 1e-5 (fp32) or max-abs 2e-2 and relative-L2 5e-3 (bf16).
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from parity import BF16_MAX_ABS, BF16_REL_L2, F32_MAX_ABS, compare_selection, out_errors
from workloads import CONFIGS, planted_decode, planted_prefill, to_f64

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"


@pytest.fixture(scope="module")
def ssa():
    import block_sparse_top_summary_b200 as m
    m.load_library()
    return m


def _check_out(gpu, ref, dtype):
    ma, rel = out_errors(gpu, ref)
    if dtype == "f32":
        assert ma <= F32_MAX_ABS, (ma, rel)
    else:
        assert ma <= BF16_MAX_ABS and rel <= BF16_REL_L2, (ma, rel)
    return ma, rel


# ------------------------------------------------------------------ summary
@pytest.mark.parametrize("batch,Hkv,N,d,B,dtype", [
    (1, 1, 1024, 64, 64, "f32"),
    (2, 3, 64 * 7 + 13, 128, 64, "bf16"),
    (1, 2, 512, 128, 128, "f32"),
    (1, 1, 300, 64, 16, "bf16"),
    (2, 2, 4096, 128, 32, "bf16"),
])
def test_summary_parity(ssa, batch, Hkv, N, d, B, dtype):
    _, K, _ = planted_prefill(batch, Hkv, Hkv, N, d, B, clusters=3, seed=1, dtype=dtype)
    S = ssa.ssa_block_summary(K.to(DEV), B)
    ref = O.block_summary(to_f64(K), B)
    assert S.shape == ref.shape
    ma, _ = out_errors(to_f64(S), ref)
    assert ma <= 1e-5


def test_summary_constant_blocks_exact(ssa):
    c = torch.randint(-8, 8, (1, 2, 6, 128)).float()
    K = c.repeat_interleave(64, dim=2).to(torch.bfloat16).contiguous()
    S = ssa.ssa_block_summary(K.to(DEV), 64)
    assert torch.equal(S.cpu(), c)


# ------------------------------------------------------------------ routing
def _route_case(ssa, batch, Hq, Hkv, N, d, B, topk, dtype, clusters, seed):
    Q, K, _ = planted_prefill(batch, Hq, Hkv, N, d, B, clusters, seed=seed, dtype=dtype)
    S = ssa.ssa_block_summary(K.to(DEV), B)
    idx, cnt = ssa.ssa_route(Q.to(DEV), S, B, topk, Hkv)
    Qf, Kf = to_f64(Q), to_f64(K)
    oidx, ocnt, osc = O.route(Qf, O.block_summary(Kf, B), B, topk, Hkv)
    return idx.cpu().numpy(), cnt.cpu().numpy(), oidx, ocnt, osc


@pytest.mark.parametrize("batch,Hq,Hkv,N,d,B,topk,dtype,clusters", [
    (1, 2, 1, 1024, 64, 64, 4, "f32", 0),            # the tiny workload
    (1, 8, 2, 64 * 70 + 9, 128, 64, 6, "bf16", 5),   # ragged tail, 9 tiles of 8
    (2, 4, 4, 2048, 64, 32, 0, "f32", 4),            # top-k = 0: sink + diagonal only
    (1, 4, 1, 128 * 20, 128, 128, 1 << 30, "bf16", 3),  # "all"
    (1, 16, 4, 128 * 33, 128, 128, 8, "bf16", 8),    # B = 128
    (1, 4, 2, 16 * 300, 64, 16, 24, "bf16", 6),      # B = 16, many blocks
])
def test_route_parity(ssa, batch, Hq, Hkv, N, d, B, topk, dtype, clusters):
    gi, gc, oi, oc, osc = _route_case(ssa, batch, Hq, Hkv, N, d, B, topk, dtype, clusters, 2)
    assert np.array_equal(gc, oc)
    w = oi.shape[-1]
    assert np.all(gi[..., w:] == -1)
    rows, near, bad = compare_selection(gi, gc, oi, oc,
                                        lambda r: {j: osc[r][j] for j in range(osc.shape[-1])})
    assert not bad, bad[:3]
    assert near <= max(1, rows // 50)


@pytest.mark.parametrize("batch,Hq,Hkv,N,d,B,topk,dtype", [
    (1, 8, 2, 64 * 70 + 9, 128, 64, 6, "bf16"),   # ragged tail, 9 tiles of 8
    (2, 4, 4, 32 * 40, 64, 32, 5, "f32"),
])
def test_route_scores_output(ssa, batch, Hq, Hkv, N, d, B, topk, dtype):
    # The optional scores output holds, for every (query block i, block j),
    # the fp32 score the selection ranked: within fp32 rounding of the
    # oracle's fp64 q-bar . S_j / sqrt(d) on the candidates 1 .. i-1, -inf
    # elsewhere.  The GPU's own selection is exactly the top-k of these
    # scores (ties to the lower index), and passing the output changes
    # neither idx nor cnt.
    Q, K, _ = planted_prefill(batch, Hq, Hkv, N, d, B, 4, seed=7, dtype=dtype)
    Qd = Q.to(DEV)
    S = ssa.ssa_block_summary(K.to(DEV), B)
    idx0, cnt0 = ssa.ssa_route(Qd, S, B, topk, Hkv)
    idx, cnt, sc = ssa.ssa_route(Qd, S, B, topk, Hkv, want_scores=True)
    assert torch.equal(idx, idx0) and torch.equal(cnt, cnt0)
    sc = sc.cpu().double().numpy()
    nq, nfull = -(-N // B), N // B
    assert sc.shape == (batch, Hkv, nq, nfull)
    ref = O.summary_scores(O.pool_query_blocks(to_f64(Q), B, Hkv), O.block_summary(to_f64(K), B))
    i_ = np.arange(nq)[:, None]
    j_ = np.arange(nfull)[None, :]
    cand = (j_ >= 1) & (j_ <= i_ - 1)
    assert np.all(np.isneginf(sc[..., ~cand]))
    assert np.max(np.abs(sc[..., cand] - ref[..., cand])) <= 1e-5
    gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
    for b in range(batch):
        for g in range(Hkv):
            for i in range(nq):
                c = np.arange(1, max(i, 1))
                order = np.lexsort((c, -sc[b, g, i, c]))  # score desc, then index asc
                want = sorted({0, i} | set(c[order[:topk]].tolist()))
                assert gi[b, g, i, :gc[b, g, i]].tolist() == want, (b, g, i)


@pytest.mark.parametrize("nq", [7001, 14003])
def test_route_long_sequences(ssa, nq):
    # Query-block counts past the 8-block tiles' shared memory: tiles of 4
    # (7001 blocks) and of 2 (14003 blocks).  Sampled rows (spread over the
    # sequence, and the last ones) are checked against the oracle's pooled
    # queries, summaries and top-k, near-ties counted; every row is checked
    # for structure.
    B, d, Hq, Hkv, topk = 16, 64, 2, 1, 8
    N = nq * B - 5
    Q, K, _ = planted_prefill(1, Hq, Hkv, N, d, B, 8, seed=61, dtype="bf16")
    S = ssa.ssa_block_summary(K.to(DEV), B)
    idx, cnt = ssa.ssa_route(Q.to(DEV), S, B, topk, Hkv)
    torch.cuda.synchronize()
    gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
    for i in range(nq):
        sel = gi[0, 0, i, :gc[0, 0, i]]
        assert gc[0, 0, i] == min(topk, max(i - 1, 0)) + (2 if i > 0 else 1)
        assert sel[0] == 0 and sel[-1] == i and np.all(np.diff(sel) > 0)
    qbar = O.pool_query_blocks(to_f64(Q), B, Hkv)
    Sf = O.block_summary(to_f64(K), B)
    rows = sorted(set(np.linspace(2, nq - 1, 40).astype(int).tolist()) | {nq - 2, nq - 1})
    oi = np.full((len(rows), topk + 2), -1)
    oc = np.zeros(len(rows), dtype=np.int64)
    scs = {}
    for r, i in enumerate(rows):
        sc = O.summary_scores(qbar[:, :, i:i + 1], Sf)[0, 0, 0]
        cand = np.arange(1, i)
        want = sorted({0, i} | set(O.select_topk(sc[cand], cand, topk).tolist()))
        oi[r, :len(want)] = want
        oc[r] = len(want)
        scs[(r,)] = {int(j): float(sc[j]) for j in cand}
    n, near, bad = compare_selection(gi[0, 0, rows], gc[0, 0, rows], oi, oc, lambda row: scs[row])
    assert not bad, bad[:3]
    assert near <= 2


def test_route_tiny_matches_golden(ssa):
    import json
    import os
    doc = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.json")))
    c = CONFIGS["tiny"]
    Q, K, _ = planted_prefill(c.batch, c.Hq, c.Hkv, c.N, c.d, c.B, c.clusters, c.seed, c.dtype)
    S = ssa.ssa_block_summary(K.to(DEV), c.B)
    idx, cnt = ssa.ssa_route(Q.to(DEV), S, c.B, c.topk, c.Hkv)
    assert cnt[0, 0].tolist() == doc["cnt"]
    assert idx[0, 0].tolist() == doc["idx"]


def test_route_exact_ties_go_to_lower_index(ssa):
    torch.manual_seed(0)
    B, d, nb = 64, 128, 12
    K = torch.randn(1, 1, nb * B, d) * 0.1
    u = torch.randn(d)
    blk = torch.randn(B, d) * 0.1 + u
    for j in (2, 5, 7, 10):
        K[0, 0, j * B:(j + 1) * B] = blk
    Q = u.expand(1, 4, nb * B, d).contiguous()
    S = ssa.ssa_block_summary(K.to(DEV), B)
    idx, cnt = ssa.ssa_route(Q.to(DEV), S, B, 2, 1)
    idx = idx.cpu()
    assert idx[0, 0, 11, :cnt[0, 0, 11]].tolist() == [0, 2, 5, 11]
    assert idx[0, 0, 8, :cnt[0, 0, 8]].tolist() == [0, 2, 5, 8]


def _tied_levels(nq, case):
    """Per-block score level c_j (a power of two) for the long-row tie cases."""
    j = np.arange(nq)
    if case == "all_equal":
        return np.ones(nq)
    c = np.full(nq, 0.25)
    c[j % 5 == 3] = 0.5
    c[j % 11 == 0] = 1.0
    return c


@pytest.mark.parametrize("case,topk", [("all_equal", 8), ("all_equal", 32), ("tie_at_kth", 32)])
def test_route_long_rows_with_exact_ties(ssa, case, topk):
    # Rows of 64 and more candidates are first cut to the candidates at or
    # above the least lane maximum; rows with more than 256 of those (every
    # candidate, when all are equal) take the whole-row radix passes.  Both
    # routes must keep the ties at the k-th score to the lower index.  Every
    # summary is c_j u and every query u, with c_j a power of two, so the fp32
    # scores are exactly c_j (u.u)/sqrt(d): equal levels tie exactly.
    torch.manual_seed(5)
    B, d, nq, G = 16, 64, 300, 2
    N = B * nq
    u = torch.randn(d)
    c = _tied_levels(nq, case)
    S = (torch.from_numpy(c).float()[:, None] * u[None, :]).reshape(1, 1, nq, d).contiguous()
    Q = u.expand(1, G, N, d).contiguous()
    idx, cnt = ssa.ssa_route(Q.to(DEV), S.to(DEV), B, topk, 1)
    idx, cnt = idx.cpu().numpy()[0, 0], cnt.cpu().numpy()[0, 0]
    for i in range(nq):
        cands = sorted(range(1, i), key=lambda j: (-c[j], j))[:topk]
        want = sorted(set([0] + cands + [i]))
        assert cnt[i] == len(want), (case, i)
        assert idx[i, :cnt[i]].tolist() == want, (case, i)


# ---------------------------------------------------------------- attention
def _attn_case(ssa, batch, Hq, Hkv, N, d, B, topk, dtype, clusters, seed=3):
    Q, K, V = planted_prefill(batch, Hq, Hkv, N, d, B, clusters, seed=seed, dtype=dtype)
    Qd, Kd, Vd = Q.to(DEV), K.to(DEV), V.to(DEV)
    out, lse, idx, cnt, _ = ssa.prefill(Qd, Kd, Vd, B, topk)
    ref, rlse = O.sparse_attention(to_f64(Q), to_f64(K), to_f64(V), idx.cpu().numpy(),
                                   cnt.cpu().numpy(), B)
    return out, lse, ref, rlse


@pytest.mark.parametrize("batch,Hq,Hkv,N,d,B,topk,dtype,clusters", [
    (1, 2, 1, 1024, 64, 64, 4, "f32", 0),             # the tiny workload
    (1, 4, 2, 64 * 9 + 17, 128, 64, 3, "f32", 2),     # ragged, fp32 d=128
    (2, 8, 2, 64 * 12 + 5, 128, 64, 4, "bf16", 4),    # bf16, G = 4, ragged
    (1, 8, 2, 128 * 9, 128, 128, 3, "bf16", 3),       # bf16, B = 128
    (1, 4, 4, 32 * 20 + 31, 64, 32, 5, "bf16", 3),    # G = 1, B = 32, d = 64
    (1, 8, 1, 64 * 10, 128, 64, 1 << 30, "bf16", 0),  # all blocks (dense), G = 8
    (1, 4, 2, 16 * 40 + 5, 64, 16, 4, "bf16", 3),     # B = 16: half a key chunk
    (1, 2, 1, 48 * 12 + 7, 128, 48, 3, "f32", 2),     # B = 48: chunks straddle blocks
])
def test_attention_parity(ssa, batch, Hq, Hkv, N, d, B, topk, dtype, clusters):
    out, lse, ref, rlse = _attn_case(ssa, batch, Hq, Hkv, N, d, B, topk, dtype, clusters)
    _check_out(to_f64(out), ref, dtype)
    np.testing.assert_allclose(to_f64(lse), rlse, rtol=0, atol=1e-4)


@pytest.mark.parametrize("B,N", [(64, 64 * 230 + 37), (128, 128 * 120 + 5)])
def test_attention_many_items_per_cta(ssa, B, N):
    # More work items (256 query rows each) than SMs: every persistent CTA of
    # the tensor-core kernel runs several items back to back, so each item's
    # Q load, first S and first P.V follow the previous item's last S and
    # epilogue, with selection lengths that change from item to item and a
    # ragged last query block.  Every row is compared with the oracle.
    assert ssa.ssa_sparse_attn_uses_tensor_cores(torch.bfloat16, 8, 2, 128, B)
    out, lse, ref, rlse = _attn_case(ssa, 1, 8, 2, N, 128, B, 4, "bf16", 4, seed=21)
    _check_out(to_f64(out), ref, "bf16")
    np.testing.assert_allclose(to_f64(lse), rlse, rtol=0, atol=1e-4)


def test_all_blocks_equals_dense_causal(ssa):
    Q, K, V = planted_prefill(1, 8, 2, 64 * 16, 128, 64, 0, seed=5, dtype="bf16")
    out, _, _, cnt, _ = ssa.prefill(Q.to(DEV), K.to(DEV), V.to(DEV), 64, 1 << 30)
    assert cnt.cpu()[0, 0].tolist() == [i + 1 for i in range(16)]
    q = to_f64(Q)
    k = torch.from_numpy(to_f64(K)).repeat_interleave(4, 1)
    v = torch.from_numpy(to_f64(V)).repeat_interleave(4, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q), k, v,
                                                           is_causal=True).numpy()
    _check_out(to_f64(out), ref, "bf16")


def test_values_one_give_output_one(ssa):
    for dtype, tol in (("f32", 1e-6), ("bf16", 1e-2)):
        Q, K, V = planted_prefill(1, 8, 2, 64 * 8 + 3, 128, 64, 2, seed=6, dtype=dtype)
        V = torch.ones_like(V)
        out, _, _, _, _ = ssa.prefill(Q.to(DEV), K.to(DEV), V.to(DEV), 64, 2)
        assert torch.max(torch.abs(out.float() - 1.0)).item() <= tol


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_poisoned_unselected_and_future_keys_do_not_change_output(ssa, dtype):
    B, N, d = 64, 64 * 10, 128
    Q, K, V = planted_prefill(1, 8, 2, N, d, B, 3, seed=7, dtype=dtype)
    Qd, Kd, Vd = Q.to(DEV), K.to(DEV), V.to(DEV)
    i, t = 7, 7 * 64 + 20  # query block 7, check rows up to t
    nq = N // B
    idx = torch.full((1, 2, nq, 4), -1, dtype=torch.int32)
    cnt = torch.ones(1, 2, nq, dtype=torch.int32)
    idx[..., 0] = 0
    idx[0, :, i, :3] = torch.tensor([0, 3, i], dtype=torch.int32)
    cnt[0, :, i] = 3
    idx, cnt = idx.to(DEV), cnt.to(DEV)
    base, _ = ssa.ssa_sparse_attn_fwd(Qd, Kd, Vd, idx, cnt, B)
    Kp, Vp = Kd.clone(), Vd.clone()
    for j in range(nq):
        if j not in (0, 3, i):
            Kp[:, :, j * B:(j + 1) * B] = float("nan")
            Vp[:, :, j * B:(j + 1) * B] = float("nan")
    Kp[:, :, t + 1:(i + 1) * B] = 1e30
    Vp[:, :, t + 1:(i + 1) * B] = -1e30
    pois, _ = ssa.ssa_sparse_attn_fwd(Qd, Kp, Vp, idx, cnt, B)
    rows = slice(i * B, t + 1)
    assert torch.equal(base[:, :, rows], pois[:, :, rows])


# ------------------------------------------------------------------ decode
@pytest.mark.parametrize("batch,Hq,Hkv,Lmax,d,B,topk,dtype,seqlens", [
    (3, 8, 2, 1000, 128, 64, 4, "bf16", [1000, 37, 64 * 5 + 1]),
    (2, 4, 1, 64 * 40, 64, 64, 6, "f32", [64 * 40, 64 * 23 + 63]),
    (4, 16, 4, 128 * 30, 128, 128, 5, "bf16", [128 * 30, 1, 128, 129]),
    (2, 8, 1, 64 * 50, 128, 64, 1 << 30, "bf16", [64 * 50, 64 * 7 + 3]),   # all blocks
    (2, 6, 2, 16 * 200, 64, 16, 12, "bf16", [16 * 200, 16 * 77 + 5]),      # G = 3, B = 16
    # f32, d = 128: a block is two units of 32 keys; a last block of 40 keys
    # has a short second unit, one of 20 keys an empty one
    (3, 8, 2, 64 * 30, 128, 64, 5, "f32", [64 * 30, 64 * 23 + 40, 64 * 12 + 20]),
    # 64 (sequence, KV head) pairs x 18 blocks over one CTA per SM: every
    # pair is shared by several CTAs (partial records + combine)
    (8, 16, 8, 64 * 64, 128, 64, 16, "bf16",
     [64 * 64, 64 * 63 + 1, 64 * 40 + 17, 64 * 64 - 5, 64 * 20, 64 * 33 + 60, 64 * 50 + 2, 64 * 17]),
])
def test_decode_parity(ssa, batch, Hq, Hkv, Lmax, d, B, topk, dtype, seqlens):
    q, Kc, Vc, L = planted_decode(batch, Hq, Hkv, Lmax, d, B, clusters=5, seed=8, dtype=dtype,
                                  seqlens=seqlens)
    qd, Kd, Vd, Ld = q.to(DEV), Kc.to(DEV), Vc.to(DEV), L.to(DEV)
    S = ssa.ssa_block_summary(Kd, B)
    out, idx = ssa.ssa_decode(qd, Kd, Vd, S, Ld, B, topk)
    gi = idx.cpu().numpy()
    qf, Kf, Vf = to_f64(q), to_f64(Kc), to_f64(Vc)
    Sf = np.stack([O.block_summary(Kf[b:b + 1], B)[0] for b in range(batch)])
    oi, oc, osc = O.decode_route(qf, Sf, L.numpy(), B, topk)
    gc = (gi >= 0).sum(-1)
    rows, near, bad = compare_selection(gi, gc, oi, oc,
                                        lambda r: {j: osc[r][j] for j in range(osc.shape[-1])})
    assert not bad, bad[:3]
    ref, _, _, _ = O.decode(qf, Kf, Vf, L.numpy(), B, topk, idx=gi, cnt=gc)
    _check_out(to_f64(out), ref, dtype)


def test_decode_all_blocks_equals_dense_row(ssa):
    q, Kc, Vc, L = planted_decode(2, 8, 2, 777, 128, 64, 0, seed=9, dtype="bf16",
                                  seqlens=[777, 400])
    Kd = Kc.to(DEV)
    S = ssa.ssa_block_summary(Kd, 64)
    out, _ = ssa.ssa_decode(q.to(DEV), Kd, Vc.to(DEV), S, L.to(DEV), 64, 1 << 30)
    for b, Lb in enumerate([777, 400]):
        k = torch.from_numpy(to_f64(Kc[b, :, :Lb])).repeat_interleave(4, 0)
        v = torch.from_numpy(to_f64(Vc[b, :, :Lb])).repeat_interleave(4, 0)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(to_f64(q[b]))[:, None, :], k, v)[:, 0].numpy()
        _check_out(to_f64(out[b]), ref, "bf16")


def test_decode_invalid_seqlen_writes_zeros(ssa):
    q, Kc, Vc, _ = planted_decode(2, 4, 2, 256, 64, 64, 0, seed=10, dtype="f32")
    L = torch.tensor([0, 256], dtype=torch.int32, device=DEV)
    Kd = Kc.to(DEV)
    S = ssa.ssa_block_summary(Kd, 64)
    out, idx = ssa.ssa_decode(q.to(DEV), Kd, Vc.to(DEV), S, L, 64, 2)
    assert torch.all(out[0] == 0)
    assert torch.all(idx[0] == -1)
    assert torch.isfinite(out[1]).all()


def test_no_device_error_after_runs(ssa):
    assert ssa.ssa_device_error() == 0


@pytest.mark.parametrize("B", [64, 128])
def test_large_score_jump_in_a_later_block(ssa, B):
    # Block 3 scores ~600 above the others (a log2-domain jump far beyond any
    # lazy-rescale slack): the kernel must move its reference max and rescale
    # the partial output, and still match the oracle.
    torch.manual_seed(11)
    N, d, Hq, Hkv = B * 8, 128, 8, 2
    u = torch.nn.functional.normalize(torch.randn(d), dim=0)
    Q = (u * 3.0).expand(1, Hq, N, d).clone() + 0.01 * torch.randn(1, Hq, N, d)
    K = torch.randn(1, Hkv, N, d)
    K[:, :, 3 * B:4 * B] = u * 200.0 + 0.1 * torch.randn(B, d)
    V = torch.randn(1, Hkv, N, d)
    Q, K, V = (x.to(torch.bfloat16).contiguous() for x in (Q, K, V))
    out, lse, idx, cnt, _ = ssa.prefill(Q.to(DEV), K.to(DEV), V.to(DEV), B, 8)
    gi = idx.cpu().numpy()
    assert all(3 in gi[0, g, i, :cnt[0, g, i]] for g in range(Hkv) for i in range(4, 8))
    ref, rlse = O.sparse_attention(to_f64(Q), to_f64(K), to_f64(V), gi, cnt.cpu().numpy(), B)
    _check_out(to_f64(out), ref, "bf16")
    assert np.max(np.abs(to_f64(lse) - rlse)) < 1e-2


# ---------------------------------------------------------------- decode: appending tokens
@pytest.mark.parametrize("dtype,d,B", [("bf16", 128, 64), ("f32", 64, 16), ("bf16", 64, 128),
                                       ("f32", 128, 32)])
def test_decode_append_parity(ssa, dtype, d, B):
    # lengths: completing a block, mid-block, empty, full cache, last free slot
    batch, Hkv, Lmax = 5, 3, B * 6
    gen = torch.Generator().manual_seed(31)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    Kc = torch.randn(batch, Hkv, Lmax, d, generator=gen).to(tdt)
    Vc = torch.randn(batch, Hkv, Lmax, d, generator=gen).to(tdt)
    S = torch.randn(batch, Hkv, Lmax // B, d, generator=gen)
    L = torch.tensor([2 * B - 1, 3 * B + 5, 0, Lmax, Lmax - 1], dtype=torch.int32)
    kn = torch.randn(batch, Hkv, d, generator=gen).to(tdt)
    vn = torch.randn(batch, Hkv, d, generator=gen).to(tdt)
    rK, rV, rS, rL = O.decode_append(to_f64(Kc), to_f64(Vc), S.double().numpy(), L.numpy(),
                                     to_f64(kn), to_f64(vn), B)
    Kd, Vd, Sd, Ld = Kc.to(DEV), Vc.to(DEV), S.to(DEV), L.to(DEV)
    ssa.ssa_decode_append(Kd, Vd, Sd, Ld, kn.to(DEV), vn.to(DEV), B)
    assert Ld.cpu().tolist() == rL.tolist()
    assert np.array_equal(to_f64(Kd.cpu()), rK) and np.array_equal(to_f64(Vd.cpu()), rV)
    got = Sd.cpu().double().numpy()
    np.testing.assert_allclose(got, rS, rtol=0, atol=F32_MAX_ABS)
    changed = np.abs(rS - S.double().numpy()).max(axis=-1) > 0
    assert np.array_equal(got[~changed], S.double().numpy()[~changed])  # the rest untouched, bitwise


def test_decode_append_many_in_a_row_narrow_cache(ssa):
    # One KV head with d = 64 in bf16 keeps 16 of the CTA's 1024 threads busy
    # copying rows, so most warps read the length long after thread 0 could
    # have raised it.  200 appends in a row, nearly all of them ending
    # mid-block, must give the oracle's cache, summaries and lengths.
    B, d, batch, Hkv, Lmax = 64, 64, 3, 1, 64 * 5
    gen = torch.Generator().manual_seed(41)
    Kc = torch.zeros(batch, Hkv, Lmax, d).to(torch.bfloat16)
    Vc = torch.zeros(batch, Hkv, Lmax, d).to(torch.bfloat16)
    S = torch.zeros(batch, Hkv, Lmax // B, d)
    L = torch.tensor([0, 37, 250], dtype=torch.int32)
    Kd, Vd, Sd, Ld = Kc.to(DEV), Vc.to(DEV), S.to(DEV), L.to(DEV)
    rK, rV, rS, rL = to_f64(Kc), to_f64(Vc), S.double().numpy(), L.numpy()
    for _ in range(200):
        kn = torch.randn(batch, Hkv, d, generator=gen).to(torch.bfloat16)
        vn = torch.randn(batch, Hkv, d, generator=gen).to(torch.bfloat16)
        ssa.ssa_decode_append(Kd, Vd, Sd, Ld, kn.to(DEV), vn.to(DEV), B)
        rK, rV, rS, rL = O.decode_append(rK, rV, rS, rL, to_f64(kn), to_f64(vn), B)
    torch.cuda.synchronize()
    assert Ld.cpu().tolist() == rL.tolist() == [200, 237, Lmax]
    assert np.array_equal(to_f64(Kd.cpu()), rK) and np.array_equal(to_f64(Vd.cpu()), rV)
    np.testing.assert_allclose(Sd.cpu().double().numpy(), rS, rtol=0, atol=F32_MAX_ABS)


def test_append_then_decode_matches_oracle(ssa):
    # A serving loop: three appends, one of which completes a block, then one
    # decode step on the grown caches.
    B, topk = 64, 3
    q, Kc, Vc, L = planted_decode(2, 8, 2, B * 20, 128, B, 3, seed=12, dtype="bf16",
                                  seqlens=[B * 5 - 2, B * 11 + 7])
    Kd, Vd, Ld = Kc.to(DEV), Vc.to(DEV), L.to(DEV)
    Sd = ssa.ssa_block_summary(Kd, B)
    rK, rV, rS, rL = to_f64(Kc), to_f64(Vc), Sd.cpu().double().numpy(), L.numpy()
    gen = torch.Generator().manual_seed(13)
    for _ in range(3):
        kn = torch.randn(2, 2, 128, generator=gen).to(torch.bfloat16)
        vn = torch.randn(2, 2, 128, generator=gen).to(torch.bfloat16)
        ssa.ssa_decode_append(Kd, Vd, Sd, Ld, kn.to(DEV), vn.to(DEV), B)
        rK, rV, rS, rL = O.decode_append(rK, rV, rS, rL, to_f64(kn), to_f64(vn), B)
    assert Ld.cpu().tolist() == rL.tolist() == [B * 5 + 1, B * 11 + 10]
    np.testing.assert_allclose(Sd.cpu().double().numpy()[0, :, 4], O.block_summary(rK[:1], B)[0, :, 4],
                               rtol=0, atol=F32_MAX_ABS)  # the block the second append completed
    out, idx = ssa.ssa_decode(q.to(DEV), Kd, Vd, Sd, Ld, B, topk)
    gi = idx.cpu().numpy()
    gc = (gi >= 0).sum(-1)
    oi, oc, osc = O.decode_route(to_f64(q), rS, rL, B, topk)
    rows, near, bad = compare_selection(gi, gc, oi, oc,
                                        lambda r: {j: osc[r][j] for j in range(osc.shape[-1])})
    assert not bad, bad[:3]
    ref, _, _, _ = O.decode(to_f64(q), rK, rV, rL, B, topk, idx=gi, cnt=gc)
    _check_out(to_f64(out), ref, "bf16")
