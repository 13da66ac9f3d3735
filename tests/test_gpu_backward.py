"""GPU-vs-oracle parity of the backward pass of the selected-block attention.

Both sides take the oracle's selection, so routing plays no part.  The GPU
backward gets the GPU forward's O (bf16) and log-sum-exp.

Tolerance, per gradient tensor: the bf16 bounds that hold for every output of
this library, relative-L2 <= 5e-3 and max-abs <= 2e-2.  An absolute bound only
means something on values of a known scale, so the upstream gradient dO is
drawn with standard deviation 1/4: every gradient then stays below 4 in
magnitude (the largest over these cases is about 2.3), where one bf16
rounding of an output costs at most half an ulp, 2^-7 = 0.0078.  (With dO of
standard deviation 1 the gradients reach 9, and a single bf16 rounding there
is already 0.031.)  The kernel also rounds P and dS to bf16 as mma operands
(2^-9 relative each) and forms delta from the bf16 O; the relative-L2 error
this gives is about 2.6e-3.  A max-abs bound relative to the tensor's largest
magnitude (2e-2) is kept as an extra check.
"""
import numpy as np
import pytest
import torch

import oracle as O
from parity import out_errors
from workloads import planted_prefill, to_f64, upstream_grad

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"
REL_L2 = 5e-3      # bf16 relative-L2 bound
MAX_ABS = 2e-2     # bf16 max-abs bound
MAX_ABS_REL = 2e-2
DO_STD = 0.25      # standard deviation of the upstream gradient


@pytest.fixture(scope="module")
def ssa():
    import block_sparse_top_summary_b200 as m
    m.load_library()
    return m


def _case(ssa, batch, Hq, Hkv, N, d, B, topk, clusters, seed):
    Q, K, V = planted_prefill(batch, Hq, Hkv, N, d, B, clusters, seed=seed, dtype="bf16")
    dO = upstream_grad(batch, Hq, N, d, seed=seed + 100, dtype="bf16", std=DO_STD)
    Qf, Kf, Vf, dOf = (to_f64(x) for x in (Q, K, V, dO))
    idx, cnt, _ = O.route(Qf, O.block_summary(Kf, B), B, topk, Hkv)
    gi = torch.from_numpy(idx.astype(np.int32)).to(DEV)
    gc = torch.from_numpy(cnt.astype(np.int32)).to(DEV)
    Qd, Kd, Vd, dOd = (x.to(DEV) for x in (Q, K, V, dO))
    Od, lse = ssa.ssa_sparse_attn_fwd(Qd, Kd, Vd, gi, gc, B)
    dQ, dK, dV = ssa.ssa_sparse_attn_bwd(Qd, Kd, Vd, Od, dOd, lse, gi, gc, B)
    torch.cuda.synchronize()
    assert ssa.ssa_device_error() == 0
    ref = O.sparse_attention_backward(Qf, Kf, Vf, idx, cnt, dOf, B)
    return (to_f64(dQ), to_f64(dK), to_f64(dV)), ref, (idx, cnt)


def _check(gpu, ref):
    for name, g, r in zip(("dQ", "dK", "dV"), gpu, ref):
        assert g.shape == r.shape, name
        assert np.all(np.isfinite(g)), name
        ma, rel = out_errors(g, r)
        scale = float(np.max(np.abs(r)))
        assert scale < 4.0, (name, scale)  # the range the absolute bound is stated for
        assert rel <= REL_L2 and ma <= MAX_ABS, (name, ma, rel)
        assert ma <= MAX_ABS_REL * scale, (name, ma, scale)


@pytest.mark.parametrize("batch,Hq,Hkv,N,d,B,topk,clusters", [
    (1, 4, 2, 64 * 9, 128, 64, 3, 4),           # GQA 2, several blocks
    (1, 4, 1, 32 * 11 + 13, 64, 32, 2, 3),      # ragged tail, d = 64, GQA 4
    (2, 8, 2, 128 * 5 + 40, 128, 128, 2, 3),    # B = 128 (8 warps), ragged, batch 2
    (1, 2, 2, 16 * 40, 64, 16, 4, 5),           # B = 16: one warp, a chunk wider than B
    (1, 4, 4, 64 * 300, 128, 64, 4, 8),         # > 128 query blocks per key-block scan
    (1, 8, 2, 64 * 150 + 5, 128, 64, 4, 5),     # GQA 4: the sink column in 3 ranges of 64
    (2, 4, 2, 128 * 70, 64, 128, 3, 4),         # B = 128, sink in 3 ranges of 32, batch 2
    # tensor-core passes (bf16, d = 128, G * B a multiple of 256):
    (1, 8, 2, 64 * 20 + 7, 128, 64, 4, 3),      # dQ and dK/dV on tcgen05, ragged tail
    (2, 16, 4, 64 * 33, 128, 64, 6, 5),         # the same, batch 2, GQA 4
    (1, 4, 2, 128 * 9 + 5, 128, 128, 3, 3),     # dQ on tcgen05 at B = 128, GQA 2
])
def test_backward_parity(ssa, batch, Hq, Hkv, N, d, B, topk, clusters):
    gpu, ref, _ = _case(ssa, batch, Hq, Hkv, N, d, B, topk, clusters, seed=21)
    _check(gpu, ref)


def test_backward_all_blocks_selected(ssa):
    # top-k past every candidate: the gradients of dense causal attention
    gpu, ref, _ = _case(ssa, 1, 4, 2, 64 * 6 + 20, 128, 64, 1 << 20, 2, seed=22)
    _check(gpu, ref)


@pytest.mark.parametrize("Hq", [4, 8])  # 8: the tensor-core passes
def test_backward_zero_outside_every_selection(ssa, Hq):
    # dO nonzero on one query block only: dK and dV are exactly zero on every
    # key that block does not attend
    batch, Hkv, N, d, B, topk = 1, 2, 64 * 12, 128, 64, 2
    Q, K, V = planted_prefill(batch, Hq, Hkv, N, d, B, 4, seed=23, dtype="bf16")
    dO = upstream_grad(batch, Hq, N, d, seed=24, dtype="bf16")
    i = 9
    dO[:, :, : i * B] = 0
    dO[:, :, (i + 1) * B :] = 0
    idx, cnt, _ = O.route(to_f64(Q), O.block_summary(to_f64(K), B), B, topk, Hkv)
    gi = torch.from_numpy(idx.astype(np.int32)).to(DEV)
    gc = torch.from_numpy(cnt.astype(np.int32)).to(DEV)
    Qd, Kd, Vd = (x.to(DEV) for x in (Q, K, V))
    Od, lse = ssa.ssa_sparse_attn_fwd(Qd, Kd, Vd, gi, gc, B)
    dQ, dK, dV = ssa.ssa_sparse_attn_bwd(Qd, Kd, Vd, Od, dO.to(DEV), lse, gi, gc, B)
    dQ, dK, dV = dQ.cpu(), dK.cpu(), dV.cpu()
    rows = torch.zeros(N, dtype=torch.bool)
    rows[i * B : (i + 1) * B] = True
    assert torch.all(dQ[:, :, ~rows] == 0)
    for g in range(Hkv):
        seen = torch.zeros(N, dtype=torch.bool)
        for j in idx[0, g, i, : cnt[0, g, i]]:
            seen[j * B : (j + 1) * B] = True
        assert torch.all(dK[0, g, ~seen] == 0) and torch.all(dV[0, g, ~seen] == 0)
        assert torch.any(dV[0, g, seen] != 0)


def test_backward_is_deterministic(ssa):
    # 150 query blocks: the sink block's dK / dV are summed over three ranges
    batch, Hq, Hkv, N, d, B, topk = 1, 8, 2, 64 * 150, 128, 64, 6
    Q, K, V = planted_prefill(batch, Hq, Hkv, N, d, B, 6, seed=25, dtype="bf16", device=DEV)
    dO = upstream_grad(batch, Hq, N, d, seed=26, dtype="bf16", device=DEV)
    idx, cnt = ssa.ssa_route(Q, ssa.ssa_block_summary(K, B), B, topk, Hkv)
    Od, lse = ssa.ssa_sparse_attn_fwd(Q, K, V, idx, cnt, B)
    a = ssa.ssa_sparse_attn_bwd(Q, K, V, Od, dO, lse, idx, cnt, B)
    b = ssa.ssa_sparse_attn_bwd(Q, K, V, Od, dO, lse, idx, cnt, B)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
