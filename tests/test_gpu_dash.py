"""GPU-vs-oracle parity of DashAttention's adaptive stages: the learned
summary (stage 0), alpha-entmax routing (stage 1) and attention with the
routing prior (stage 2), through the C ABI.

The support of alpha-entmax is decided by a threshold tau that the GPU finds
by bisection in fp32 and the oracle in fp64, so a candidate whose probability
is within the fp32 resolution of zero may be in one support and not the
other.  Such entries are counted and must be below 1e-4 on both sides; every
other probability must agree within 1e-4.  The prior attention is compared
with the oracle run on the GPU's own probabilities (as every output here is
compared on the GPU's own selection).
"""
import numpy as np
import pytest
import torch

import oracle as O
from parity import BF16_MAX_ABS, BF16_REL_L2, F32_MAX_ABS, out_errors
from workloads import planted_prefill, to_f64

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]
DEV = "cuda"
W_TOL = 1e-4


@pytest.fixture(scope="module")
def ssa():
    import block_sparse_top_summary_b200 as m
    m.load_library()
    return m


@pytest.mark.parametrize("N,d,B,dtype", [(64 * 9 + 5, 128, 64, "bf16"), (32 * 12, 64, 32, "f32"),
                                         (128 * 5, 128, 128, "bf16")])
def test_learned_summary_parity(ssa, N, d, B, dtype):
    _, K, _ = planted_prefill(2, 4, 2, N, d, B, 3, seed=50, dtype=dtype)
    qbar = torch.randn(2, d, generator=torch.Generator().manual_seed(51)) * 2.0
    S = ssa.ssa_learned_summary(K.to(DEV), qbar.to(DEV), B)
    ref = O.learned_block_summary(to_f64(K), B, qbar.double().numpy())
    assert S.shape == ref.shape
    ma, _ = out_errors(to_f64(S), ref)
    assert ma <= F32_MAX_ABS, ma


def test_learned_summary_with_zero_query_is_the_block_mean(ssa):
    _, K, _ = planted_prefill(1, 2, 2, 64 * 6, 128, 64, 3, seed=54, dtype="bf16")
    Kd = K.to(DEV)
    S = ssa.ssa_learned_summary(Kd, torch.zeros(2, 128, device=DEV), 64)
    ma, _ = out_errors(to_f64(S), to_f64(ssa.ssa_block_summary(Kd, 64)))
    assert ma <= 1e-6, ma


def _route(ssa, alpha, gamma, sigma, N=64 * 20 + 9, B=64, d=128, Hq=8, Hkv=2, seed=52):
    Q, K, V = planted_prefill(1, Hq, Hkv, N, d, B, 4, seed=seed, dtype="bf16")
    S = ssa.ssa_block_summary(K.to(DEV), B)
    idx, cnt, bias, w = ssa.ssa_route_entmax(Q.to(DEV), S, B, Hkv, alpha, gamma, sigma,
                                             want_w=True)
    torch.cuda.synchronize()
    return Q, K, V, S, idx, cnt, bias, w


@pytest.mark.parametrize("alpha,gamma", [(1.5, 8.0), (2.0, 4.0), (1.25, 16.0), (3.0, 6.0)])
def test_entmax_route_parity(ssa, alpha, gamma):
    sigma = 0.5
    Q, _, _, S, idx, cnt, bias, w = _route(ssa, alpha, gamma, sigma)
    ref = O.entmax_route(to_f64(Q), to_f64(S), 64, 2, alpha, gamma)
    wg = to_f64(w)
    assert np.max(np.abs(wg - ref)) <= W_TOL
    diff = (wg > 0) != (ref > 0)
    assert np.all(np.maximum(wg, ref)[diff] <= W_TOL), "support differs above the threshold"
    assert diff.sum() <= max(2, diff.size // 1000)
    # rows are distributions over the candidates (zero row for block 0)
    sums = wg.sum(-1)
    assert np.allclose(sums[..., 1:], 1.0, atol=1e-5) and np.all(sums[..., 0] == 0)
    # idx / cnt / bias are the support of the GPU's own w, ascending, then the diagonal
    cn, ix, bs = cnt.cpu().numpy(), idx.cpu().numpy(), bias.cpu().numpy()
    nq = cn.shape[2]
    for g in range(2):
        for i in range(nq):
            sel = list(ix[0, g, i, : cn[0, g, i]])
            assert sel[-1] == i and sel == sorted(sel)
            assert sel[:-1] == [j for j in range(min(i, wg.shape[3])) if wg[0, g, i, j] > 0]
            assert np.all(ix[0, g, i, cn[0, g, i]:] == -1)
            assert bs[0, g, i, cn[0, g, i] - 1] == 0.0
            for e, j in enumerate(sel[:-1]):
                assert abs(bs[0, g, i, e] - sigma * np.log(wg[0, g, i, j])) <= 1e-5


def test_entmax_route_sparsemax_is_sparse_and_matches(ssa):
    # alpha = 2 with a sharp gamma: a handful of blocks per row
    Q, _, _, S, idx, cnt, _, w = _route(ssa, 2.0, 32.0, 1.0, seed=55)
    ref = O.entmax_route(to_f64(Q), to_f64(S), 64, 2, 2.0, 32.0)
    assert np.max(np.abs(to_f64(w) - ref)) <= W_TOL
    cn = cnt.cpu().numpy()
    assert cn[0, :, 5:].mean() < 8  # sparse: far fewer blocks than candidates


@pytest.mark.parametrize("sigma,dtype,d,B,Hq", [
    (0.0, "bf16", 128, 64, 4), (0.7, "bf16", 128, 64, 4), (1.0, "f32", 64, 32, 4),
    (0.5, "bf16", 64, 16, 4),
    # the tensor-core kernel (bf16, d = 128, (Hq / Hkv) * B a multiple of 256)
    (0.7, "bf16", 128, 64, 8), (1.0, "bf16", 128, 128, 4), (0.0, "bf16", 128, 64, 8)])
def test_prior_attention_parity(ssa, sigma, dtype, d, B, Hq):
    N = B * 12 + 17
    Q, K, V = planted_prefill(1, Hq, 2, N, d, B, 3, seed=53, dtype=dtype)
    Qd, Kd, Vd = Q.to(DEV), K.to(DEV), V.to(DEV)
    S = ssa.ssa_block_summary(Kd, B)
    idx, cnt, bias, w = ssa.ssa_route_entmax(Qd, S, B, 2, 1.5, 8.0, sigma, want_w=True)
    out, lse = ssa.ssa_sparse_attn_fwd_prior(Qd, Kd, Vd, idx, cnt, bias, B)
    torch.cuda.synchronize()
    assert ssa.ssa_device_error() == 0
    ref, rlse = O.prior_sparse_attention(to_f64(Q), to_f64(K), to_f64(V), to_f64(w), B, sigma)
    ma, rel = out_errors(to_f64(out), ref)
    if dtype == "f32":
        assert ma <= F32_MAX_ABS, ma
    else:
        assert ma <= BF16_MAX_ABS and rel <= BF16_REL_L2, (ma, rel)
    np.testing.assert_allclose(to_f64(lse), rlse, rtol=0, atol=1e-4)


@pytest.mark.parametrize("Hq,d", [(4, 64), (8, 128)])  # (8, 128): the tensor-core kernel
def test_prior_attention_with_zero_sigma_is_topk_attention_on_the_support(ssa, Hq, d):
    # sigma = 0: no prior, so the result is the plain selected-block attention
    # over the entmax support plus the diagonal -- bitwise the kernel of
    # ssa_sparse_attn_fwd run on the same block lists
    B, N = 64, 64 * 10 + 3
    Q, K, V = planted_prefill(1, Hq, 2, N, d, B, 3, seed=56, dtype="bf16")
    Qd, Kd, Vd = Q.to(DEV), K.to(DEV), V.to(DEV)
    S = ssa.ssa_block_summary(Kd, B)
    idx, cnt, bias, _ = ssa.ssa_route_entmax(Qd, S, B, 2, 1.5, 8.0, 0.0)
    assert torch.all(bias == 0)
    a, la = ssa.ssa_sparse_attn_fwd_prior(Qd, Kd, Vd, idx, cnt, bias, B)
    b, lb = ssa.ssa_sparse_attn_fwd(Qd, Kd, Vd, idx, cnt, B)
    assert ssa.ssa_sparse_attn_uses_tensor_cores(torch.bfloat16, Hq, 2, d, B) == (Hq == 8)
    assert torch.equal(a, b) and torch.equal(la, lb)
