"""GPU parity of decode and append over a paged KV cache.

Each case builds one cache twice, contiguous and cut into pages in a shuffled
page order.  The paged GPU calls are compared with the oracle's paged
functions (selection exactly, near-ties counted; outputs on the GPU's
selection at the usual tolerances) and, where both describe the same cache,
bitwise with the contiguous GPU path.  Cases: shared prefix pages, blocks
past the length without a page, rows past the length poisoned with NaN, and
an append whose next block has no page.
"""
import numpy as np
import pytest
import torch

import oracle as O
from parity import BF16_MAX_ABS, BF16_REL_L2, F32_MAX_ABS, compare_selection, out_errors
from workloads import planted_decode, to_f64

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]
DEV = "cuda"


@pytest.fixture(scope="module")
def ssa():
    import block_sparse_top_summary_b200 as m
    m.load_library()
    return m


def _to_pages(C, B, order, extra=0):
    """Cut a contiguous cache [b, Hkv, nb * B, d] into pages in the given order."""
    b, Hkv, L, d = C.shape
    nb = L // B
    P = torch.zeros(len(order) + extra, Hkv, B, d, dtype=C.dtype)
    pt = torch.empty(b, nb, dtype=torch.int32)
    for bi in range(b):
        for j in range(nb):
            page = int(order[bi * nb + j])
            P[page] = C[bi, :, j * B:(j + 1) * B]
            pt[bi, j] = page
    return P, pt


def _check(dtype, got, ref):
    ma, rel = out_errors(got, ref)
    if dtype == "f32":
        assert ma <= F32_MAX_ABS, (ma, rel)
    else:
        assert ma <= BF16_MAX_ABS and rel <= BF16_REL_L2, (ma, rel)


@pytest.mark.parametrize("dtype,d,B", [("bf16", 128, 64), ("f32", 64, 32), ("bf16", 64, 16),
                                       ("bf16", 128, 128)])
def test_paged_decode_matches_oracle_and_contiguous_path(ssa, dtype, d, B):
    batch, Hq, Hkv, topk = 3, 8, 2, 3
    nb = 12
    Lmax = B * nb
    q, Kc, Vc, L = planted_decode(batch, Hq, Hkv, Lmax, d, B, 3, seed=70, dtype=dtype,
                                  seqlens=[Lmax, B * 7 + 5, 9])
    order = np.random.default_rng(71).permutation(batch * nb + 4)
    Kp, pt = _to_pages(Kc, B, order)
    Vp, _ = _to_pages(Vc, B, order)
    S = ssa.ssa_block_summary(Kc.to(DEV), B)
    Op, ip = ssa.ssa_decode_paged(q.to(DEV), Kp.to(DEV), Vp.to(DEV), S, pt.to(DEV), L.to(DEV), B,
                                  topk)
    Oc, ic = ssa.ssa_decode(q.to(DEV), Kc.to(DEV), Vc.to(DEV), S, L.to(DEV), B, topk)
    torch.cuda.synchronize()
    assert ssa.ssa_device_error() == 0
    assert torch.equal(ip, ic) and torch.equal(Op, Oc)
    gi = ip.cpu().numpy()
    gc = (gi >= 0).sum(-1)
    ref, _, oi, oc = O.decode_paged(to_f64(q), to_f64(Kp), to_f64(Vp), pt.numpy(), L.numpy(), B,
                                    topk, S=to_f64(S))
    sc = O.decode_route(to_f64(q), to_f64(S), L.numpy(), B, topk)[2]
    rows, near, bad = compare_selection(gi, gc, oi, oc,
                                        lambda r: {j: sc[r][j] for j in range(sc.shape[-1])})
    assert not bad, bad[:3]
    ref2, _, _, _ = O.decode(to_f64(q), to_f64(Kc), to_f64(Vc), L.numpy(), B, topk, idx=gi, cnt=gc)
    _check(dtype, to_f64(Op), ref2)
    if near == 0:
        _check(dtype, to_f64(Op), ref)


def test_paged_decode_unmapped_tail_poisoned_rows_and_shared_prefix(ssa):
    # Sequence 1 shares sequence 0's first two pages (a common prefix); the
    # pages of blocks wholly past a sequence's length are unmapped (-1), and
    # every row at or past a length is NaN in the page pools.
    B, d, batch, Hq, Hkv, nb, topk = 64, 128, 3, 8, 2, 10, 2
    Lmax = B * nb
    q, Kc, Vc, L = planted_decode(batch, Hq, Hkv, Lmax, d, B, 3, seed=74, dtype="bf16",
                                  seqlens=[B * 9 + 17, B * 6 + 1, B * 3])
    Kc[1, :, :2 * B] = Kc[0, :, :2 * B]
    Vc[1, :, :2 * B] = Vc[0, :, :2 * B]
    order = np.random.default_rng(75).permutation(batch * nb + 3)
    Kp, pt = _to_pages(Kc, B, order)
    Vp, _ = _to_pages(Vc, B, order)
    pt[1, :2] = pt[0, :2]
    Ls = L.tolist()
    for bi in range(batch):
        for j in range(nb):
            page = int(pt[bi, j])
            if j * B >= Ls[bi]:
                pt[bi, j] = -1
            if bi == 1 and j < 2:
                continue  # shared with sequence 0, whose rows are all valid
            r0 = max(0, Ls[bi] - j * B)
            if r0 < B:
                Kp[page, :, r0:] = float("nan")
                Vp[page, :, r0:] = float("nan")
    S = ssa.ssa_block_summary(Kc.to(DEV), B)
    Op, ip = ssa.ssa_decode_paged(q.to(DEV), Kp.to(DEV), Vp.to(DEV), S, pt.to(DEV), L.to(DEV), B,
                                  topk)
    Oc, ic = ssa.ssa_decode(q.to(DEV), Kc.to(DEV), Vc.to(DEV), S, L.to(DEV), B, topk)
    torch.cuda.synchronize()
    assert ssa.ssa_device_error() == 0
    assert torch.isfinite(Op.float()).all()
    assert torch.equal(ip, ic) and torch.equal(Op, Oc)
    gi = ip.cpu().numpy()
    ref, _, _, _ = O.decode(to_f64(q), to_f64(Kc), to_f64(Vc), L.numpy(), B, topk, idx=gi,
                            cnt=(gi >= 0).sum(-1))
    _check("bf16", to_f64(Op), ref)


@pytest.mark.parametrize("dtype,d,B", [("bf16", 128, 64), ("f32", 64, 16)])
def test_paged_append_matches_oracle_and_contiguous_append(ssa, dtype, d, B):
    batch, Hkv, nb = 3, 2, 4
    Lmax = nb * B
    t = torch.bfloat16 if dtype == "bf16" else torch.float32
    order = np.random.default_rng(72).permutation(batch * nb + 2)
    Kc = torch.zeros(batch, Hkv, Lmax, d, dtype=t, device=DEV)
    Vc = torch.zeros_like(Kc)
    Kp = torch.zeros(len(order), Hkv, B, d, dtype=t, device=DEV)
    Vp = torch.zeros_like(Kp)
    pt_h = order[: batch * nb].reshape(batch, nb).astype(np.int32)
    pt = torch.from_numpy(pt_h).to(DEV)
    Sc = torch.zeros(batch, Hkv, nb, d, dtype=torch.float32, device=DEV)
    Sp = torch.zeros_like(Sc)
    Lc = torch.tensor([0, B - 1, 2 * B + 3], dtype=torch.int32, device=DEV)
    Lp = Lc.clone()
    rK, rV, rS, rL = (to_f64(Kp), to_f64(Vp), Sp.cpu().double().numpy(), Lp.cpu().numpy())
    g = torch.Generator(device=DEV).manual_seed(73)
    for _ in range(B + 2):
        kn = torch.randn(batch, Hkv, d, generator=g, device=DEV).to(t)
        vn = torch.randn(batch, Hkv, d, generator=g, device=DEV).to(t)
        ssa.ssa_decode_append(Kc, Vc, Sc, Lc, kn, vn, B)
        ssa.ssa_decode_append_paged(Kp, Vp, Sp, pt, Lp, kn, vn, B)
        rK, rV, rS, rL = O.decode_append_paged(rK, rV, rS, pt_h, rL, to_f64(kn), to_f64(vn), B)
    torch.cuda.synchronize()
    assert torch.equal(Lp, Lc)
    assert Lp.cpu().tolist() == rL.tolist()
    assert np.array_equal(to_f64(Kp), rK) and np.array_equal(to_f64(Vp), rV)
    np.testing.assert_allclose(Sp.cpu().double().numpy(), rS, rtol=0, atol=F32_MAX_ABS)
    gK = O.gather_pages(to_f64(Kp), pt_h)
    gV = O.gather_pages(to_f64(Vp), pt_h)
    assert np.array_equal(gK, to_f64(Kc)) and np.array_equal(gV, to_f64(Vc))
    assert torch.equal(Sp, Sc)


def test_paged_append_without_a_next_page_leaves_the_sequence_alone(ssa):
    B, d, Hkv = 16, 64, 1
    gen = torch.Generator().manual_seed(76)
    Kp = torch.randn(4, Hkv, B, d, generator=gen).to(torch.bfloat16)
    Vp = torch.randn(4, Hkv, B, d, generator=gen).to(torch.bfloat16)
    S = torch.zeros(2, Hkv, 3, d)
    pt = torch.tensor([[2, -1, -1], [0, 1, 3]], dtype=torch.int32)
    L = torch.tensor([B, B + 6], dtype=torch.int32)  # sequence 0's block 1 has no page
    kn = torch.randn(2, Hkv, d, generator=gen).to(torch.bfloat16)
    vn = torch.randn(2, Hkv, d, generator=gen).to(torch.bfloat16)
    rK, rV, rS, rL = O.decode_append_paged(to_f64(Kp), to_f64(Vp), S.double().numpy(), pt.numpy(),
                                           L.numpy(), to_f64(kn), to_f64(vn), B)
    Kd, Vd, Sd, Ld = Kp.to(DEV), Vp.to(DEV), S.to(DEV), L.to(DEV)
    ssa.ssa_decode_append_paged(Kd, Vd, Sd, pt.to(DEV), Ld, kn.to(DEV), vn.to(DEV), B)
    torch.cuda.synchronize()
    assert Ld.cpu().tolist() == rL.tolist() == [B, B + 7]
    assert np.array_equal(to_f64(Kd), rK) and np.array_equal(to_f64(Vd), rV)
    assert torch.equal(Kd.cpu()[2], Kp[2]) and torch.equal(Sd.cpu(), S)
