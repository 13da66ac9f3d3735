"""Pins for the paged-cache oracle: each case builds the same cache twice,
contiguous and paged in a shuffled page order, and checks the paged functions
against the pinned contiguous ones."""
import numpy as np

import oracle as O


def _paged_copy(Kc, B, rng, extra_pages=3):
    """Cut a contiguous cache [b, Hkv, nb*B, d] into pages in a random order."""
    b, Hkv, L, d = Kc.shape
    nb = L // B
    n = b * nb + extra_pages
    order = rng.permutation(n)
    P = np.full((n, Hkv, B, d), np.nan)
    pt = np.empty((b, nb), dtype=np.int64)
    for bi in range(b):
        for j in range(nb):
            page = order[bi * nb + j]
            pt[bi, j] = page
            P[page] = Kc[bi, :, j * B : (j + 1) * B]
    return P, pt, order


def _case(seed, b=3, Hq=8, Hkv=2, nb=7, d=16, B=8):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((b, Hq, d))
    Kc = rng.standard_normal((b, Hkv, nb * B, d))
    Vc = rng.standard_normal((b, Hkv, nb * B, d))
    return rng, q, Kc, Vc, B


def test_paged_decode_equals_contiguous_decode_in_any_page_order():
    rng, q, Kc, Vc, B = _case(60)
    L = np.array([56, 33, 9])
    Kp, pt, _ = _paged_copy(Kc, B, rng)
    Vp = np.full_like(Kp, np.nan)
    for bi in range(Kc.shape[0]):
        for j in range(pt.shape[1]):
            Vp[pt[bi, j]] = Vc[bi, :, j * B : (j + 1) * B]
    out, lse, idx, cnt = O.decode_paged(q, Kp, Vp, pt, L, B, 2)
    ref, rlse, ridx, rcnt = O.decode(q, Kc, Vc, L, B, 2)
    np.testing.assert_array_equal(idx, ridx)
    np.testing.assert_array_equal(cnt, rcnt)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rlse, rtol=0, atol=1e-12)


def test_paged_decode_reads_no_unmapped_page_and_no_row_past_the_length():
    rng, q, Kc, Vc, B = _case(61)
    L = np.array([50, 20, 41])
    Kp, pt, _ = _paged_copy(Kc, B, rng)
    Vp = np.full_like(Kp, np.nan)  # V in the same page order as K
    for bi in range(Kc.shape[0]):
        for j in range(pt.shape[1]):
            Vp[pt[bi, j]] = Vc[bi, :, j * B : (j + 1) * B]
    # poison every row at or past each sequence's length, and drop the pages
    # of blocks wholly past it from the table
    for bi, Lb in enumerate(L):
        for j in range(pt.shape[1]):
            rows = np.arange(j * B, (j + 1) * B) >= Lb
            Kp[pt[bi, j], :, rows] = np.nan
            Vp[pt[bi, j], :, rows] = np.nan
            if j * B >= Lb:
                pt[bi, j] = -1
    S = np.stack([O.block_summary(Kc[bi : bi + 1], B)[0] for bi in range(Kc.shape[0])])
    out, _, _, _ = O.decode_paged(q, Kp, Vp, pt, L, B, 3, S=S)
    ref, _, _, _ = O.decode(q, Kc, Vc, L, B, 3, S=S)
    assert np.all(np.isfinite(out))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_sequences_sharing_prefix_pages_attend_the_shared_blocks():
    rng, q, Kc, Vc, B = _case(62, b=2)
    Kc[1, :, : 2 * B] = Kc[0, :, : 2 * B]  # the same two-block prefix
    Vc[1, :, : 2 * B] = Vc[0, :, : 2 * B]
    L = np.array([56, 47])
    Kp, pt, _ = _paged_copy(Kc, B, rng)
    Vp = np.full_like(Kp, np.nan)
    for bi in range(2):
        for j in range(pt.shape[1]):
            Vp[pt[bi, j]] = Vc[bi, :, j * B : (j + 1) * B]
    pt[1, :2] = pt[0, :2]  # sequence 1 reads sequence 0's prefix pages
    out, _, _, _ = O.decode_paged(q, Kp, Vp, pt, L, B, 2)
    ref, _, _, _ = O.decode(q, Kc, Vc, L, B, 2)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_paged_append_equals_contiguous_append():
    rng = np.random.default_rng(63)
    b, Hkv, nb, d, B = 3, 2, 5, 8, 4
    pt = rng.permutation(b * nb + 2)[: b * nb].reshape(b, nb)
    n_pages = b * nb + 2
    Kp = np.zeros((n_pages, Hkv, B, d))
    Vp = np.zeros((n_pages, Hkv, B, d))
    Kc = np.zeros((b, Hkv, nb * B, d))
    Vc = np.zeros((b, Hkv, nb * B, d))
    S = np.zeros((b, Hkv, nb, d))
    Sc = np.zeros((b, Hkv, nb, d))
    L = np.zeros(b, dtype=np.int64)
    Lc = np.zeros(b, dtype=np.int64)
    for step in range(nb * B + 2):  # the last steps find the caches full
        kn = rng.standard_normal((b, Hkv, d))
        vn = rng.standard_normal((b, Hkv, d))
        Kp, Vp, S, L = O.decode_append_paged(Kp, Vp, S, pt, L, kn, vn, B)
        Kc, Vc, Sc, Lc = O.decode_append(Kc, Vc, Sc, Lc, kn, vn, B)
        np.testing.assert_array_equal(L, Lc)
        np.testing.assert_array_equal(O.gather_pages(Kp, pt), Kc)
        np.testing.assert_array_equal(O.gather_pages(Vp, pt), Vc)
        np.testing.assert_allclose(S, Sc, rtol=0, atol=1e-12)
    assert list(L) == [nb * B] * b


def test_paged_append_leaves_a_sequence_without_a_next_page_alone():
    rng = np.random.default_rng(64)
    B, d = 4, 8
    Kp = rng.standard_normal((4, 1, B, d))
    Vp = rng.standard_normal((4, 1, B, d))
    S = np.zeros((2, 1, 3, d))
    pt = np.array([[2, -1, -1], [0, 1, 3]])
    L = np.array([4, 6])
    kn = rng.standard_normal((2, 1, d))
    Kp2, Vp2, S2, L2 = O.decode_append_paged(Kp, Vp, S, pt, L, kn, kn, B)
    assert list(L2) == [4, 7]
    np.testing.assert_array_equal(Kp2[2], Kp[2])      # sequence 0: block 1 has no page
    np.testing.assert_array_equal(Kp2[1, 0, 2], kn[1, 0])  # sequence 1: row 6 = page 1, row 2


def test_gather_reads_unmapped_blocks_as_zeros():
    P = np.arange(2 * 1 * 4 * 3, dtype=np.float64).reshape(2, 1, 4, 3) + 1.0
    out = O.gather_pages(P, np.array([[-1, 0, -1, 1]]))
    assert np.all(out[0, :, 0:4] == 0.0) and np.all(out[0, :, 8:12] == 0.0)
    np.testing.assert_array_equal(out[0, :, 4:8], P[0])
    np.testing.assert_array_equal(out[0, :, 12:16], P[1])
