"""ssa_decode_noalloc agrees with ssa_decode.

ssa_decode_noalloc is for callers that cannot allocate device memory when they
call (their device memory belongs to an allocator they cannot reach, or their
serving loop may not call cudaMalloc, which can synchronise the device).  Its
scratch is one fixed array inside the library, shared by every call.  Two calls
in a row, on different inputs, must each give exactly what ssa_decode (which
takes a caller-allocated workspace) gives: both run the same kernels, and the
split-KV merge combines its partial records in a fixed order, so the results
are bitwise equal.  Any difference would mean a previous call's leftovers in
the shared array leaked into the next one.
This file is collected last so that a first-failure run has already run every
other test.
"""
import ctypes

import pytest
import torch

from workloads import planted_decode

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"


def _inputs(seed, seqlens):
    q, Kc, Vc, L = planted_decode(4, 16, 4, 64 * 96, 128, 64, clusters=6, seed=seed,
                                  dtype="bf16", seqlens=seqlens)
    return q.to(DEV), Kc.to(DEV), Vc.to(DEV), L.to(DEV)


def test_noalloc_matches_decode_on_two_calls_in_a_row():
    import block_sparse_top_summary_b200 as ssa
    cases = [(21, [64 * 96, 1000, 65, 3001]), (22, [17, 64 * 96, 64 * 50, 2])]
    for seed, seqlens in cases:
        q, Kc, Vc, L = _inputs(seed, seqlens)
        S = ssa.ssa_block_summary(Kc, 64)
        ref_o, ref_idx = ssa.ssa_decode(q, Kc, Vc, S, L, 64, 8)
        out, idx = ssa.ssa_decode_noalloc(q, Kc, Vc, S, L, 64, 8)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)
        assert torch.equal(out, ref_o)
        assert torch.isfinite(out.float()).all()
    assert ssa.ssa_device_error() == 0


def test_noalloc_rejects_sizes_beyond_its_array():
    import block_sparse_top_summary_b200 as ssa
    lib = ssa.load_library()
    fake = ctypes.c_void_p(0x100000)  # never dereferenced: the size check fails first
    need = ssa.ssa_decode_workspace_size(2048, 32, 8, 65536, 128, 64, 32)
    assert need > (40 << 20)
    fn = lib.ssa_decode_noalloc
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fn.argtypes = [vp, vp, vp, i, vp, vp, i, i, i, i, i, i, i, f, vp, vp, vp]
    fn.restype = i
    r = fn(fake, fake, fake, 1, fake, fake, 2048, 32, 8, 65536, 128, 64, 32,
           ctypes.c_float(0.088), fake, None, None)
    assert r == 2  # SSA_ERR_UNSUPPORTED
