"""Host-side checks of the C ABI that need no GPU.

The library must load, export every function include/ssa.h declares, and
reject bad arguments on the host before any launch (so these calls never touch
a device).
"""
import ctypes
import os
import re

import pytest

from block_sparse_top_summary_b200 import abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(ssa_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    return abi.load_library()


def test_every_declared_symbol_is_exported(lib):
    declared = _declared_functions()
    assert "ssa_route" in declared and "ssa_decode" in declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(abi.EXPORTS) == set(declared)


def test_status_strings_and_version(lib):
    assert lib.ssa_status_string(0) == b"SSA_OK"
    assert lib.ssa_status_string(4) == b"SSA_ERR_TIMEOUT"
    assert lib.ssa_status_string(99) == b"SSA_ERR_UNKNOWN"
    assert lib.ssa_version() >= 200


NULL = None
FAKE = ctypes.c_void_p(0x100000)  # never dereferenced: every call below fails a host check


def test_summary_rejects_bad_arguments(lib):
    assert lib.ssa_block_summary(NULL, 1, 1, 1, 128, 128, 64, FAKE, NULL) == 1  # null K
    assert lib.ssa_block_summary(FAKE, 1, 1, 1, 128, 96, 64, FAKE, NULL) == 2  # d=96
    assert lib.ssa_block_summary(FAKE, 1, 1, 1, 128, 128, 40, FAKE, NULL) == 2  # B % 16
    assert lib.ssa_block_summary(FAKE, 7, 1, 1, 128, 128, 64, FAKE, NULL) == 1  # dtype
    assert lib.ssa_block_summary(ctypes.c_void_p(0x100008), 1, 1, 1, 128, 128, 64, FAKE, NULL) == 1
    assert lib.ssa_block_summary(FAKE, 1, 1, 1, 32, 128, 64, FAKE, NULL) == 0  # N < B: no work


def test_route_rejects_bad_arguments(lib):
    args = dict(Q=FAKE, dt=1, S=FAKE, b=1, Hq=4, Hkv=2, N=1024, d=128, B=64, k=4, w=6,
                scores=NULL)

    def call(**kw):
        a = {**args, **kw}
        return lib.ssa_route(a["Q"], a["dt"], a["S"], a["b"], a["Hq"], a["Hkv"], a["N"], a["d"],
                             a["B"], a["k"], a["w"], FAKE, FAKE, a["scores"], NULL)

    assert call(Hq=5) == 1           # Hq % Hkv
    assert call(k=-1) == 1           # negative top-k
    assert call(w=5) == 1            # idx row too narrow for k + 2
    assert call(Q=NULL) == 1
    assert call(N=64 * 17000) == 2   # more query blocks than the kernel holds
    assert call(scores=ctypes.c_void_p(0x100004)) == 1  # scores not 16-byte aligned


def test_check_device_error_needs_an_output(lib):
    assert lib.ssa_check_device_error(NULL, NULL) == 1


def test_attn_rejects_bad_arguments(lib):
    def call(scale=0.088, **kw):
        a = dict(Q=FAKE, K=FAKE, V=FAKE, idx=FAKE, cnt=FAKE, O=FAKE)
        a.update(kw)
        return lib.ssa_sparse_attn_fwd(a["Q"], a["K"], a["V"], 1, a["idx"], a["cnt"], 1, 4, 2,
                                       1024, 128, 64, 6, ctypes.c_float(scale), a["O"], NULL, NULL)

    assert call(scale=0.0) == 1
    assert call(scale=-1.0) == 1
    assert call(V=NULL) == 1
    assert call(O=ctypes.c_void_p(0x100004)) == 1


def test_decode_workspace_and_rejections(lib):
    n = abi.ssa_decode_workspace_size(64, 32, 8, 65536, 128, 64, 32)
    assert n > 0 and n % 256 == 0
    # "all" blocks: the width is clipped to the cache's block count
    assert abi.ssa_decode_workspace_size(2, 4, 2, 1024, 64, 64, 1 << 30) < 1 << 20
    size = ctypes.c_size_t(n)
    r = lib.ssa_decode(FAKE, FAKE, FAKE, 1, FAKE, FAKE, 64, 32, 8, 65536, 128, 64, 32,
                       ctypes.c_float(0.088), FAKE, NULL, FAKE, ctypes.c_size_t(n - 1), NULL)
    assert r == 1  # workspace too small
    r = lib.ssa_decode(FAKE, FAKE, FAKE, 1, FAKE, FAKE, 64, 36, 4, 65536, 128, 64, 32,
                       ctypes.c_float(0.088), FAKE, NULL, FAKE, size, NULL)
    assert r == 2  # 9 query heads per KV head
    r = lib.ssa_decode(FAKE, FAKE, FAKE, 1, FAKE, FAKE, 64, 32, 8, 65536, 128, 64, 32,
                       ctypes.c_float(0.088), FAKE, NULL, ctypes.c_void_p(0x100010), size, NULL)
    assert r == 1  # workspace not 256-byte aligned


def test_decode_append_rejections(lib):
    fn = lib.ssa_decode_append
    ok = (FAKE, FAKE, 1, FAKE, FAKE, FAKE, FAKE, 4, 2, 1024, 128, 64, NULL)

    def call(**kw):
        args = list(ok)
        for k, v in kw.items():
            args[{"Kc": 0, "Vc": 1, "dt": 2, "S": 3, "L": 4, "kn": 5, "vn": 6, "batch": 7,
                  "Hkv": 8, "Lmax": 9, "d": 10, "B": 11}[k]] = v
        return fn(*args)

    assert call(d=96) == 2                   # d not 64 or 128
    assert call(B=40) == 2                   # B not a multiple of 16
    assert call(dt=7) == 1                   # unknown dtype
    assert call(batch=0) == 1
    assert call(Lmax=0) == 1
    assert call(Kc=NULL) == 1
    assert call(L=NULL) == 1
    assert call(S=NULL) == 1                 # the cache holds complete blocks
    assert call(kn=ctypes.c_void_p(0x100008)) == 1  # not 16-byte aligned


def test_attention_backward_rejections(lib):
    fn = lib.ssa_sparse_attn_bwd
    names = ["Q", "K", "V", "O", "dO", "lse", "dt", "idx", "cnt", "batch", "Hq", "Hkv", "N", "d",
             "B", "max_sel", "scale", "dQ", "dK", "dV", "ws", "ws_bytes", "stream"]
    need = abi.ssa_sparse_attn_bwd_workspace_size(1, 8, 2, 4096, 128, 64)
    ok = [FAKE] * 6 + [1, FAKE, FAKE, 1, 8, 2, 4096, 128, 64, 18, 0.088, FAKE, FAKE, FAKE, FAKE,
                       need, NULL]

    def call(**kw):
        args = list(ok)
        for k, v in kw.items():
            args[names.index(k)] = v
        return fn(*args)

    assert call(dt=0) == 2                   # fp32: not implemented
    assert call(dt=7) == 1                   # unknown dtype
    assert call(d=96) == 2
    assert call(B=40) == 2
    assert call(Hq=6, Hkv=4) == 1            # Hq not a multiple of Hkv
    assert call(N=0) == 1
    assert call(max_sel=0) == 1
    assert call(scale=0.0) == 1
    for name in ("Q", "K", "V", "O", "dO", "lse", "idx", "cnt", "dQ", "dK", "dV", "ws"):
        assert call(**{name: NULL}) == 1, name
    assert call(dK=ctypes.c_void_p(0x100008)) == 1  # not 16-byte aligned
    assert call(ws=ctypes.c_void_p(0x100010)) == 1  # workspace not 256-byte aligned
    assert call(ws_bytes=need - 1) == 1             # workspace too small
    # delta for every query row, then the sink block's partial sums
    assert need >= 1 * 8 * 4096 * 4 + 1 * 2 * 2 * 64 * 128 * 4


def test_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(ImportError):
        abi.load_library(str(tmp_path / "missing.so"))
