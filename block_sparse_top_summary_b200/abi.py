"""ctypes binding of ``libssa.so`` (argument marshalling only).

Every function here has the name of the C entry point it calls, takes torch
CUDA tensors, passes their device pointers and the current CUDA stream, and
raises ``SSAError`` on a non-OK status.  Outputs that the caller does not
pass are allocated with torch (device memory is torch's job; the library
allocates nothing).  No step of the method runs here.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libssa.so")

SSA_F32 = 0
SSA_BF16 = 1

_STATUS = {0: "SSA_OK", 1: "SSA_ERR_INVALID_ARG", 2: "SSA_ERR_UNSUPPORTED", 3: "SSA_ERR_CUDA",
           4: "SSA_ERR_TIMEOUT"}

# Every symbol include/ssa.h and include/ssa_debug.h declare.
EXPORTS = ("ssa_status_string", "ssa_version", "ssa_block_summary", "ssa_route",
           "ssa_sparse_attn_fwd", "ssa_sparse_attn_bwd", "ssa_sparse_attn_uses_tensor_cores",
           "ssa_decode_workspace_size", "ssa_decode", "ssa_decode_append", "ssa_decode_noalloc",
           "ssa_decode_paged", "ssa_decode_append_paged", "ssa_learned_summary",
           "ssa_route_entmax", "ssa_sparse_attn_fwd_prior", "ssa_route_hierarchical",
           "ssa_decode_per_head", "ssa_decode_per_head_workspace_size",
           "ssa_sparse_attn_bwd_workspace_size",
           "ssa_device_error", "ssa_check_device_error", "ssa_debug_wait_timeout")


class SSAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {_STATUS.get(status, status)}")
        self.status = status


_lib = None


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load (once) and return the library.  Raises if it was not built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or _LIB_PATH
    if not os.path.exists(p):
        raise ImportError(
            f"libssa.so not found at {p}: build it with "
            "`python -m block_sparse_top_summary_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(p)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.ssa_status_string.restype = ctypes.c_char_p
    lib.ssa_status_string.argtypes = [i]
    lib.ssa_version.restype = i
    lib.ssa_block_summary.argtypes = [vp, i, i, i, i, i, i, vp, vp]
    lib.ssa_route.argtypes = [vp, i, vp, i, i, i, i, i, i, i, i, vp, vp, vp, vp]
    lib.ssa_sparse_attn_fwd.argtypes = [vp, vp, vp, i, vp, vp, i, i, i, i, i, i, i, f, vp, vp, vp]
    lib.ssa_decode_workspace_size.argtypes = [i, i, i, i, i, i, i, ctypes.POINTER(sz)]
    lib.ssa_decode.argtypes = [vp, vp, vp, i, vp, vp, i, i, i, i, i, i, i, f, vp, vp, vp, sz, vp]
    lib.ssa_device_error.argtypes = [ctypes.POINTER(i)]
    lib.ssa_check_device_error.argtypes = [vp, ctypes.POINTER(i)]
    lib.ssa_decode_noalloc.argtypes = [vp, vp, vp, i, vp, vp, i, i, i, i, i, i, i, f, vp, vp, vp]
    lib.ssa_decode_append.argtypes = [vp, vp, i, vp, vp, vp, vp, i, i, i, i, i, vp]
    lib.ssa_sparse_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, i, vp, vp, i, i, i, i, i, i, i, f,
                                        vp, vp, vp, vp, sz, vp]
    lib.ssa_sparse_attn_bwd_workspace_size.argtypes = [i, i, i, i, i, i, ctypes.POINTER(sz)]
    lib.ssa_debug_wait_timeout.argtypes = [i, vp]
    lib.ssa_decode_paged.argtypes = [vp, vp, vp, i, vp, vp, i, i, vp, i, i, i, i, i, i, f, vp, vp,
                                     vp, sz, vp]
    lib.ssa_decode_append_paged.argtypes = [vp, vp, i, vp, vp, i, i, vp, vp, vp, i, i, i, i, vp]
    lib.ssa_learned_summary.argtypes = [vp, i, vp, i, i, i, i, i, vp, vp]
    lib.ssa_route_hierarchical.argtypes = [vp, i, vp, i, i, i, i, i, i, i, i, i, i, vp, vp, vp]
    lib.ssa_decode_per_head_workspace_size.argtypes = [i, i, i, i, i, i, i, ctypes.POINTER(sz)]
    lib.ssa_decode_per_head.argtypes = [vp, vp, vp, i, vp, vp, i, i, i, i, i, i, i, f, vp, vp, vp,
                                        sz, vp]
    lib.ssa_route_entmax.argtypes = [vp, i, vp, i, i, i, i, i, i, f, f, f, i, vp, vp, vp, vp, vp]
    lib.ssa_sparse_attn_fwd_prior.argtypes = [vp, vp, vp, i, vp, vp, vp, i, i, i, i, i, i, i, f,
                                              vp, vp, vp]
    lib.ssa_sparse_attn_uses_tensor_cores.argtypes = [i, i, i, i, i]
    for name in EXPORTS:
        if name not in ("ssa_status_string", "ssa_version"):
            getattr(lib, name).restype = i
    if path is None:
        _lib = lib
    return lib


def _check(fn: str, status: int):
    if status != 0:
        raise SSAError(fn, status)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SSA_F32
    if t.dtype == torch.bfloat16:
        return SSA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def ssa_block_summary(K: torch.Tensor, B: int, S: torch.Tensor | None = None, stream=None):
    """Block mean summaries ``S`` ``[batch, Hkv, N // B, d]`` fp32 of ``K``."""
    _need(K, "K")
    batch, Hkv, N, d = K.shape
    if S is None:
        S = torch.empty(batch, Hkv, N // B, d, dtype=torch.float32, device=K.device)
    _check("ssa_block_summary", load_library().ssa_block_summary(
        _ptr(K), _dtype_code(K), batch, Hkv, N, d, B, _ptr(S), _stream(stream)))
    return S


def route_width(N: int, B: int, topk: int) -> int:
    """Smallest idx row width for ssa_route."""
    nq = -(-N // B)
    return min(topk, max(nq - 2, 0)) + 2


def ssa_route(Q: torch.Tensor, S: torch.Tensor, B: int, topk: int, Hkv: int,
              max_sel: int | None = None, idx=None, cnt=None, scores=None,
              want_scores: bool = False, stream=None):
    """Top-k routing per (batch, KV head, query block): returns ``(idx, cnt)``,
    or ``(idx, cnt, scores)`` when ``scores`` is given or ``want_scores`` is set
    (``scores``: ``[batch, Hkv, nq, N // B]`` fp32, -inf off the candidates)."""
    _need(Q, "Q")
    batch, Hq, N, d = Q.shape
    nq = -(-N // B)
    if max_sel is None:
        max_sel = route_width(N, B, topk)
    if idx is None:
        idx = torch.empty(batch, Hkv, nq, max_sel, dtype=torch.int32, device=Q.device)
    if cnt is None:
        cnt = torch.empty(batch, Hkv, nq, dtype=torch.int32, device=Q.device)
    ret_scores = scores is not None or want_scores
    if scores is None and want_scores:
        scores = torch.empty(batch, Hkv, nq, N // B, dtype=torch.float32, device=Q.device)
    if scores is not None:
        _need(scores, "scores")
    _check("ssa_route", load_library().ssa_route(
        _ptr(Q), _dtype_code(Q), _ptr(S), batch, Hq, Hkv, N, d, B, topk, max_sel, _ptr(idx),
        _ptr(cnt), _ptr(scores), _stream(stream)))
    return (idx, cnt, scores) if ret_scores else (idx, cnt)


def ssa_sparse_attn_fwd(Q, K, V, idx, cnt, B: int, scale: float | None = None, O=None, lse=None,
                        want_lse: bool = True, stream=None):
    """Attention over the selected blocks: returns ``(O, lse)`` (``lse`` may be None)."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V"), (idx, "idx"), (cnt, "cnt")):
        _need(t, n)
    batch, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty(batch, Hq, N, dtype=torch.float32, device=Q.device)
    _check("ssa_sparse_attn_fwd", load_library().ssa_sparse_attn_fwd(
        _ptr(Q), _ptr(K), _ptr(V), _dtype_code(Q), _ptr(idx), _ptr(cnt), batch, Hq, Hkv, N, d, B,
        idx.shape[-1], ctypes.c_float(scale), _ptr(O), _ptr(lse), _stream(stream)))
    return O, lse


def ssa_sparse_attn_uses_tensor_cores(dtype: torch.dtype, Hq: int, Hkv: int, d: int,
                                      B: int) -> bool:
    code = SSA_BF16 if dtype == torch.bfloat16 else SSA_F32
    return bool(load_library().ssa_sparse_attn_uses_tensor_cores(code, Hq, Hkv, d, B))


def ssa_decode_workspace_size(batch: int, Hq: int, Hkv: int, Lmax: int, d: int, B: int,
                              topk: int) -> int:
    n = ctypes.c_size_t(0)
    _check("ssa_decode_workspace_size", load_library().ssa_decode_workspace_size(
        batch, Hq, Hkv, Lmax, d, B, topk, ctypes.byref(n)))
    return n.value


def decode_width(Lmax: int, B: int, topk: int) -> int:
    return min(topk, -(-Lmax // B)) + 2


def ssa_decode(q, Kc, Vc, S, seqlens, B: int, topk: int, scale: float | None = None, O=None,
               idx=None, want_idx: bool = True, workspace=None, stream=None):
    """One decode step: returns ``(O, idx)`` (``idx`` None unless wanted)."""
    for t, n in ((q, "q"), (Kc, "Kc"), (Vc, "Vc"), (seqlens, "seqlens")):
        _need(t, n)
    batch, Hq, d = q.shape
    Hkv, Lmax = Kc.shape[1], Kc.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(q)
    if idx is None and want_idx:
        idx = torch.empty(batch, Hkv, decode_width(Lmax, B, topk), dtype=torch.int32,
                          device=q.device)
    ws_bytes = ssa_decode_workspace_size(batch, Hq, Hkv, Lmax, d, B, topk)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    _check("ssa_decode", load_library().ssa_decode(
        _ptr(q), _ptr(Kc), _ptr(Vc), _dtype_code(q), _ptr(S), _ptr(seqlens), batch, Hq, Hkv, Lmax,
        d, B, topk, ctypes.c_float(scale), _ptr(O), _ptr(idx), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return O, idx


def ssa_device_error() -> int:
    """Synchronise, then read and reset the device-side error word."""
    code = ctypes.c_int(0)
    _check("ssa_device_error", load_library().ssa_device_error(ctypes.byref(code)))
    return code.value


def ssa_check_device_error(stream=None) -> int:
    """Read and reset the device-side error word in the order of ``stream``,
    waiting for that stream only."""
    code = ctypes.c_int(0)
    _check("ssa_check_device_error", load_library().ssa_check_device_error(
        _stream(stream), ctypes.byref(code)))
    return code.value


def prefill(Q, K, V, B: int, topk: int, scale: float | None = None, stream=None):
    """The three prefill calls in order: summary, route, attention.

    Returns ``(O, lse, idx, cnt, S)``.
    """
    S = ssa_block_summary(K, B, stream=stream)
    idx, cnt = ssa_route(Q, S, B, topk, K.shape[1], stream=stream)
    O, lse = ssa_sparse_attn_fwd(Q, K, V, idx, cnt, B, scale=scale, stream=stream)
    return O, lse, idx, cnt, S


def ssa_decode_noalloc(q, Kc, Vc, S, seqlens, B: int, topk: int, scale: float | None = None,
                       O=None, idx=None, want_idx: bool = True, stream=None):
    """ssa_decode with the library's fixed scratch array instead of a workspace.

    For callers that cannot allocate device memory at call time.  Returns
    ``(O, idx)`` like ``ssa_decode``.
    """
    for t, n in ((q, "q"), (Kc, "Kc"), (Vc, "Vc"), (seqlens, "seqlens")):
        _need(t, n)
    fn = load_library().ssa_decode_noalloc
    batch, Hq, d = q.shape
    Hkv, Lmax = Kc.shape[1], Kc.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(q)
    if idx is None and want_idx:
        idx = torch.empty(batch, Hkv, decode_width(Lmax, B, topk), dtype=torch.int32,
                          device=q.device)
    _check("ssa_decode_noalloc", fn(
        _ptr(q), _ptr(Kc), _ptr(Vc), _dtype_code(q), _ptr(S), _ptr(seqlens), batch, Hq, Hkv, Lmax,
        d, B, topk, ctypes.c_float(scale), _ptr(O), _ptr(idx), _stream(stream)))
    return O, idx


def ssa_decode_append(Kc, Vc, S, seqlens, k_new, v_new, B: int, stream=None):
    """Append one token per sequence to the cache, in place.

    Writes ``k_new`` / ``v_new`` ``[batch, Hkv, d]`` at each sequence's length,
    raises ``seqlens`` by one and refreshes the summary ``S`` of a block the
    append completes.  Sequences whose cache is full are left unchanged.
    """
    for t, n in ((Kc, "Kc"), (Vc, "Vc"), (S, "S"), (seqlens, "seqlens"), (k_new, "k_new"),
                 (v_new, "v_new")):
        _need(t, n)
    fn = load_library().ssa_decode_append
    batch, Hkv, Lmax, d = Kc.shape
    _check("ssa_decode_append", fn(
        _ptr(Kc), _ptr(Vc), _dtype_code(Kc), _ptr(S), _ptr(seqlens), _ptr(k_new), _ptr(v_new),
        batch, Hkv, Lmax, d, B, _stream(stream)))
    return Kc, Vc, S, seqlens


def ssa_decode_paged(q, Kp, Vp, S, page_table, seqlens, B: int, topk: int,
                     scale: float | None = None, O=None, idx=None, want_idx: bool = True,
                     workspace=None, stream=None):
    """One decode step over a paged cache: returns ``(O, idx)``.

    ``Kp``/``Vp``: page pools ``[num_pages, Hkv, B, d]``; ``page_table``:
    ``[batch, max_blocks]`` int32 (-1: no page); ``S``: ``[batch, Hkv,
    max_blocks, d]`` fp32 summaries in logical block order.
    """
    for t, n in ((q, "q"), (Kp, "Kp"), (Vp, "Vp"), (S, "S"), (page_table, "page_table"),
                 (seqlens, "seqlens")):
        _need(t, n)
    batch, Hq, d = q.shape
    num_pages, Hkv = Kp.shape[0], Kp.shape[1]
    max_blocks = page_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(q)
    if idx is None and want_idx:
        idx = torch.empty(batch, Hkv, decode_width(max_blocks * B, B, topk), dtype=torch.int32,
                          device=q.device)
    nbytes = ssa_decode_workspace_size(batch, Hq, Hkv, max_blocks * B, d, B, topk)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    _check("ssa_decode_paged", load_library().ssa_decode_paged(
        _ptr(q), _ptr(Kp), _ptr(Vp), _dtype_code(q), _ptr(S), _ptr(page_table), max_blocks,
        num_pages, _ptr(seqlens), batch, Hq, Hkv, d, B, topk, ctypes.c_float(scale), _ptr(O),
        _ptr(idx), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    return O, idx


def ssa_decode_append_paged(Kp, Vp, S, page_table, seqlens, k_new, v_new, B: int, stream=None):
    """Append one token per sequence to a paged cache, in place (the row goes
    to row ``L % B`` of page ``page_table[b, L // B]``; a sequence whose next
    block has no page is left unchanged)."""
    for t, n in ((Kp, "Kp"), (Vp, "Vp"), (S, "S"), (page_table, "page_table"),
                 (seqlens, "seqlens"), (k_new, "k_new"), (v_new, "v_new")):
        _need(t, n)
    num_pages, Hkv, _, d = Kp.shape
    batch, max_blocks = page_table.shape
    _check("ssa_decode_append_paged", load_library().ssa_decode_append_paged(
        _ptr(Kp), _ptr(Vp), _dtype_code(Kp), _ptr(S), _ptr(page_table), max_blocks, num_pages,
        _ptr(seqlens), _ptr(k_new), _ptr(v_new), batch, Hkv, d, B, _stream(stream)))
    return Kp, Vp, S, seqlens


def ssa_learned_summary(K, qbar, B: int, S=None, stream=None):
    """Learned block summaries ``[batch, Hkv, N // B, d]`` fp32 (DashAttention's
    stage 0); ``qbar``: ``[Hkv, d]`` fp32, one learned query per KV head."""
    _need(K, "K")
    _need(qbar, "qbar")
    batch, Hkv, N, d = K.shape
    if S is None:
        S = torch.empty(batch, Hkv, N // B, d, dtype=torch.float32, device=K.device)
    _check("ssa_learned_summary", load_library().ssa_learned_summary(
        _ptr(K), _dtype_code(K), _ptr(qbar), batch, Hkv, N, d, B, _ptr(S), _stream(stream)))
    return S


def entmax_width(N: int, B: int) -> int:
    """Row width of ssa_route_entmax's idx / bias: every candidate + the diagonal."""
    nq, nfull = -(-N // B), N // B
    return min(nq - 1, nfull) + 1


def ssa_route_entmax(Q, S, B: int, Hkv: int, alpha: float, gamma: float, sigma: float,
                     want_w: bool = False, stream=None):
    """alpha-entmax routing (DashAttention's stage 1): returns ``(idx, cnt, bias,
    w)``; ``w`` (``[batch, Hkv, nq, N // B]``) is None unless wanted."""
    _need(Q, "Q")
    batch, Hq, N, d = Q.shape
    nq, nfull = -(-N // B), N // B
    width = entmax_width(N, B)
    idx = torch.empty(batch, Hkv, nq, width, dtype=torch.int32, device=Q.device)
    cnt = torch.empty(batch, Hkv, nq, dtype=torch.int32, device=Q.device)
    bias = torch.empty(batch, Hkv, nq, width, dtype=torch.float32, device=Q.device)
    w = torch.empty(batch, Hkv, nq, nfull, dtype=torch.float32, device=Q.device) if want_w else None
    _check("ssa_route_entmax", load_library().ssa_route_entmax(
        _ptr(Q), _dtype_code(Q), _ptr(S), batch, Hq, Hkv, N, d, B, ctypes.c_float(alpha),
        ctypes.c_float(gamma), ctypes.c_float(sigma), width, _ptr(idx), _ptr(cnt), _ptr(bias),
        _ptr(w), _stream(stream)))
    return idx, cnt, bias, w


def ssa_sparse_attn_fwd_prior(Q, K, V, idx, cnt, bias, B: int, scale: float | None = None,
                              O=None, lse=None, stream=None):
    """Attention with the routing prior (DashAttention's stage 2): returns
    ``(O, lse)``."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V"), (idx, "idx"), (cnt, "cnt"), (bias, "bias")):
        _need(t, n)
    batch, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None:
        lse = torch.empty(batch, Hq, N, dtype=torch.float32, device=Q.device)
    _check("ssa_sparse_attn_fwd_prior", load_library().ssa_sparse_attn_fwd_prior(
        _ptr(Q), _ptr(K), _ptr(V), _dtype_code(Q), _ptr(idx), _ptr(cnt), _ptr(bias), batch, Hq,
        Hkv, N, d, B, idx.shape[-1], ctypes.c_float(scale), _ptr(O), _ptr(lse), _stream(stream)))
    return O, lse


def ssa_route_hierarchical(Q, S, B: int, M: int, k_seg: int, k_blk: int, Hkv: int,
                           idx=None, cnt=None, stream=None):
    """Two-level routing (segments of ``M`` blocks, then blocks): returns
    ``(idx, cnt)`` in the layout of ``ssa_route``."""
    _need(Q, "Q")
    batch, Hq, N, d = Q.shape
    nq = -(-N // B)
    width = min(k_blk, nq) + 2
    if idx is None:
        idx = torch.empty(batch, Hkv, nq, width, dtype=torch.int32, device=Q.device)
    if cnt is None:
        cnt = torch.empty(batch, Hkv, nq, dtype=torch.int32, device=Q.device)
    _check("ssa_route_hierarchical", load_library().ssa_route_hierarchical(
        _ptr(Q), _dtype_code(Q), _ptr(S), batch, Hq, Hkv, N, d, B, M, k_seg, k_blk,
        idx.shape[-1], _ptr(idx), _ptr(cnt), _stream(stream)))
    return idx, cnt


def ssa_decode_per_head_workspace_size(batch: int, Hq: int, Hkv: int, Lmax: int, d: int, B: int,
                                       topk: int) -> int:
    n = ctypes.c_size_t(0)
    _check("ssa_decode_per_head_workspace_size",
           load_library().ssa_decode_per_head_workspace_size(batch, Hq, Hkv, Lmax, d, B, topk,
                                                             ctypes.byref(n)))
    return n.value


def ssa_decode_per_head(q, Kc, Vc, S, seqlens, B: int, topk: int, scale: float | None = None,
                        O=None, idx=None, want_idx: bool = True, workspace=None, stream=None):
    """Decode with one block selection per query head: returns ``(O, idx)``,
    ``idx`` ``[batch, Hq, width]``."""
    for t, n in ((q, "q"), (Kc, "Kc"), (Vc, "Vc"), (seqlens, "seqlens")):
        _need(t, n)
    batch, Hq, d = q.shape
    Hkv, Lmax = Kc.shape[1], Kc.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(q)
    if idx is None and want_idx:
        idx = torch.empty(batch, Hq, decode_width(Lmax, B, topk), dtype=torch.int32,
                          device=q.device)
    nbytes = ssa_decode_per_head_workspace_size(batch, Hq, Hkv, Lmax, d, B, topk)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    _check("ssa_decode_per_head", load_library().ssa_decode_per_head(
        _ptr(q), _ptr(Kc), _ptr(Vc), _dtype_code(q), _ptr(S), _ptr(seqlens), batch, Hq, Hkv, Lmax,
        d, B, topk, ctypes.c_float(scale), _ptr(O), _ptr(idx), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return O, idx


def ssa_sparse_attn_bwd_workspace_size(batch: int, Hq: int, Hkv: int, N: int, d: int,
                                       B: int) -> int:
    n = ctypes.c_size_t(0)
    _check("ssa_sparse_attn_bwd_workspace_size",
           load_library().ssa_sparse_attn_bwd_workspace_size(batch, Hq, Hkv, N, d, B,
                                                            ctypes.byref(n)))
    return n.value


def ssa_sparse_attn_bwd(Q, K, V, O, dO, lse, idx, cnt, B: int, scale: float | None = None,
                        dQ=None, dK=None, dV=None, workspace=None, stream=None):
    """Gradients of the selected-block attention: returns ``(dQ, dK, dV)``.

    ``O`` and ``lse`` are the outputs of ``ssa_sparse_attn_fwd`` on the same
    ``Q, K, V, idx, cnt``; ``dO`` is the gradient of the loss with respect to
    ``O``.  ``workspace`` (uint8, ``ssa_sparse_attn_bwd_workspace_size`` bytes)
    is scratch.
    """
    for t, n in ((Q, "Q"), (K, "K"), (V, "V"), (O, "O"), (dO, "dO"), (lse, "lse"), (idx, "idx"),
                 (cnt, "cnt")):
        _need(t, n)
    batch, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dQ = torch.empty_like(Q) if dQ is None else dQ
    dK = torch.empty_like(K) if dK is None else dK
    dV = torch.empty_like(V) if dV is None else dV
    if workspace is None:
        workspace = torch.empty(ssa_sparse_attn_bwd_workspace_size(batch, Hq, Hkv, N, d, B),
                                dtype=torch.uint8, device=Q.device)
    _check("ssa_sparse_attn_bwd", load_library().ssa_sparse_attn_bwd(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(lse), _dtype_code(Q), _ptr(idx),
        _ptr(cnt), batch, Hq, Hkv, N, d, B, idx.shape[-1], ctypes.c_float(scale), _ptr(dQ),
        _ptr(dK), _ptr(dV), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    return dQ, dK, dV


# ------------------------------------------------------------- test hooks
def ssa_debug_wait_timeout(limit_us: int, stream=None):
    """Run the bounded-wait self-test (include/ssa_debug.h); read the result with
    ssa_device_error()."""
    fn = load_library().ssa_debug_wait_timeout
    _check("ssa_debug_wait_timeout", fn(limit_us, _stream(stream)))
