"""Oracle work for the full-size parity tests, spread over worker processes.

Test infrastructure only.  The fp64 oracle runs one work unit per process: one
KV head of a prefill workload, or one sequence of the decode workload.  The
pool uses the spawn start method, so no worker inherits the parent's CUDA
context.  Tensors travel as raw bf16 bits (int16) or float32 and are widened
to float64 exactly in the worker.  Each worker compares the GPU's outputs
with the oracle's and returns error sums, so no full-size float64 output
crosses back.
"""
from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np
import torch

import oracle as O
from parity import compare_selection


def make_pool(n_tasks: int):
    """A spawn pool with at most one worker per task and per two host cores."""
    cores = len(os.sched_getaffinity(0))
    return mp.get_context("spawn").Pool(max(1, min(n_tasks, cores // 2 or 1, 16)))


def pack(t: torch.Tensor):
    """Host copy of a tensor as (kind, array): bf16 as its int16 bits."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return ("bf16", t.view(torch.int16).numpy())
    return ("raw", t.numpy())


def unpack(p) -> np.ndarray:
    """Exact float64 value of a packed tensor."""
    kind, a = p
    if kind == "bf16":
        return (a.astype(np.int32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


def _err_sums(gpu: np.ndarray, ref: np.ndarray):
    d = gpu - ref
    return (float(np.sum(d * d)), float(np.sum(ref * ref)),
            float(np.max(np.abs(d))) if d.size else 0.0, int(d.size))


def prefill_head(task):
    """Oracle attention of every query block of one (batch, KV head), on the
    GPU's selection, against the GPU's O and LSE.  Returns error sums."""
    Qp, Kp, Vp, idx, cnt, B, Op, lsep, units = task
    Q, K, V = unpack(Qp), unpack(Kp), unpack(Vp)
    out, lse = unpack(Op), unpack(lsep)
    if units is None:
        ref, rlse = O.sparse_attention(Q, K, V, idx, cnt, B)
        o_sums = _err_sums(out.ravel(), ref.ravel())
        l_max = float(np.max(np.abs(lse - rlse)))
        return o_sums, l_max
    ref, rlse = O.sparse_attention(Q, K, V, idx, cnt, B, units=[(0, 0, i) for i in units])
    N = Q.shape[2]
    rows = np.concatenate([np.arange(i * B, min(N, (i + 1) * B)) for i in units])
    o_sums = _err_sums(out[:, :, rows].ravel(), ref[:, :, rows].ravel())
    l_max = float(np.max(np.abs(lse[:, :, rows] - rlse[:, :, rows])))
    return o_sums, l_max


def decode_sequence(task):
    """Oracle routing and attention of one decode sequence.

    The oracle recomputes the sequence's block summaries in float64 from the
    cache, routes, and compares its selection with the GPU's (near-ties
    counted); the attention is then recomputed on the GPU's selection and
    compared with the GPU's O.  Returns ``(rows, near, bad, err_sums)``.
    """
    qp, Kp, Vp, L, B, topk, gi, Op = task
    q, Kc, Vc, out = unpack(qp), unpack(Kp), unpack(Vp), unpack(Op)
    Ls = np.array([L])
    S = O.block_summary(Kc, B)
    oi, oc, osc = O.decode_route(q, S, Ls, B, topk)
    gc = (gi >= 0).sum(-1)
    rows, near, bad = compare_selection(gi, gc, oi, oc,
                                        lambda r: {j: osc[r][j] for j in range(osc.shape[-1])})
    ref, _, _, _ = O.decode(q, Kc, Vc, Ls, B, topk, idx=gi, cnt=gc)
    return rows, near, [(tuple(int(x) for x in r), g, o) for r, g, o in bad], \
        _err_sums(out.ravel(), ref.ravel())


def combine(sums):
    """(max-abs, relative-L2) over several error sums."""
    dd = sum(s[0] for s in sums)
    rr = sum(s[1] for s in sums)
    ma = max(s[2] for s in sums)
    return ma, float(np.sqrt(dd / rr)) if rr > 0 else float(np.sqrt(dd))
