"""Seeded synthetic inputs for block-sparse attention with top-k summary routing.

This module is shared by the CPU oracle's tests, the GPU parity tests and the
benchmark.  It only draws random tensors and describes workload shapes: it holds
none of the method's arithmetic (no summaries, scores, selection or softmax).

Recipe ("planted clusters"), drawn from one ``torch.Generator`` in a fixed order:

1. ``V ~ N(0, 1)``, shape ``[batch, Hkv, N, d]``.
2. ``K ~ N(0, 1)`` plus, per (batch, KV head), ``C`` Gaussian directions scaled
   to norm 4.  Every key block ``j >= 1`` draws one cluster id uniformly and
   the scaled direction is added to each of its rows.  Block 0 (the sink)
   carries no cluster.
3. ``Q ~ N(0, 1)``, shape ``[batch, Hq, N, d]``, plus, per (batch, KV head,
   query block), one uniformly drawn cluster direction added to every row of
   every query head of that KV head's group.

With ``C == 0`` the tensors are plain ``N(0, 1)``.  Values are drawn in fp32
and rounded once to the storage dtype, so every consumer sees identical bytes.
The workloads stand in for the long-context LLM runs of the pages (16K-128K
tokens, GQA) whose models and datasets are not available here.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

__all__ = [
    "PrefillConfig",
    "DecodeConfig",
    "CONFIGS",
    "planted_prefill",
    "planted_decode",
    "upstream_grad",
    "to_f64",
]


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    batch: int
    Hq: int
    Hkv: int
    N: int
    d: int
    B: int
    topk: int
    dtype: str  # "f32" | "bf16"
    clusters: int
    seed: int = 0
    topk_sweep: tuple = field(default_factory=tuple)


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    batch: int
    Hq: int
    Hkv: int
    L: int
    d: int
    B: int
    topk: int
    dtype: str
    clusters: int
    seed: int = 0


# topk value that means "every candidate block" (any value >= number of blocks).
TOPK_ALL = 1 << 30

CONFIGS = {
    "tiny": PrefillConfig("tiny", 1, 2, 1, 1024, 64, 64, 4, "f32", 0),
    "prefill32k": PrefillConfig("prefill32k", 1, 32, 8, 32768, 128, 64, 16, "bf16", 16),
    "prefill128k": PrefillConfig("prefill128k", 1, 32, 8, 131072, 128, 64, 32, "bf16", 64),
    "decode": DecodeConfig("decode", 64, 32, 8, 65536, 128, 64, 32, "bf16", 16),
    "sweep": PrefillConfig("sweep", 2, 16, 4, 65536, 128, 128, 4, "bf16", 8,
                           topk_sweep=(4, 8, 16, 32, 64, TOPK_ALL)),
}


def _torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _unit_dirs(gen, shape, d, device):
    u = torch.randn(*shape, d, generator=gen, device=device)
    return u / u.norm(dim=-1, keepdim=True) * 4.0


def planted_prefill(batch, Hq, Hkv, N, d, B, clusters, seed=0, dtype="bf16", device="cpu"):
    """Return ``(Q, K, V)`` in BHND layout (``[batch, heads, N, d]``, contiguous).

    ``device`` selects where (and with which generator) the values are drawn;
    CPU and CUDA generators give different streams for the same seed.
    """
    assert Hq % Hkv == 0
    G = Hq // Hkv
    nb = -(-N // B)
    Np = nb * B
    gen = torch.Generator(device=device).manual_seed(seed)
    V = torch.randn(batch, Hkv, N, d, generator=gen, device=device)
    K = torch.randn(batch, Hkv, Np, d, generator=gen, device=device)
    if clusters > 0:
        U = _unit_dirs(gen, (batch, Hkv, clusters), d, device)
        kid = torch.randint(0, clusters, (batch, Hkv, nb), generator=gen, device=device)
        add = torch.gather(U, 2, kid[..., None].expand(batch, Hkv, nb, d))
        add[:, :, 0] = 0.0
        K.view(batch, Hkv, nb, B, d).add_(add[:, :, :, None, :])
    K = K[:, :, :N]
    Q = torch.randn(batch, Hq, Np, d, generator=gen, device=device)
    if clusters > 0:
        qid = torch.randint(0, clusters, (batch, Hkv, nb), generator=gen, device=device)
        addq = torch.gather(U, 2, qid[..., None].expand(batch, Hkv, nb, d))
        Q.view(batch, Hkv, G, nb, B, d).add_(addq[:, :, None, :, None, :])
    Q = Q[:, :, :N]
    t = _torch_dtype(dtype)
    return (Q.to(t).contiguous(), K.to(t).contiguous(), V.to(t).contiguous())


def planted_decode(batch, Hq, Hkv, Lmax, d, B, clusters, seed=0, dtype="bf16",
                   device="cpu", seqlens=None):
    """Return ``(q, Kc, Vc, seqlens)`` for one decode step.

    ``q``: ``[batch, Hq, d]``; caches ``Kc, Vc``: ``[batch, Hkv, Lmax, d]``;
    ``seqlens``: int32 ``[batch]`` (default: every sequence full, ``Lmax``).
    The caches are drawn one sequence at a time to bound temporary memory.
    Each (sequence, KV head) query draws one cluster direction, added to the
    ``q`` of every head of its group.
    """
    assert Hq % Hkv == 0
    G = Hq // Hkv
    nb = -(-Lmax // B)
    Lp = nb * B
    t = _torch_dtype(dtype)
    gen = torch.Generator(device=device).manual_seed(seed)
    Vc = torch.empty(batch, Hkv, Lmax, d, dtype=t, device=device)
    Kc = torch.empty(batch, Hkv, Lmax, d, dtype=t, device=device)
    for b in range(batch):
        Vc[b] = torch.randn(Hkv, Lmax, d, generator=gen, device=device).to(t)
    U = None
    if clusters > 0:
        U = _unit_dirs(gen, (batch, Hkv, clusters), d, device)
    for b in range(batch):
        kb = torch.randn(Hkv, Lp, d, generator=gen, device=device)
        if clusters > 0:
            kid = torch.randint(0, clusters, (Hkv, nb), generator=gen, device=device)
            add = torch.gather(U[b], 1, kid[..., None].expand(Hkv, nb, d))
            add[:, 0] = 0.0
            kb.view(Hkv, nb, B, d).add_(add[:, :, None, :])
        Kc[b] = kb[:, :Lmax].to(t)
    q = torch.randn(batch, Hq, d, generator=gen, device=device)
    if clusters > 0:
        qid = torch.randint(0, clusters, (batch, Hkv), generator=gen, device=device)
        addq = torch.gather(U, 2, qid[..., None, None].expand(batch, Hkv, 1, d))[:, :, 0]
        q.view(batch, Hkv, G, d).add_(addq[:, :, None, :])
    if seqlens is None:
        seqlens = torch.full((batch,), Lmax, dtype=torch.int32)
    seqlens = torch.as_tensor(seqlens, dtype=torch.int32).to(device)
    return q.to(t).contiguous(), Kc, Vc, seqlens


def upstream_grad(batch, Hq, N, d, seed=0, dtype="bf16", device="cpu", std=1.0):
    """Gradient of a loss with respect to the attention output: ``[batch, Hq, N, d]``
    normal entries of standard deviation ``std`` (the backward pass's ``dO``)."""
    gen = torch.Generator(device=device).manual_seed(seed)
    g = torch.randn(batch, Hq, N, d, generator=gen, device=device)
    if std != 1.0:
        g = g * std
    return g.to(_torch_dtype(dtype)).contiguous()


def to_f64(x) -> np.ndarray:
    """Exact upcast of a torch tensor (fp32/bf16, any device) or array to float64 numpy."""
    if isinstance(x, torch.Tensor):
        x = x.detach().to("cpu")
        if x.dtype in (torch.bfloat16, torch.float16):
            x = x.float()
        return x.numpy().astype(np.float64)
    return np.asarray(x, dtype=np.float64)
