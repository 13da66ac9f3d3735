"""Benchmark of the block-sparse attention hot path on B200.

One step = one pass of the whole hot path:
  prefill on the headline workload, by default the 128K one (1 x 32 query
  heads / 8 KV heads, N = 131072, d = 128, bf16, B = 64, top-k = 32 + sink +
  diagonal):
      ssa_block_summary -> ssa_route -> ssa_sparse_attn_fwd
  followed by one decode step on the decode workload (64 sequences x 65536
  cached tokens, 32 / 8 heads, d = 128, bf16, B = 64, top-k = 32 + sink + last):
      ssa_decode (route + split-KV attention + log-sum-exp combine).
`--workload prefill32k` makes the 32K workload (N = 32768, top-k = 16) the
step's prefill instead.

`value` is the prefill selected-block TFLOP/s: algorithmic FLOPs of the
attention (4 * d per unmasked (query, key) pair of the selected blocks,
counted from the routing output) over the device time of the prefill pass
(summary + route + attention).  Decode tokens/s and HBM GB/s are reported
beside it.  Inputs are seeded synthetic tensors (planted clusters) drawn on
the device and resident in HBM; the working sets exceed the 126 MB L2 (Q
alone is 1 GiB at 128K, a decode step reads ~840 MB), so no flush is done
between steps.

Timed apart from the step and reported under their own keys:
- `prefill32k`: the prefill pass on the other prefill workload;
- `sweep`: the sparsity sweep (2 x 16 / 4 heads, N = 65536, B = 128) at
  top-k = 4, 8, 16, 32, 64 and all: attention TFLOP/s against k;
- `kernels.ssa_decode_append`: the decode-cache append (a CUDA graph of 20
  calls, every append completing a block);
- `kernels.ssa_sparse_attn_bwd`: the backward of the 32K prefill attention on
  its own selection (8 * d FLOPs per unmasked pair: the dV, dP, dQ and dK
  contractions);
- `widened`: the calls beyond the four steps -- decode over a paged copy of the
  decode cache (checked bitwise against the contiguous decode) and with one
  selection per query head, two-level routing on the 128K prefill, and
  DashAttention's learned summary, alpha-entmax routing and prior attention
  on the 32K prefill -- each with its bytes or FLOPs and fraction of peak.
Every kernel line carries its fraction of the measured peak (MEASURED_PEAKS)
and of the nominal one (2.25 PFLOP/s dense bf16, 8 TB/s HBM).

`--impl reference` times the fp64 CPU oracle on a bounded sample of the same
workload instead (there is no runnable upstream implementation).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import CONFIGS, TOPK_ALL, planted_decode, planted_prefill, upstream_grad  # noqa: E402

METRIC = "prefill selected-block TFLOP/s & % BF16 peak; decode tokens/s & HBM GB/s"

# Nominal B200 peaks the targets are stated against.
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 8000.0


# ------------------------------------------------------------- work accounting
def attn_flops(cnt: np.ndarray, N: int, B: int, G: int, d: int) -> float:
    """4*d per unmasked (query, key) pair of the selected blocks, all heads."""
    nq = cnt.shape[-1]
    rows = np.minimum(B, N - np.arange(nq) * B).astype(np.float64)
    pairs = rows * B * (cnt.astype(np.float64) - 1) + rows * (rows + 1) / 2
    return float(pairs.sum()) * G * 4 * d


def decode_bytes(idx: np.ndarray, seqlens: np.ndarray, B: int, d: int, G: int, esize: int) -> float:
    """K and V rows of the selected blocks, the candidate summaries, q and O."""
    total = 0.0
    batch, Hkv, _ = idx.shape
    for b in range(batch):
        L = int(seqlens[b])
        last = (L - 1) // B
        for g in range(Hkv):
            sel = idx[b, g][idx[b, g] >= 0]
            rows = np.minimum(B, L - sel * B).sum()
            total += 2.0 * rows * d * esize
            total += max(last - 1, 0) * d * 4.0
    total += 2.0 * batch * Hkv * G * d * esize
    return total


def per_head_decode_bytes(idx: np.ndarray, seqlens: np.ndarray, B: int, d: int, G: int,
                          esize: int) -> float:
    """The bytes decode with one selection per query head (idx ``[batch, Hq, w]``)
    must move: the K and V rows of the union of the selections of a KV head's G
    query heads (a block two heads select is read once), the KV head's candidate
    summaries once, and every head's q and O rows."""
    total = 0.0
    batch, Hq, _ = idx.shape
    Hkv = Hq // G
    for b in range(batch):
        L = int(seqlens[b])
        last = (L - 1) // B
        for g in range(Hkv):
            grp = idx[b, g * G:(g + 1) * G]
            sel = np.unique(grp[grp >= 0])
            rows = np.minimum(B, L - sel * B).sum()
            total += 2.0 * rows * d * esize + max(last - 1, 0) * d * 4.0
    total += 2.0 * batch * Hq * d * esize
    return total


def traffic_per_launch(record: str, source: str):
    """DRAM bytes (read + write) per launch from a committed ncu record under
    profiles/, or None when the kernel source changed since the capture."""
    import hashlib
    rec = os.path.join(ROOT, "profiles", record)
    src = os.path.join(ROOT, "block_sparse_top_summary_b200", "csrc", source)
    if not (os.path.exists(rec) and os.path.exists(src)):
        return None
    kv = {}
    for line in open(rec):
        if "=" in line and not line.startswith("#"):
            k, v = line.strip().split("=", 1)
            kv[k] = v
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
    if kv.get("kernel_source_sha256") != digest:
        return None
    return int(kv["dram_bytes_read"]) + int(kv["dram_bytes_write"])


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return j["hbm_gbs"], j["bf16_tflops"], "measured"
    return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons with NVML on a thread (every 5 ms)
    while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, dev_index: int):
        self.dev = dev_index
        self.samples = []
        self.thread = None

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            phys = int(vis.split(",")[self.dev]) if vis and vis.split(",")[0].isdigit() else self.dev
            self.h = pynvml.nvmlDeviceGetHandleByIndex(phys)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None
            return
        self.stop_flag = False

        def run():
            while not self.stop_flag:
                try:
                    mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                    rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    self.samples.append((mhz, rs))
                except Exception:
                    pass
                time.sleep(0.005)

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return None
        self.stop_flag = True
        self.thread.join()
        if not self.samples:
            return None
        mhz = [m for m, _ in self.samples]
        reasons = sorted({n for _, r in self.samples for n, bit in self.REASONS.items() if r & bit})
        return {"sm_mhz": float(np.median(mhz)), "sm_max_mhz": float(self.max_mhz),
                "reasons": reasons, "samples": len(mhz), "source": "nvml, 5 ms"}


# ------------------------------------------------------------ distributed
# The hot path partitions into independent problems: each rank runs the same
# workloads on its own seeded inputs (weak scaling, no data-path collective).
# torch.distributed is used only for the timing barrier and the max / sum of
# per-rank numbers.
def dist_setup(gpus: int, backend: str = "nccl"):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        if backend == "nccl":
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def rank_seed(base: int, rank: int) -> int:
    """Seed of a rank's own problem."""
    return base + rank


def _reduce_device():
    if torch.distributed.is_initialized() and torch.distributed.get_backend() == "nccl":
        return "cuda"
    return "cpu"


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], device=_reduce_device(), dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], device=_reduce_device(), dtype=torch.float64)
    torch.distributed.all_reduce(t)
    return float(t.item())


def fracs(achieved: float, measured: float, nominal: float) -> dict:
    """Fractions of the measured and of the nominal peak."""
    return {"frac": achieved / measured, "frac_nominal": achieved / nominal}


def describe(c, topk=None) -> str:
    """The workload's name and sizes (`topk` overrides its top-k; a string is
    printed as is)."""
    k = c.topk if topk is None else topk
    k = "all" if not isinstance(k, str) and k >= TOPK_ALL else k
    return (f"{c.name} ({c.batch}x{c.Hq}q/{c.Hkv}kv, N={c.N}, d={c.d}, {c.dtype}, B={c.B}, "
            f"top-k={k})")


# ------------------------------------------------------------- our arm
class Prefill:
    """Device buffers and the three prefill calls of one prefill workload."""

    def __init__(self, ssa, c, dev, seed, topk=None):
        self.ssa, self.c = ssa, c
        self.topk = c.topk if topk is None else topk
        self.Q, self.K, self.V = planted_prefill(c.batch, c.Hq, c.Hkv, c.N, c.d, c.B, c.clusters,
                                                 seed=seed, dtype=c.dtype, device=dev)
        nq = -(-c.N // c.B)
        self.max_sel = ssa.route_width(c.N, c.B, self.topk)
        self.S = torch.empty(c.batch, c.Hkv, c.N // c.B, c.d, dtype=torch.float32, device=dev)
        self.idx = torch.empty(c.batch, c.Hkv, nq, self.max_sel, dtype=torch.int32, device=dev)
        self.cnt = torch.empty(c.batch, c.Hkv, nq, dtype=torch.int32, device=dev)
        self.O = torch.empty_like(self.Q)
        self.lse = torch.empty(c.batch, c.Hq, c.N, dtype=torch.float32, device=dev)

    def set_topk(self, topk):
        c = self.c
        self.topk = topk
        nq = -(-c.N // c.B)
        self.max_sel = self.ssa.route_width(c.N, c.B, topk)
        self.idx = torch.empty(c.batch, c.Hkv, nq, self.max_sel, dtype=torch.int32,
                               device=self.Q.device)

    def run(self, evs=None, stream=None):
        ssa, c = self.ssa, self.c
        if evs:
            evs[0].record(stream)
        ssa.ssa_block_summary(self.K, c.B, S=self.S)
        if evs:
            evs[1].record(stream)
        ssa.ssa_route(self.Q, self.S, c.B, self.topk, c.Hkv, max_sel=self.max_sel, idx=self.idx,
                      cnt=self.cnt)
        if evs:
            evs[2].record(stream)
        ssa.ssa_sparse_attn_fwd(self.Q, self.K, self.V, self.idx, self.cnt, c.B, O=self.O,
                                lse=self.lse)
        if evs:
            evs[3].record(stream)

    def flops(self):
        c = self.c
        cnt = self.cnt.cpu().numpy()
        return sum(attn_flops(cnt[b, g], c.N, c.B, c.Hq // c.Hkv, c.d)
                   for b in range(c.batch) for g in range(c.Hkv))

    def summary_bytes(self):
        return self.K.numel() * self.K.element_size() + self.S.numel() * 4

    def route_bytes(self):
        return (self.Q.numel() * self.Q.element_size() + self.S.numel() * 4 +
                self.idx.numel() * 4 + self.cnt.numel() * 4)


def _ev():
    return torch.cuda.Event(enable_timing=True)


def time_prefill(p: Prefill, iters: int, warmup: int, stream, world):
    """Mean per-call device times (ms) of summary, route and attention."""
    for _ in range(warmup):
        p.run()
    torch.cuda.synchronize()
    evs = [[_ev() for _ in range(4)] for _ in range(iters)]
    barrier(world)
    for k in range(iters):
        p.run(evs[k], stream)
    torch.cuda.synchronize()
    seg = np.array([[evs[k][s].elapsed_time(evs[k][s + 1]) for s in range(3)]
                    for k in range(iters)])
    return [max_over_ranks(float(x), world) for x in seg.mean(axis=0)]


def prefill_report(p: Prefill, seg, flops, hbm_peak, bf16_peak, tc):
    sm, rt, at = seg
    pass_ms = sm + rt + at
    att = flops / (at * 1e-3) / 1e12
    sgb = p.summary_bytes() / (sm * 1e-3) / 1e9
    rgb = p.route_bytes() / (rt * 1e-3) / 1e9
    return {
        "workload": describe(p.c, p.topk),
        "pass_ms": pass_ms, "TFLOP/s": flops / (pass_ms * 1e-3) / 1e12,
        "attn_flops": flops,
        "ssa_block_summary": {"ms": sm, "bound": "hbm", "GB/s": sgb,
                              **fracs(sgb, hbm_peak, NOMINAL_HBM_GBS),
                              "bytes": p.summary_bytes()},
        "ssa_route": {"ms": rt, "bound": "hbm", "GB/s": rgb,
                      **fracs(rgb, hbm_peak, NOMINAL_HBM_GBS), "bytes": p.route_bytes()},
        "ssa_sparse_attn_fwd": {"ms": at, "bound": "tensor" if tc else "alu", "TFLOP/s": att,
                                **fracs(att, bf16_peak, NOMINAL_BF16_TFLOPS)},
    }


def time_call(f, iters: int, warmup: int, stream, world) -> float:
    """Mean device time (ms) of f() over `iters` calls after `warmup` calls."""
    for _ in range(warmup):
        f()
    torch.cuda.synchronize()
    barrier(world)
    a, b_ = _ev(), _ev()
    a.record(stream)
    for _ in range(iters):
        f()
    b_.record(stream)
    torch.cuda.synchronize()
    return max_over_ranks(a.elapsed_time(b_) / iters, world)


def widened(ssa, p128, p32, q, Kc, Vc, Sc, L, cd, dev, stream, world, hbm_peak, bf16_peak):
    """The rows beyond the four hot-path steps, each on a workload of the
    benchmark, with its own work count and fraction of peak."""
    out = {}

    def hbm(ms, nbytes, workload, **kw):
        gbs = nbytes / (ms * 1e-3) / 1e9
        return {"ms": ms, "GB/s": gbs, **fracs(gbs, hbm_peak, NOMINAL_HBM_GBS), "bytes": nbytes,
                "workload": workload, **kw}

    # paged decode: the decode workload's cache cut into pages in a shuffled order
    nblk = cd.L // cd.B
    gen = torch.Generator(device=dev).manual_seed(7)
    perm = torch.randperm(cd.batch * nblk, generator=gen, device=dev)
    Kp = torch.empty(cd.batch * nblk, cd.Hkv, cd.B, cd.d, dtype=Kc.dtype, device=dev)
    Vp = torch.empty_like(Kp)
    Kp[perm] = Kc.view(cd.batch, cd.Hkv, nblk, cd.B, cd.d).transpose(1, 2).reshape(-1, cd.Hkv, cd.B, cd.d)
    Vp[perm] = Vc.view(cd.batch, cd.Hkv, nblk, cd.B, cd.d).transpose(1, 2).reshape(-1, cd.Hkv, cd.B, cd.d)
    table = perm.view(cd.batch, nblk).to(torch.int32).contiguous()
    ws = torch.empty(ssa.ssa_decode_workspace_size(cd.batch, cd.Hq, cd.Hkv, cd.L, cd.d, cd.B,
                                                   cd.topk), dtype=torch.uint8, device=dev)
    Op = torch.empty_like(q)
    ip = torch.empty(cd.batch, cd.Hkv, ssa.decode_width(cd.L, cd.B, cd.topk), dtype=torch.int32,
                     device=dev)
    f = lambda: ssa.ssa_decode_paged(q, Kp, Vp, Sc, table, L, cd.B, cd.topk, O=Op, idx=ip,
                                     workspace=ws)
    ms = time_call(f, 20, 3, stream, world)
    Oc, ic = ssa.ssa_decode(q, Kc, Vc, Sc, L, cd.B, cd.topk)
    assert torch.equal(Op, Oc) and torch.equal(ip, ic), "paged decode differs from the contiguous one"
    nb = decode_bytes(ip.cpu().numpy(), L.cpu().numpy(), cd.B, cd.d, cd.Hq // cd.Hkv, 2)
    out["ssa_decode_paged"] = hbm(ms, nb, "decode (64 seq x 65536) in 65536 pages, shuffled",
                                  tokens_per_s=cd.batch / (ms * 1e-3))
    del Kp, Vp
    # per-head decode routing on the decode workload
    wsh = torch.empty(ssa.ssa_decode_per_head_workspace_size(cd.batch, cd.Hq, cd.Hkv, cd.L, cd.d,
                                                             cd.B, cd.topk),
                      dtype=torch.uint8, device=dev)
    Oh = torch.empty_like(q)
    ih = torch.empty(cd.batch, cd.Hq, ssa.decode_width(cd.L, cd.B, cd.topk), dtype=torch.int32,
                     device=dev)
    f = lambda: ssa.ssa_decode_per_head(q, Kc, Vc, Sc, L, cd.B, cd.topk, O=Oh, idx=ih,
                                        workspace=wsh)
    ms = time_call(f, 20, 3, stream, world)
    nb = per_head_decode_bytes(ih.cpu().numpy(), L.cpu().numpy(), cd.B, cd.d, cd.Hq // cd.Hkv, 2)
    out["ssa_decode_per_head"] = hbm(ms, nb, "decode (64 seq x 65536), one selection per query head",
                                     tokens_per_s=cd.batch / (ms * 1e-3))
    # two-level routing on the 128K prefill: segments of 8 blocks, 8 kept, 32 blocks
    c = p128.c
    hi = torch.empty(c.batch, c.Hkv, -(-c.N // c.B), min(c.topk, -(-c.N // c.B)) + 2,
                     dtype=torch.int32, device=dev)
    hc = torch.empty(c.batch, c.Hkv, -(-c.N // c.B), dtype=torch.int32, device=dev)
    f = lambda: ssa.ssa_route_hierarchical(p128.Q, p128.S, c.B, 8, 8, c.topk, c.Hkv, idx=hi,
                                           cnt=hc)
    ms = time_call(f, 10, 3, stream, world)
    out["ssa_route_hierarchical"] = hbm(ms, p128.route_bytes(),
                                        describe(c) + ", segments of 8 blocks, 8 kept")
    # DashAttention's stages: the learned summary on the 128K keys (a stream,
    # like the block summary), the routing and prior attention on the 32K prefill
    c = p128.c
    qbar = torch.randn(c.Hkv, c.d, generator=gen, device=dev)
    S_l = torch.empty_like(p128.S)
    f = lambda: ssa.ssa_learned_summary(p128.K, qbar, c.B, S=S_l)
    ms = time_call(f, 20, 3, stream, world)
    out["ssa_learned_summary"] = hbm(ms, p128.summary_bytes(), describe(c))
    del S_l
    c = p32.c
    f = lambda: ssa.ssa_route_entmax(p32.Q, p32.S, c.B, c.Hkv, 1.5, 8.0, 0.5)
    ms = time_call(f, 10, 3, stream, world)
    ei, ec, eb, _ = ssa.ssa_route_entmax(p32.Q, p32.S, c.B, c.Hkv, 1.5, 8.0, 0.5)
    nb = p32.Q.numel() * 2 + p32.S.numel() * 4 + ei.numel() * 8 + ec.numel() * 4
    out["ssa_route_entmax"] = hbm(ms, nb, describe(c) + ", alpha 1.5, gamma 8, sigma 0.5",
                                  mean_blocks=float(ec.float().mean()))
    Oe = torch.empty_like(p32.Q)
    f = lambda: ssa.ssa_sparse_attn_fwd_prior(p32.Q, p32.K, p32.V, ei, ec, eb, c.B, O=Oe)
    ms = time_call(f, 10, 3, stream, world)
    ecn = ec.cpu().numpy()
    fl = sum(attn_flops(ecn[b, g], c.N, c.B, c.Hq // c.Hkv, c.d)
             for b in range(c.batch) for g in range(c.Hkv))
    tf = fl / (ms * 1e-3) / 1e12
    out["ssa_sparse_attn_fwd_prior"] = {"ms": ms, "TFLOP/s": tf, "bound": "tensor",
                                        "flops": fl, "workload": describe(c) + ", entmax selection",
                                        "note": "the tcgen05 attention kernel with the prior "
                                                "as a per-block logit offset",
                                        **fracs(tf, bf16_peak, NOMINAL_BF16_TFLOPS)}
    return out


def run_ours(args, world, rank, local):
    import block_sparse_top_summary_b200 as ssa
    ssa.load_library()
    dev = torch.device("cuda", local)
    hbm_peak, bf16_peak, peak_kind = load_peaks()
    head = args.workload
    other = "prefill32k" if head == "prefill128k" else "prefill128k"
    cp = CONFIGS[head]
    cd = CONFIGS["decode"]
    stream = torch.cuda.current_stream(dev)

    # --- inputs, drawn on the device (seed offset by rank: each rank works on
    # its own problem)
    P = Prefill(ssa, cp, dev, rank_seed(cp.seed, rank))
    q, Kc, Vc, L = planted_decode(cd.batch, cd.Hq, cd.Hkv, cd.L, cd.d, cd.B, cd.clusters,
                                  seed=rank_seed(cd.seed, rank), dtype=cd.dtype, device=dev)
    Sc = ssa.ssa_block_summary(Kc, cd.B)  # precomputed cache summaries (decode input)
    Odec = torch.empty_like(q)
    didx = torch.empty(cd.batch, cd.Hkv, ssa.decode_width(cd.L, cd.B, cd.topk), dtype=torch.int32,
                       device=dev)
    ws = torch.empty(ssa.ssa_decode_workspace_size(cd.batch, cd.Hq, cd.Hkv, cd.L, cd.d, cd.B,
                                                   cd.topk), dtype=torch.uint8, device=dev)
    G = cp.Hq // cp.Hkv

    def step(evs=None):
        P.run(evs, stream)
        ssa.ssa_decode(q, Kc, Vc, Sc, L, cd.B, cd.topk, O=Odec, idx=didx, workspace=ws)
        if evs:
            evs[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert ssa.ssa_device_error() == 0
    flops = P.flops()
    dbytes = decode_bytes(didx.cpu().numpy(), L.cpu().numpy(), cd.B, cd.d, cd.Hq // cd.Hkv, 2)

    clocks = ClockSampler(torch.cuda.current_device())
    evs = [[_ev() for _ in range(5)] for _ in range(args.steps)]
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = _ev(), _ev()
    t0.record(stream)
    for k in range(args.steps):
        step(evs[k])
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    total_ms = max_over_ranks(t0.elapsed_time(t1), world)
    seg = np.array([[evs[k][s].elapsed_time(evs[k][s + 1]) for s in range(4)]
                    for k in range(args.steps)])  # ms: summary, route, attn, decode
    seg_mean = [max_over_ranks(float(x), world) for x in seg.mean(axis=0)]
    prefill_ms = max_over_ranks(float(seg[:, :3].sum(axis=1).mean()), world)
    decode_ms = seg_mean[3]

    all_flops = sum_over_ranks(flops, world)
    value = all_flops / (prefill_ms * 1e-3) / 1e12
    tc = ssa.ssa_sparse_attn_uses_tensor_cores(torch.bfloat16, cp.Hq, cp.Hkv, cp.d, cp.B)
    head_rep = prefill_report(P, seg_mean[:3], flops, hbm_peak, bf16_peak, tc)
    attn_tflops = head_rep["ssa_sparse_attn_fwd"]["TFLOP/s"]
    dec_tok = sum_over_ranks(cd.batch, world) / (decode_ms * 1e-3)
    dec_gbs = dbytes / (decode_ms * 1e-3) / 1e9

    # --- end to end through the C ABI from pinned host buffers: the step's
    # prefill inputs and decode query in, both outputs out, every step
    Qh = P.Q.cpu().pin_memory()
    Kh = P.K.cpu().pin_memory()
    Vh = P.V.cpu().pin_memory()
    qh, Lh = q.cpu().pin_memory(), L.cpu().pin_memory()
    Oh = torch.empty_like(Qh).pin_memory()
    Odh = torch.empty(q.shape, dtype=q.dtype).pin_memory()

    def e2e_step():
        P.Q.copy_(Qh, non_blocking=True)
        P.K.copy_(Kh, non_blocking=True)
        P.V.copy_(Vh, non_blocking=True)
        q.copy_(qh, non_blocking=True)
        L.copy_(Lh, non_blocking=True)
        step()
        Oh.copy_(P.O, non_blocking=True)
        Odh.copy_(Odec, non_blocking=True)

    e2e_steps = max(1, min(args.steps, 5))
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    a, b_ = _ev(), _ev()
    a.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    b_.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b_) / e2e_steps, world)
    h2d = (Qh.numel() + Kh.numel() + Vh.numel() + qh.numel()) * 2 + Lh.numel() * 4
    d2h = Oh.numel() * 2 + Odh.numel() * 2
    del Qh, Kh, Vh, Oh

    # --- the other prefill workload, timed apart
    po = Prefill(ssa, CONFIGS[other], dev, rank_seed(CONFIGS[other].seed, rank))
    seg_o = time_prefill(po, iters=10, warmup=3, stream=stream, world=world)
    other_rep = prefill_report(po, seg_o, po.flops(), hbm_peak, bf16_peak,
                               ssa.ssa_sparse_attn_uses_tensor_cores(
                                   torch.bfloat16, po.c.Hq, po.c.Hkv, po.c.d, po.c.B))
    p32 = P if head == "prefill32k" else po  # the backward runs on the 32K workload

    # --- the sparsity sweep: attention TFLOP/s against k, "all" last
    cs = CONFIGS["sweep"]
    ps = Prefill(ssa, cs, dev, rank_seed(cs.seed, rank))
    sweep = []
    for k in cs.topk_sweep:
        ps.set_topk(k)
        seg_s = time_prefill(ps, iters=5 if k >= TOPK_ALL else 10, warmup=3, stream=stream,
                             world=world)
        rep = prefill_report(ps, seg_s, ps.flops(), hbm_peak, bf16_peak,
                             ssa.ssa_sparse_attn_uses_tensor_cores(torch.bfloat16, cs.Hq, cs.Hkv,
                                                                   cs.d, cs.B))
        sweep.append({"topk": "all" if k >= TOPK_ALL else k, "attn_flops": rep["attn_flops"],
                      "attn_ms": rep["ssa_sparse_attn_fwd"]["ms"],
                      "attn_TFLOP/s": rep["ssa_sparse_attn_fwd"]["TFLOP/s"],
                      "attn_frac": rep["ssa_sparse_attn_fwd"]["frac"],
                      "attn_frac_nominal": rep["ssa_sparse_attn_fwd"]["frac_nominal"],
                      "pass_ms": rep["pass_ms"], "pass_TFLOP/s": rep["TFLOP/s"]})
    del ps

    # --- appending one token per sequence (incremental decoding), timed on its
    # own after the step, as it rewrites a cache row.  Every call is set up so
    # that its append completes a block (the costlier case): 20 calls, each
    # with its own copy of the lengths, are captured in a CUDA graph and
    # replayed, so the device time carries no host gaps; the lengths are
    # restored between replays, outside the timed events.
    app_len = torch.full_like(L, (cd.L // cd.B - 1) * cd.B - 1)
    app_Ls = [app_len.clone() for _ in range(20)]
    kn = torch.randn(cd.batch, cd.Hkv, cd.d, device=dev).to(torch.bfloat16)
    vn = torch.randn(cd.batch, cd.Hkv, cd.d, device=dev).to(torch.bfloat16)
    ssa.ssa_decode_append(Kc, Vc, Sc, app_Ls[0], kn, vn, cd.B, stream=stream)  # warm-up
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for t_ in app_Ls:
            ssa.ssa_decode_append(Kc, Vc, Sc, t_, kn, vn, cd.B)
    app_ms = []
    for it in range(3 + 10):
        for t_ in app_Ls:
            t_.copy_(app_len)
        torch.cuda.synchronize()
        a, b_ = _ev(), _ev()
        a.record(stream)
        graph.replay()
        b_.record(stream)
        torch.cuda.synchronize()
        if it >= 3:
            app_ms.append(a.elapsed_time(b_) / len(app_Ls))
    del graph
    app_ms = max_over_ranks(float(np.mean(app_ms)), world)
    # per sequence and KV head: two rows written, the completed block's B key rows
    # read back, one fp32 summary row written
    app_bytes = cd.batch * cd.Hkv * (2 * cd.d * 2 + cd.B * cd.d * 2 + cd.d * 4)
    app_gbs = app_bytes / (app_ms * 1e-3) / 1e9

    # --- backward of the 32K attention (training), timed apart from the step
    # on that workload's own selection, O and log-sum-exp
    c32 = p32.c
    p32.run()
    dOd = upstream_grad(c32.batch, c32.Hq, c32.N, c32.d, seed=rank_seed(c32.seed + 1, rank),
                        dtype=c32.dtype, device=dev)
    dQb, dKb, dVb = torch.empty_like(p32.Q), torch.empty_like(p32.K), torch.empty_like(p32.V)
    bws = torch.empty(ssa.ssa_sparse_attn_bwd_workspace_size(c32.batch, c32.Hq, c32.Hkv, c32.N,
                                                             c32.d, c32.B),
                      dtype=torch.uint8, device=dev)

    def bwd():
        ssa.ssa_sparse_attn_bwd(p32.Q, p32.K, p32.V, p32.O, dOd, p32.lse, p32.idx, p32.cnt,
                                c32.B, dQ=dQb, dK=dKb, dV=dVb, workspace=bws)

    bwd_ms = []
    for it in range(2 + 5):
        a, b_ = _ev(), _ev()
        a.record(stream)
        bwd()
        b_.record(stream)
        torch.cuda.synchronize()
        if it >= 2:
            bwd_ms.append(a.elapsed_time(b_))
    bwd_ms = max_over_ranks(float(np.mean(bwd_ms)), world)
    # 8 d per unmasked (query, key) pair: the dV, dP, dQ and dK contractions
    bwd_flops = 2.0 * p32.flops()
    bwd_tflops = bwd_flops / (bwd_ms * 1e-3) / 1e12
    del dQb, dKb, dVb, bws
    wide = widened(ssa, P if head == "prefill128k" else po, p32, q, Kc, Vc, Sc, L, cd, dev, stream,
                   world, hbm_peak, bf16_peak)
    assert ssa.ssa_device_error() == 0

    kernels = {k: head_rep[k] for k in ("ssa_block_summary", "ssa_route", "ssa_sparse_attn_fwd")}
    kernels["ssa_decode"] = {"ms": decode_ms, "bound": "hbm", "GB/s": dec_gbs,
                             "tokens/s": dec_tok, **fracs(dec_gbs, hbm_peak, NOMINAL_HBM_GBS),
                             "bytes": dbytes}
    kernels["ssa_decode_append"] = {
        "ms": app_ms, "bound": "hbm", "GB/s": app_gbs, **fracs(app_gbs, hbm_peak, NOMINAL_HBM_GBS),
        "note": "timed apart from the step (CUDA graph of 20 calls); every append completes a "
                "block; launch-bound at 8.9 MB per call"}
    kernels["ssa_sparse_attn_bwd"] = {
        "ms": bwd_ms, "bound": "tensor", "TFLOP/s": bwd_tflops,
        **fracs(bwd_tflops, bf16_peak, NOMINAL_BF16_TFLOPS),
        "work_per_launch": f"{bwd_flops:.4e} FLOP", "workload": describe(c32),
        "note": "timed apart from the step; FLOPs = 8 d per unmasked (query, key) pair, the "
                "recomputed S not counted"}
    roof = {"kernel": "ssa_sparse_attn_fwd", "bound": "tensor" if tc else "alu",
            "achieved": attn_tflops, "peak": bf16_peak, "unit": "TFLOP/s",
            "frac": attn_tflops / bf16_peak,
            "traffic": traffic_per_launch(f"attn_tc_{head}_traffic.txt", "attn_tc.cu"),
            "traffic_unit": "bytes per launch (ncu dram read+write, profiles/)",
            "peak_source": f"{peak_kind} bf16 dense (burst), MEASURED_PEAKS.json",
            "frac_nominal": attn_tflops / NOMINAL_BF16_TFLOPS,
            "nominal_peak": NOMINAL_BF16_TFLOPS,
            "work_per_launch": f"{flops:.4e} FLOP"}

    result = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded planted-cluster Q/K/V drawn on the device; no model weights)",
        "config": {"workload": f"{describe(cp)} + decode (64 seq x 65536, 32q/8kv, d=128, bf16, "
                               f"B=64, top-k=32)",
                   "l2": "no flush: inputs larger than L2 (Q 1 GiB at 128K, 256 MiB at 32K; "
                         "decode reads ~840 MB)",
                   "parallelism": f"replicas x{world} (independent problems, no collective)"},
        "prefill_ms": prefill_ms,
        "decode": {"tokens_per_s": dec_tok, "ms": decode_ms, "GB/s": dec_gbs,
                   **fracs(dec_gbs, hbm_peak, NOMINAL_HBM_GBS), "bytes_per_step": dbytes},
        "kernels": kernels, "roofline": roof,
        other: other_rep,
        "sweep": {"workload": describe(cs, "k"),
                  "points": sweep},
        "widened": wide,
        "e2e": {"value": all_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": args.steps * 5,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(head, budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(result))
    if world > 1:
        torch.distributed.destroy_process_group()


# ------------------------------------------------------------ oracle (CPU) arm
def _oracle_prefill_sample(name: str, nblocks: int, seed: int = 0):
    """Oracle summary + routing + attention on KV head 0 of a prefill workload
    (its 4 query heads), attention restricted to `nblocks` query blocks spread
    over the sequence.  Returns (selected-block FLOPs of the attended blocks,
    seconds)."""
    import oracle as O
    from workloads import to_f64
    cp = CONFIGS[name]
    G = cp.Hq // cp.Hkv
    Q, K, V = planted_prefill(1, G, 1, cp.N, cp.d, cp.B, cp.clusters, seed=cp.seed + seed,
                              dtype=cp.dtype)
    Qf, Kf, Vf = to_f64(Q), to_f64(K), to_f64(V)
    del Q, K, V
    t0 = time.perf_counter()
    S = O.block_summary(Kf, cp.B)
    idx, cnt, _ = O.route(Qf, S, cp.B, cp.topk, 1)
    nq = cnt.shape[-1]
    picks = np.linspace(0, nq - 1, nblocks).astype(int)
    O.sparse_attention(Qf, Kf, Vf, idx, cnt, cp.B, units=[(0, 0, int(i)) for i in picks])
    dt = time.perf_counter() - t0
    rows = np.minimum(cp.B, cp.N - picks * cp.B).astype(np.float64)
    pairs = (rows * cp.B * (cnt[0, 0, picks] - 1) + rows * (rows + 1) / 2).sum()
    return pairs * G * 4 * cp.d, dt


def _oracle_decode_sample(nseq: int, seed: int = 0):
    """Oracle decode step (fp64 summaries of the cache, routing, attention) on
    `nseq` sequences of the decode workload.  Returns (tokens, seconds)."""
    import oracle as O
    from workloads import to_f64
    cd = CONFIGS["decode"]
    q, Kc, Vc, L = planted_decode(nseq, cd.Hq, cd.Hkv, cd.L, cd.d, cd.B, cd.clusters,
                                  seed=cd.seed + seed, dtype=cd.dtype)
    qf, Ls = to_f64(q), L.numpy()
    Kc, Vc = Kc.float().numpy(), Vc.float().numpy()  # exact; widened to fp64 by the oracle
    t0 = time.perf_counter()
    S = np.stack([O.block_summary(Kc[b:b + 1], cd.B)[0] for b in range(nseq)])
    O.decode(qf, Kc, Vc, Ls, cd.B, cd.topk, S=S)
    return nseq, time.perf_counter() - t0


def cpu_baseline(name: str, budget_s: float = 15.0):
    cores = len(os.sched_getaffinity(0))
    # calibrate the number of attended query blocks to fit the budget
    f, dt = _oracle_prefill_sample(name, 4)
    n = int(max(4, min(CONFIGS[name].N // CONFIGS[name].B, 4 * budget_s / max(dt, 1e-3))))
    f, dt = _oracle_prefill_sample(name, n)
    tok, ddt = _oracle_decode_sample(2)
    nq = CONFIGS[name].N // CONFIGS[name].B
    return {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 numpy oracle on the {name} workload, KV head 0 (its 4 query heads): "
                      f"summary + routing of all {nq} query blocks, attention of {n} query blocks "
                      f"spread over the sequence; {dt:.1f} s; FLOPs = selected-block FLOPs of "
                      f"the attended blocks",
            "threads": torch.get_num_threads(),
            "decode": {"tokens_per_s": tok / ddt, "seconds": ddt,
                       "sample": f"{tok} of the 64 decode sequences: fp64 summaries of the "
                                 f"65536-token cache, routing and attention"}}


def run_reference(args, world, rank):
    if rank != 0:
        return
    name = args.workload
    cores = len(os.sched_getaffinity(0))
    for _ in range(args.warmup):
        _oracle_prefill_sample(name, 2)
    times, flops = [], 0.0
    for k in range(args.steps):
        f, dt = _oracle_prefill_sample(name, 4, seed=k)
        times.append(dt)
        flops = f
    tok, ddt = _oracle_decode_sample(1)
    ms = float(np.mean(times)) * 1e3
    value = flops / (ms * 1e-3) / 1e12
    c = CONFIGS[name]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded planted-cluster Q/K/V; no model weights)",
        "config": {"workload": f"{describe(c)}; CPU sample: KV head 0, summary + routing of "
                               f"every query block and attention of 4 query blocks per step"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"fp64 oracle: summary + routing of KV head 0 of {name}, "
                                   f"attention of 4 query blocks per step",
                         "decode_tokens_per_s": tok / ddt},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def run_ncu_case(case: str, launches: int):
    """Run one kernel of the hot path `launches` times on a bounded workload
    (a few GB on the device, working set above the 126 MB L2) for profiling:
    summary / route / attn / bwd on the 32K prefill workload, attn128k on the
    128K one, decode on 16 of the 64 sequences of the decode workload."""
    import block_sparse_top_summary_b200 as ssa
    ssa.load_library()
    dev = torch.device("cuda", 0)
    if case == "decode":
        cd = CONFIGS["decode"]
        q, Kc, Vc, L = planted_decode(16, cd.Hq, cd.Hkv, cd.L, cd.d, cd.B, cd.clusters,
                                      seed=cd.seed, dtype=cd.dtype, device=dev)
        Sc = ssa.ssa_block_summary(Kc, cd.B)
        torch.cuda.synchronize()
        for _ in range(launches):
            ssa.ssa_decode(q, Kc, Vc, Sc, L, cd.B, cd.topk)
    else:
        cp = CONFIGS["prefill128k" if case.endswith("128k") else "prefill32k"]
        p = Prefill(ssa, cp, dev, cp.seed)
        p.run()
        torch.cuda.synchronize()
        if case == "bwd":
            dO = upstream_grad(cp.batch, cp.Hq, cp.N, cp.d, seed=1, dtype=cp.dtype, device=dev)
        for _ in range(launches):
            if case == "summary":
                ssa.ssa_block_summary(p.K, cp.B, S=p.S)
            elif case.startswith("route"):
                ssa.ssa_route(p.Q, p.S, cp.B, cp.topk, cp.Hkv, idx=p.idx, cnt=p.cnt)
            elif case == "bwd":
                ssa.ssa_sparse_attn_bwd(p.Q, p.K, p.V, p.O, dO, p.lse, p.idx, p.cnt, cp.B)
            else:
                ssa.ssa_sparse_attn_fwd(p.Q, p.K, p.V, p.idx, p.cnt, cp.B, O=p.O, lse=p.lse)
    torch.cuda.synchronize()
    assert ssa.ssa_device_error() == 0
    print(f"ncu case {case}: {launches} launches done")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["prefill128k", "prefill32k"], default="prefill128k",
                    help="the prefill workload of the timed step")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ncu-case", default=None,
                    choices=["summary", "route", "attn", "bwd", "decode", "route128k",
                             "attn128k"],
                    help="run one kernel on a bounded workload for profiling, then exit")
    ap.add_argument("--ncu-launches", type=int, default=2)
    args = ap.parse_args()
    if args.ncu_case:
        run_ncu_case(args.ncu_case, args.ncu_launches)
        return
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup(args.gpus)
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
