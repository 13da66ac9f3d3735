"""Benchmark of the block-sparse attention hot path on B200.

One step = one pass of the whole hot path:
  prefill on the 32K workload (1 x 32 query heads / 8 KV heads, N = 32768,
  d = 128, bf16, B = 64, top-k = 16 + sink + diagonal):
      ssa_block_summary -> ssa_route -> ssa_sparse_attn_fwd
  followed by one decode step on the decode workload (64 sequences x 65536
  cached tokens, 32 / 8 heads, d = 128, bf16, B = 64, top-k = 32 + sink + last):
      ssa_decode (route + split-KV attention + log-sum-exp combine).

`value` is the prefill selected-block TFLOP/s: algorithmic FLOPs of the
attention (4 * d per unmasked (query, key) pair of the selected blocks,
counted from the routing output) over the device time of the prefill pass
(summary + route + attention).  Decode tokens/s and HBM GB/s are reported
beside it.  Inputs are seeded synthetic tensors (planted clusters) resident in
HBM; the working sets exceed the 126 MB L2 (Q alone is 256 MiB, a decode step
reads ~840 MB), so no flush is done between steps.

Two calls are timed apart from the step and reported under `kernels`: the
decode-cache append (a CUDA graph of 20 calls, every append completing a
block) and the backward of the prefill attention on the step's own selection
(8 * d FLOPs per unmasked pair: the dV, dP, dQ and dK contractions).

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

from workloads import CONFIGS, planted_decode, planted_prefill, upstream_grad  # noqa: E402

METRIC = "prefill selected-block TFLOP/s & % BF16 peak; decode tokens/s & HBM GB/s"


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


def attn_traffic_per_launch():
    """DRAM bytes (read + write) per attention launch from the committed ncu
    record, or None when the kernel source changed since the capture."""
    import hashlib
    rec = os.path.join(ROOT, "profiles", "attn_tc_prefill32k_traffic.txt")
    src = os.path.join(ROOT, "block_sparse_top_summary_b200", "csrc", "attn_tc.cu")
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


# ------------------------------------------------------------- our arm
def run_ours(args, world, rank, local):
    import block_sparse_top_summary_b200 as ssa
    ssa.load_library()
    dev = torch.device("cuda", local)
    hbm_peak, bf16_peak, peak_kind = load_peaks()
    cp = CONFIGS["prefill32k"]
    cd = CONFIGS["decode"]
    G = cp.Hq // cp.Hkv

    # --- inputs (seed offset by rank: each rank works on its own problem)
    Q, K, V = planted_prefill(cp.batch, cp.Hq, cp.Hkv, cp.N, cp.d, cp.B, cp.clusters,
                              seed=rank_seed(cp.seed, rank), dtype=cp.dtype)
    Qh, Kh, Vh = Q.pin_memory(), K.pin_memory(), V.pin_memory()
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    q, Kc, Vc, L = planted_decode(cd.batch, cd.Hq, cd.Hkv, cd.L, cd.d, cd.B, cd.clusters,
                                  seed=rank_seed(cd.seed, rank), dtype=cd.dtype, device=dev)
    Sc = ssa.ssa_block_summary(Kc, cd.B)  # precomputed cache summaries (decode input)
    qh, Lh = q.cpu().pin_memory(), L.cpu().pin_memory()

    stream = torch.cuda.current_stream(dev)
    nq = -(-cp.N // cp.B)
    max_sel = ssa.route_width(cp.N, cp.B, cp.topk)
    S = torch.empty(cp.batch, cp.Hkv, cp.N // cp.B, cp.d, dtype=torch.float32, device=dev)
    idx = torch.empty(cp.batch, cp.Hkv, nq, max_sel, dtype=torch.int32, device=dev)
    cnt = torch.empty(cp.batch, cp.Hkv, nq, dtype=torch.int32, device=dev)
    Od = torch.empty_like(Qd)
    lse = torch.empty(cp.batch, cp.Hq, cp.N, dtype=torch.float32, device=dev)
    Odec = torch.empty_like(q)
    didx = torch.empty(cd.batch, cd.Hkv, ssa.decode_width(cd.L, cd.B, cd.topk), dtype=torch.int32,
                       device=dev)
    ws = torch.empty(ssa.ssa_decode_workspace_size(cd.batch, cd.Hq, cd.Hkv, cd.L, cd.d, cd.B,
                                                   cd.topk), dtype=torch.uint8, device=dev)

    def ev():
        return torch.cuda.Event(enable_timing=True)

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        ssa.ssa_block_summary(Kd, cp.B, S=S)
        if evs:
            evs[1].record(stream)
        ssa.ssa_route(Qd, S, cp.B, cp.topk, cp.Hkv, max_sel=max_sel, idx=idx, cnt=cnt)
        if evs:
            evs[2].record(stream)
        ssa.ssa_sparse_attn_fwd(Qd, Kd, Vd, idx, cnt, cp.B, O=Od, lse=lse)
        if evs:
            evs[3].record(stream)
        ssa.ssa_decode(q, Kc, Vc, Sc, L, cd.B, cd.topk, O=Odec, idx=didx, workspace=ws)
        if evs:
            evs[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    flops = attn_flops(cnt[0].cpu().numpy(), cp.N, cp.B, G, cp.d) * cp.batch
    dbytes = decode_bytes(didx.cpu().numpy(), L.cpu().numpy(), cd.B, cd.d, cd.Hq // cd.Hkv, 2)
    sum_bytes = K.numel() * 2 + S.numel() * 4
    route_bytes = Q.numel() * 2 + S.numel() * 4 + idx.numel() * 4 + cnt.numel() * 4

    clocks = ClockSampler(torch.cuda.current_device())
    evs = [[ev() for _ in range(5)] for _ in range(args.steps)]
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = ev(), ev()
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
    seg_mean = seg.mean(axis=0)
    prefill_ms = max_over_ranks(float(seg[:, :3].sum(axis=1).mean()), world)
    decode_ms = max_over_ranks(float(seg_mean[3]), world)
    attn_ms = float(seg_mean[2])

    all_flops = sum_over_ranks(flops, world)
    value = all_flops / (prefill_ms * 1e-3) / 1e12
    attn_tflops = flops / (attn_ms * 1e-3) / 1e12
    dec_tok = sum_over_ranks(cd.batch, world) / (decode_ms * 1e-3)
    dec_gbs = dbytes / (decode_ms * 1e-3) / 1e9

    # --- end to end through the C ABI from pinned host buffers
    Oh = torch.empty_like(Qh).pin_memory()
    Odh = torch.empty(q.shape, dtype=q.dtype).pin_memory()

    def e2e_step():
        Qd.copy_(Qh, non_blocking=True)
        Kd.copy_(Kh, non_blocking=True)
        Vd.copy_(Vh, non_blocking=True)
        q.copy_(qh, non_blocking=True)
        L.copy_(Lh, non_blocking=True)
        step()
        Oh.copy_(Od, non_blocking=True)
        Odh.copy_(Odec, non_blocking=True)

    e2e_steps = max(1, min(args.steps, 5))
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    a, b_ = ev(), ev()
    a.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    b_.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b_) / e2e_steps, world)
    h2d = (Q.numel() + K.numel() + V.numel() + q.numel()) * 2 + L.numel() * 4
    d2h = Q.numel() * 2 + q.numel() * 2

    # --- appending one token per sequence (incremental decoding), timed on its
    # own after everything else, as it rewrites a cache row.  Every call is
    # set up so that its append completes a block (the costlier case): 20
    # calls, each with its own copy of the lengths, are captured in a CUDA graph
    # and replayed, so the device time carries no host gaps; the lengths are
    # restored between replays, outside the timed events.
    app_len = torch.full_like(L, (cd.L // cd.B - 1) * cd.B - 1)
    app_Ls = [app_len.clone() for _ in range(20)]
    kn = torch.randn(cd.batch, cd.Hkv, cd.d, device=q.device).to(torch.bfloat16)
    vn = torch.randn(cd.batch, cd.Hkv, cd.d, device=q.device).to(torch.bfloat16)
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
        a, b_ = ev(), ev()
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

    # --- backward of the attention (training), timed apart from the step on the
    # step's own selection, O and log-sum-exp
    dOd = upstream_grad(cp.batch, cp.Hq, cp.N, cp.d, seed=rank_seed(cp.seed + 1, rank),
                        dtype=cp.dtype, device=dev)
    dQb, dKb, dVb = torch.empty_like(Qd), torch.empty_like(Kd), torch.empty_like(Vd)
    delta = torch.empty(cp.batch, cp.Hq, cp.N, dtype=torch.float32, device=dev)

    def bwd():
        ssa.ssa_sparse_attn_bwd(Qd, Kd, Vd, Od, dOd, lse, idx, cnt, cp.B, dQ=dQb, dK=dKb, dV=dVb,
                                delta=delta)

    bwd_ms = []
    for it in range(2 + 5):
        a, b_ = ev(), ev()
        a.record(stream)
        bwd()
        b_.record(stream)
        torch.cuda.synchronize()
        if it >= 2:
            bwd_ms.append(a.elapsed_time(b_))
    bwd_ms = max_over_ranks(float(np.mean(bwd_ms)), world)
    # 8 d per unmasked (query, key) pair: the dV, dP, dQ and dK contractions
    bwd_flops = 2.0 * flops
    bwd_tflops = bwd_flops / (bwd_ms * 1e-3) / 1e12

    tc = ssa.ssa_sparse_attn_uses_tensor_cores(Q.dtype, cp.Hq, cp.Hkv, cp.d, cp.B)
    kernels = {
        "ssa_block_summary": {"ms": float(seg_mean[0]), "bound": "hbm",
                              "GB/s": sum_bytes / (seg_mean[0] * 1e-3) / 1e9},
        "ssa_route": {"ms": float(seg_mean[1]), "bound": "hbm",
                      "GB/s": route_bytes / (seg_mean[1] * 1e-3) / 1e9},
        "ssa_sparse_attn_fwd": {"ms": attn_ms, "bound": "tensor" if tc else "alu",
                                "TFLOP/s": attn_tflops},
        "ssa_decode": {"ms": float(seg_mean[3]), "bound": "hbm", "GB/s": dec_gbs,
                       "tokens/s": dec_tok},
        "ssa_decode_append": {"ms": app_ms, "bound": "hbm",
                              "GB/s": app_bytes / (app_ms * 1e-3) / 1e9,
                              "note": "timed apart from the step (CUDA graph of 20 calls); "
                                      "every append completes a block"},
        "ssa_sparse_attn_bwd": {"ms": bwd_ms, "bound": "tensor", "TFLOP/s": bwd_tflops,
                                "frac_bf16": bwd_tflops / bf16_peak,
                                "work_per_launch": f"{bwd_flops:.4e} FLOP",
                                "note": "timed apart from the step; FLOPs = 8 d per unmasked "
                                        "(query, key) pair, the recomputed S not counted"},
    }
    for k, v in kernels.items():
        if "GB/s" in v:
            v["frac_hbm"] = v["GB/s"] / hbm_peak
    kernels["ssa_sparse_attn_fwd"]["frac_bf16"] = attn_tflops / bf16_peak
    roof = {"kernel": "ssa_sparse_attn_fwd", "bound": "tensor" if tc else "alu",
            "achieved": attn_tflops, "peak": bf16_peak, "unit": "TFLOP/s",
            "frac": attn_tflops / bf16_peak, "traffic": attn_traffic_per_launch(),
            "traffic_unit": "bytes per launch (ncu dram read+write, profiles/)",
            "peak_source": f"{peak_kind} bf16 dense (burst)",
            "work_per_launch": f"{flops:.4e} FLOP"}

    result = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded planted-cluster Q/K/V; no model weights)",
        "config": {"workload": "prefill32k (1x32q/8kv, N=32768, d=128, bf16, B=64, top-k=16) "
                               "+ decode (64 seq x 65536, 32q/8kv, d=128, bf16, B=64, top-k=32)",
                   "l2": "no flush: inputs larger than L2 (Q 256 MiB; decode reads ~840 MB)",
                   "parallelism": f"replicas x{world} (independent problems, no collective)"},
        "prefill_ms": prefill_ms, "decode": {"tokens_per_s": dec_tok, "ms": decode_ms,
                                             "GB/s": dec_gbs, "frac_hbm": dec_gbs / hbm_peak,
                                             "bytes_per_step": dbytes},
        "kernels": kernels, "roofline": roof,
        "e2e": {"value": all_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": args.steps * 5,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(result))
    if world > 1:
        torch.distributed.destroy_process_group()


# ------------------------------------------------------------ oracle (CPU) arm
def _oracle_prefill_sample(nblocks: int, seed: int = 0):
    """Oracle summary + routing + attention on KV head 0 of the 32K workload,
    attention restricted to `nblocks` query blocks spread over the sequence."""
    import oracle as O
    from workloads import to_f64
    cp = CONFIGS["prefill32k"]
    G = cp.Hq // cp.Hkv
    Q, K, V = planted_prefill(cp.batch, cp.Hq, cp.Hkv, cp.N, cp.d, cp.B, cp.clusters,
                              seed=cp.seed + seed, dtype=cp.dtype)
    Qf = to_f64(Q[:, :G])
    Kf = to_f64(K[:, :1])
    Vf = to_f64(V[:, :1])
    t0 = time.perf_counter()
    S = O.block_summary(Kf, cp.B)
    idx, cnt, _ = O.route(Qf, S, cp.B, cp.topk, 1)
    nq = cnt.shape[-1]
    picks = np.linspace(0, nq - 1, nblocks).astype(int)
    O.sparse_attention(Qf, Kf, Vf, idx, cnt, cp.B, units=[(0, 0, int(i)) for i in picks])
    dt = time.perf_counter() - t0
    sub = np.zeros_like(cnt[0, 0])
    sub[picks] = cnt[0, 0, picks]
    rows = np.minimum(cp.B, cp.N - picks * cp.B).astype(np.float64)
    pairs = (rows * cp.B * (cnt[0, 0, picks] - 1) + rows * (rows + 1) / 2).sum()
    flops = pairs * G * 4 * cp.d
    return flops, dt


def cpu_baseline(budget_s: float = 15.0):
    cores = len(os.sched_getaffinity(0))
    # calibrate the number of attended query blocks to fit the budget
    f, dt = _oracle_prefill_sample(8)
    n = int(max(8, min(512, 8 * budget_s / max(dt, 1e-3))))
    f, dt = _oracle_prefill_sample(n)
    return {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 numpy oracle on the 32K prefill workload, KV head 0 (4 query heads): "
                      f"summary + routing of all 512 query blocks, attention of {n} query blocks "
                      f"spread over the sequence; {dt:.1f} s; FLOPs = selected-block FLOPs of "
                      f"the attended blocks",
            "threads": torch.get_num_threads()}


def run_reference(args, world, rank):
    if rank != 0:
        return
    cores = len(os.sched_getaffinity(0))
    for _ in range(args.warmup):
        _oracle_prefill_sample(4)
    times, flops = [], 0.0
    for k in range(args.steps):
        f, dt = _oracle_prefill_sample(16, seed=k)
        times.append(dt)
        flops = f
    ms = float(np.mean(times)) * 1e3
    value = flops / (ms * 1e-3) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded planted-cluster Q/K/V; no model weights)",
        "config": {"workload": "prefill32k (1x32q/8kv, N=32768, d=128, bf16, B=64, top-k=16); "
                               "CPU sample: KV head 0, 16 attended query blocks per step"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": "fp64 oracle: summary + routing of KV head 0, attention of "
                                   "16 query blocks per step"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def run_ncu_case(case: str, launches: int):
    """Run one kernel of the hot path `launches` times on a bounded workload
    (a few GB on the device, working set above the 126 MB L2) for profiling:
    summary / route / attn on the 32K prefill workload, decode on 16 of the 64
    sequences of the decode workload."""
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
        cp = CONFIGS["prefill32k"]
        Q, K, V = planted_prefill(cp.batch, cp.Hq, cp.Hkv, cp.N, cp.d, cp.B, cp.clusters,
                                  seed=cp.seed, dtype=cp.dtype)
        Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
        S = ssa.ssa_block_summary(Kd, cp.B)
        idx, cnt = ssa.ssa_route(Qd, S, cp.B, cp.topk, cp.Hkv)
        torch.cuda.synchronize()
        for _ in range(launches):
            if case == "summary":
                ssa.ssa_block_summary(Kd, cp.B, S=S)
            elif case == "route":
                ssa.ssa_route(Qd, S, cp.B, cp.topk, cp.Hkv, idx=idx, cnt=cnt)
            else:
                ssa.ssa_sparse_attn_fwd(Qd, Kd, Vd, idx, cnt, cp.B)
    torch.cuda.synchronize()
    assert ssa.ssa_device_error() == 0
    print(f"ncu case {case}: {launches} launches done")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ncu-case", choices=["summary", "route", "attn", "decode"], default=None,
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
