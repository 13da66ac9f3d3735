"""The multi-process (N > 1) path of bench.py on CPU: two gloo ranks.

The hot path partitions into independent problems, so each rank works on its
own seeded inputs and only timing numbers cross ranks (max for time, sum for
work).  This checks that plumbing and that the ranks' problems differ.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import oracle as O
    from workloads import planted_prefill, to_f64
    w, r, _ = bench.dist_setup(world, backend="gloo")
    assert (w, r) == (world, rank)
    bench.barrier(w)
    mx = bench.max_over_ranks(float(rank + 1), w)
    sm = bench.sum_over_ranks(float(rank + 1), w)
    Q, K, V = planted_prefill(1, 4, 2, 64 * 6, 16, 64, 2, seed=bench.rank_seed(5, r), dtype="f32")
    idx, cnt, _ = O.route(to_f64(Q), O.block_summary(to_f64(K), 64), 64, 2, 2)
    flops = bench.attn_flops(cnt[0, 0], 64 * 6, 64, 2, 16)
    total = bench.sum_over_ranks(flops, w)
    out[rank] = (mx, sm, float(Q.sum()), flops, total)
    torch.distributed.destroy_process_group()


def test_two_gloo_ranks_reduce_timing_and_work():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout=120)
        assert p.exitcode == 0
    a, b = out[0], out[1]
    assert a[0] == b[0] == 2.0          # max over ranks
    assert a[1] == b[1] == 3.0          # sum over ranks
    assert a[2] != b[2]                 # each rank has its own seeded problem
    assert a[4] == b[4] == pytest.approx(a[3] + b[3])
