"""GPU-vs-oracle parity at the full workload sizes, through the C ABI, in the
launch configuration the benchmark times.

* block selection: every row of every workload compared with the oracle's
  fp64 routing; only near-ties (fp64 score gap < 1e-4 relative) may differ,
  and they are counted;
* outputs, recomputed by the oracle on the GPU's selection:
  - prefill 32K: every (batch, KV head, query block) unit;
  - decode: every one of the 64 sequences;
  - prefill 128K and each sweep point: 64 units, the first, the last and 62
    seeded random ones (the oracle would take hours on all of them);
  max-abs <= 2e-2 and relative-L2 <= 5e-3 (bf16); LSE within 1e-3;
* the "all blocks" point of the sweep equals dense causal attention.
The oracle work runs in a spawn process pool (tests/oracle_pool.py).  The
counts of every workload go to the session's parity report, printed at the
end of the run (and written as JSON when SSA_PARITY_REPORT names a directory).
"""
import numpy as np
import pytest
import torch

import oracle as O
import oracle_pool as OP
from parity import BF16_MAX_ABS, BF16_REL_L2, compare_selection, record
from workloads import CONFIGS, TOPK_ALL, planted_decode, planted_prefill, to_f64

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"
LSE_MAX_ABS = 1e-3


def _oracle_route_grouped(Q, K, B, topk, Hkv):
    """Oracle routing one KV head at a time (bounded host memory)."""
    b, Hq, N, d = Q.shape
    G = Hq // Hkv
    nq = -(-N // B)
    w = min(topk, nq) + 2
    idx = np.full((b, Hkv, nq, w), -1, dtype=np.int64)
    cnt = np.zeros((b, Hkv, nq), dtype=np.int64)
    sc = np.zeros((b, Hkv, nq, N // B))
    for g in range(Hkv):
        Qg = to_f64(Q[:, g * G:(g + 1) * G])
        Sg = O.block_summary(to_f64(K[:, g:g + 1]), B)
        i_, c_, s_ = O.route(Qg, Sg, B, topk, 1)
        idx[:, g] = i_[:, 0]
        cnt[:, g] = c_[:, 0]
        sc[:, g] = s_[:, 0]
    return idx, cnt, sc


def _sample_units(b, Hkv, nq, n, seed):
    """First, last and seeded random (batch, KV head, query block) units."""
    rng = np.random.default_rng(seed)
    us = {(0, 0, 0), (b - 1, Hkv - 1, nq - 1)}
    while len(us) < n:
        us.add((int(rng.integers(b)), int(rng.integers(Hkv)), int(rng.integers(nq))))
    return sorted(us)


def _prefill_case(name, topk=None, n_units=None):
    """Run the workload's prefill on the GPU and compare it with the oracle.
    n_units None compares every unit's output; else a sample of n_units."""
    import block_sparse_top_summary_b200 as ssa
    c = CONFIGS[name]
    topk = c.topk if topk is None else topk
    Q, K, V = planted_prefill(c.batch, c.Hq, c.Hkv, c.N, c.d, c.B, c.clusters, c.seed, c.dtype)
    Qd, Kd, Vd = Q.to(DEV), K.to(DEV), V.to(DEV)
    S = ssa.ssa_block_summary(Kd, c.B)
    idx, cnt = ssa.ssa_route(Qd, S, c.B, topk, c.Hkv)
    out, lse = ssa.ssa_sparse_attn_fwd(Qd, Kd, Vd, idx, cnt, c.B)
    torch.cuda.synchronize()
    assert ssa.ssa_device_error() == 0
    out_h, lse_h = out.cpu(), lse.cpu()
    del Qd, Kd, Vd, out, lse
    # summary
    s_err = 0.0
    for g in range(c.Hkv):
        s_err = max(s_err, float(np.max(np.abs(
            to_f64(S[:, g]) - O.block_summary(to_f64(K[:, g:g + 1]), c.B)[:, 0]))))
    assert s_err <= 1e-5
    # selection, every row
    gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
    oi, oc, osc = _oracle_route_grouped(Q, K, c.B, topk, c.Hkv)
    assert np.array_equal(gc, oc)
    rows, near, bad = compare_selection(gi, gc, oi, oc,
                                        lambda r: {j: osc[r][j] for j in range(osc.shape[-1])})
    assert not bad, bad[:3]
    # outputs on the GPU's selection
    nq = gc.shape[-1]
    G = c.Hq // c.Hkv
    if n_units is None:
        by_head = {(b, g): None for b in range(c.batch) for g in range(c.Hkv)}
        n_checked = c.batch * c.Hkv * nq
    else:
        by_head = {}
        for (b, g, i) in _sample_units(c.batch, c.Hkv, nq, n_units, seed=1):
            by_head.setdefault((b, g), []).append(i)
        n_checked = sum(len(v) for v in by_head.values())
    tasks = []
    for (b, g), units in by_head.items():
        hs = slice(g * G, (g + 1) * G)
        tasks.append((OP.pack(Q[b:b + 1, hs]), OP.pack(K[b:b + 1, g:g + 1]),
                      OP.pack(V[b:b + 1, g:g + 1]), gi[b:b + 1, g:g + 1], gc[b:b + 1, g:g + 1],
                      c.B, OP.pack(out_h[b:b + 1, hs]), OP.pack(lse_h[b:b + 1, hs]), units))
    with OP.make_pool(len(tasks)) as pool:
        res = pool.map(OP.prefill_head, tasks, chunksize=1)
    ma, rel = OP.combine([r[0] for r in res])
    lerr = max(r[1] for r in res)
    assert ma <= BF16_MAX_ABS and rel <= BF16_REL_L2, (ma, rel)
    assert lerr <= LSE_MAX_ABS, lerr
    doc = {"selection_rows": rows, "near_ties": near, "mismatches": len(bad),
           "summary_max_abs": s_err, "output_units": n_checked,
           "output_units_total": c.batch * c.Hkv * nq, "out_max_abs": ma, "out_rel_l2": rel,
           "lse_max_abs": lerr, "topk": int(min(topk, nq)),
           "tensor_cores": bool(ssa.ssa_sparse_attn_uses_tensor_cores(
               torch.bfloat16, c.Hq, c.Hkv, c.d, c.B))}
    return doc, (Q, K, V, out_h, gc)


def test_prefill32k_full_size():
    doc, _ = _prefill_case("prefill32k")
    record("prefill32k", doc)


def test_prefill128k_full_size():
    doc, _ = _prefill_case("prefill128k", n_units=64)
    record("prefill128k", doc)


@pytest.mark.parametrize("topk", CONFIGS["sweep"].topk_sweep)
def test_sweep_full_size(topk):
    doc, (Q, K, V, out, gc) = _prefill_case("sweep", topk=topk, n_units=64)
    c = CONFIGS["sweep"]
    if topk >= TOPK_ALL:
        nq = c.N // c.B
        assert np.array_equal(gc, np.broadcast_to(np.arange(1, nq + 1), gc.shape))
        # every query row sees every earlier key: compare sampled rows with dense SDPA
        G = c.Hq // c.Hkv
        rows = np.array([0, 1, 127, 128, 30000, c.N - 1])
        errs = []
        for (b, h) in [(0, 0), (1, c.Hq - 1), (0, 7)]:
            g = h // G
            q = torch.from_numpy(to_f64(Q[b, h, rows]))
            k = torch.from_numpy(to_f64(K[b, g]))
            v = torch.from_numpy(to_f64(V[b, g]))
            logits = (q @ k.T) / np.sqrt(c.d)
            mask = torch.arange(c.N)[None, :] > torch.from_numpy(rows)[:, None]
            p = torch.softmax(logits.masked_fill(mask, -np.inf), -1)
            errs.append(np.max(np.abs(to_f64(out[b, h, rows]) - (p @ v).numpy())))
        doc["dense_rows_max_abs"] = float(max(errs))
        assert doc["dense_rows_max_abs"] <= BF16_MAX_ABS
    record(f"sweep_k{topk if topk < TOPK_ALL else 'all'}", doc)


def test_decode_full_size():
    import block_sparse_top_summary_b200 as ssa
    c = CONFIGS["decode"]
    q, Kc, Vc, L = planted_decode(c.batch, c.Hq, c.Hkv, c.L, c.d, c.B, c.clusters, c.seed,
                                  c.dtype, device=DEV)
    S = ssa.ssa_block_summary(Kc, c.B)
    out, idx = ssa.ssa_decode(q, Kc, Vc, S, L, c.B, c.topk)
    torch.cuda.synchronize()
    assert ssa.ssa_device_error() == 0
    gi = idx.cpu().numpy()
    Ls = L.cpu().numpy()

    def tasks():
        # one sequence at a time: each task holds one sequence's caches (256 MiB)
        for b in range(c.batch):
            yield (OP.pack(q[b:b + 1]), OP.pack(Kc[b:b + 1]), OP.pack(Vc[b:b + 1]), int(Ls[b]),
                   c.B, c.topk, gi[b:b + 1], OP.pack(out[b:b + 1]))

    rows = near = 0
    bad = []
    sums = []
    with OP.make_pool(c.batch) as pool:
        for r, n, bd, s in pool.imap(OP.decode_sequence, tasks(), chunksize=1):
            rows += r
            near += n
            bad += bd
            sums.append(s)
    assert not bad, bad[:3]
    ma, rel = OP.combine(sums)
    assert ma <= BF16_MAX_ABS and rel <= BF16_REL_L2, (ma, rel)
    record("decode", {"sequences_checked": len(sums), "sequences_total": c.batch,
                      "selection_rows": rows, "near_ties": near, "mismatches": len(bad),
                      "out_max_abs": ma, "out_rel_l2": rel})
