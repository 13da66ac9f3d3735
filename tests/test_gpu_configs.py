"""GPU-vs-oracle parity at the full workload sizes, through the C ABI, in the
launch configuration the benchmark times.

* block selection: every row compared with the oracle's fp64 routing; only
  near-ties (fp64 score gap < 1e-4 relative) may differ, and they are counted;
* outputs: sampled (batch, KV head, query block) units -- first, last and
  seeded random ones -- recomputed by the oracle on the GPU's selection;
  max-abs <= 2e-2 and relative-L2 <= 5e-3 (bf16);
* the "all blocks" point of the sweep equals dense causal attention.
Set SSA_PARITY_REPORT=<dir> to write the per-workload counts as JSON.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle as O
from parity import BF16_MAX_ABS, BF16_REL_L2, compare_selection, out_errors
from workloads import CONFIGS, TOPK_ALL, planted_decode, planted_prefill, to_f64

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"


def _report(name, doc):
    d = os.environ.get("SSA_PARITY_REPORT")
    if d:
        os.makedirs(d, exist_ok=True)
        with open(os.path.join(d, f"parity_{name}.json"), "w") as f:
            json.dump(doc, f, indent=1)
    print(name, doc)


def _oracle_route_grouped(Q, S_gpu_shape, K, B, topk, Hkv):
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


def _units(b, Hkv, nq, n_rand, seed):
    rng = np.random.default_rng(seed)
    us = {(0, 0, 0), (b - 1, Hkv - 1, nq - 1), (0, Hkv - 1, nq // 2)}
    while len(us) < n_rand + 3:
        us.add((int(rng.integers(b)), int(rng.integers(Hkv)), int(rng.integers(nq))))
    return sorted(us)


def _prefill_case(name, topk=None, n_units=12):
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
    # summary
    s_err = 0.0
    for g in range(c.Hkv):
        s_err = max(s_err, float(np.max(np.abs(
            to_f64(S[:, g]) - O.block_summary(to_f64(K[:, g:g + 1]), c.B)[:, 0]))))
    assert s_err <= 1e-5
    # selection
    gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
    oi, oc, osc = _oracle_route_grouped(Q, S.shape, K, c.B, topk, c.Hkv)
    assert np.array_equal(gc, oc)
    rows, near, bad = compare_selection(gi, gc, oi, oc,
                                        lambda r: {j: osc[r][j] for j in range(osc.shape[-1])})
    assert not bad, bad[:3]
    # sampled outputs on the GPU's selection
    nq = gc.shape[-1]
    units = _units(c.batch, c.Hkv, nq, n_units, seed=1)
    G = c.Hq // c.Hkv
    sel_o, sel_r, sel_l, sel_rl = [], [], [], []
    for (b, g, i) in units:
        n_sub = min(c.N, (i + 1) * c.B)  # causal: later keys never matter
        hs = slice(g * G, (g + 1) * G)
        ref, rlse = O.sparse_attention(
            to_f64(Q[b:b + 1, hs, :n_sub]), to_f64(K[b:b + 1, g:g + 1, :n_sub]),
            to_f64(V[b:b + 1, g:g + 1, :n_sub]), gi[b:b + 1, g:g + 1, :i + 1],
            gc[b:b + 1, g:g + 1, :i + 1], c.B, units=[(0, 0, i)])
        rows_ = slice(i * c.B, n_sub)
        sel_o.append(to_f64(out[b, hs, rows_]).ravel())
        sel_r.append(ref[0, :, rows_].ravel())
        sel_l.append(to_f64(lse[b, hs, rows_]).ravel())
        sel_rl.append(rlse[0, :, rows_].ravel())
    ma, rel = out_errors(np.concatenate(sel_o), np.concatenate(sel_r))
    lerr = float(np.max(np.abs(np.concatenate(sel_l) - np.concatenate(sel_rl))))
    assert ma <= BF16_MAX_ABS and rel <= BF16_REL_L2, (ma, rel)
    assert lerr <= 1e-3
    doc = {"rows": rows, "near_ties": near, "mismatches": len(bad), "summary_max_abs": s_err,
           "units": len(units), "out_max_abs": ma, "out_rel_l2": rel, "lse_max_abs": lerr,
           "topk": int(topk), "tensor_cores": bool(ssa.ssa_sparse_attn_uses_tensor_cores(
               torch.bfloat16, c.Hq, c.Hkv, c.d, c.B))}
    return doc, (Q, K, V, out, gc)


def test_prefill32k_full_size():
    doc, _ = _prefill_case("prefill32k")
    _report("prefill32k", doc)


def test_prefill128k_full_size():
    doc, _ = _prefill_case("prefill128k", n_units=8)
    _report("prefill128k", doc)


@pytest.mark.parametrize("topk", CONFIGS["sweep"].topk_sweep)
def test_sweep_full_size(topk):
    doc, (Q, K, V, out, gc) = _prefill_case("sweep", topk=topk, n_units=6)
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
    _report(f"sweep_k{topk if topk < TOPK_ALL else 'all'}", doc)


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
    gc = (gi >= 0).sum(-1)
    seqs = [0, 1, 17, 40, c.batch - 1]
    qf = to_f64(q)
    Ls = L.cpu().numpy()
    near = bad_n = rows = 0
    errs_o, errs_r = [], []
    for b in seqs:
        Kb = to_f64(Kc[b:b + 1])
        Vb = to_f64(Vc[b:b + 1])
        Sb = O.block_summary(Kb, c.B)
        oi, oc, osc = O.decode_route(qf[b:b + 1], Sb, Ls[b:b + 1], c.B, c.topk)
        r, n, bad = compare_selection(gi[b:b + 1], gc[b:b + 1], oi, oc,
                                      lambda rr: {j: osc[rr][j] for j in range(osc.shape[-1])})
        rows += r
        near += n
        bad_n += len(bad)
        assert not bad, bad[:3]
        ref, _, _, _ = O.decode(qf[b:b + 1], Kb, Vb, Ls[b:b + 1], c.B, c.topk,
                                idx=gi[b:b + 1], cnt=gc[b:b + 1])
        errs_o.append(to_f64(out[b]).ravel())
        errs_r.append(ref[0].ravel())
    ma, rel = out_errors(np.concatenate(errs_o), np.concatenate(errs_r))
    assert ma <= BF16_MAX_ABS and rel <= BF16_REL_L2, (ma, rel)
    _report("decode", {"sequences_checked": len(seqs), "rows": rows, "near_ties": near,
                       "mismatches": bad_n, "out_max_abs": ma, "out_rel_l2": rel})
