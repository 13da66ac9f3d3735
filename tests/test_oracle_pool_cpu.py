"""The process-pool plumbing of the full-size parity tests, on the CPU.

Fed the oracle's own results in place of the GPU's, every worker must report
zero error and no selection mismatch; fed a perturbed output, the error must
show.  This checks the packing of bf16 bits, the spawn workers and the error
sums without a GPU.
"""
import numpy as np
import torch

import oracle as O
import oracle_pool as OP
from workloads import planted_decode, planted_prefill, to_f64


def test_pack_unpack_is_exact():
    x = torch.randn(3, 70).to(torch.bfloat16)
    x[0, 0] = -0.0
    x[0, 1] = float("-inf")
    assert np.array_equal(OP.unpack(OP.pack(x)), to_f64(x))
    y = torch.randn(5, 7)
    assert np.array_equal(OP.unpack(OP.pack(y)), to_f64(y))


def test_prefill_and_decode_workers_report_zero_error_on_oracle_results():
    B, topk, G = 64, 3, 2
    Q, K, V = planted_prefill(1, 4, 2, 64 * 9 + 5, 128, B, 3, seed=3, dtype="bf16")
    Qf, Kf, Vf = to_f64(Q), to_f64(K), to_f64(V)
    idx, cnt, _ = O.route(Qf, O.block_summary(Kf, B), B, topk, 2)
    ref, rlse = O.sparse_attention(Qf, Kf, Vf, idx, cnt, B)
    tasks = []
    for g in range(2):
        hs = slice(g * G, (g + 1) * G)
        units = None if g == 0 else [0, 4, 9]
        tasks.append((OP.pack(Q[:, hs]), OP.pack(K[:, g:g + 1]), OP.pack(V[:, g:g + 1]),
                      idx[:, g:g + 1], cnt[:, g:g + 1], B, ("raw", ref[:, hs]),
                      ("raw", rlse[:, hs]), units))
    bad = ("raw", ref[:, :G] + 1e-3)
    tasks.append(tasks[0][:6] + (bad,) + tasks[0][7:])

    q, Kc, Vc, L = planted_decode(2, 4, 2, 64 * 12, 128, B, 3, seed=4, dtype="bf16",
                                  seqlens=[64 * 12, 300])
    qf = to_f64(q)
    S = np.stack([O.block_summary(to_f64(Kc[b:b + 1]), B)[0] for b in range(2)])
    di, dc, _ = O.decode_route(qf, S, L.numpy(), B, topk)
    dref, _, _, _ = O.decode(qf, to_f64(Kc), to_f64(Vc), L.numpy(), B, topk, idx=di, cnt=dc)
    dtasks = [(OP.pack(q[b:b + 1]), OP.pack(Kc[b:b + 1]), OP.pack(Vc[b:b + 1]), int(L[b]), B,
               topk, di[b:b + 1].astype(np.int32), ("raw", dref[b:b + 1])) for b in range(2)]

    with OP.make_pool(3) as pool:
        res = pool.map(OP.prefill_head, tasks, chunksize=1)
        dres = pool.map(OP.decode_sequence, dtasks, chunksize=1)
    for r in res[:2]:
        assert r[0][0] == 0.0 and r[0][2] == 0.0 and r[1] == 0.0
    assert res[0][0][3] == 2 * G * Q.shape[2] * 128 // G  # every row of the head pair
    assert abs(res[2][0][2] - 1e-3) < 1e-12
    ma, rel = OP.combine([res[0][0], res[2][0]])
    assert ma > 0 and rel > 0
    for rows, near, bd, s in dres:
        assert rows == 2 and near == 0 and bd == [] and s[0] == 0.0
