"""Write the tiny-workload golden fixture from the fp64 oracle.

The pages print no worked example, so the stored values come from the oracle
alone (it is pinned by tests/test_oracle_pins.py).  Run from the repository root:
``python tests/golden/make_golden.py``.  It imports only ``oracle`` and the seeded
input generators.
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle as O  # noqa: E402
from workloads import CONFIGS, planted_prefill, to_f64  # noqa: E402

ROWS = [0, 1, 63, 64, 500, 1023]


def main():
    c = CONFIGS["tiny"]
    Q, K, V = planted_prefill(c.batch, c.Hq, c.Hkv, c.N, c.d, c.B, c.clusters, c.seed, c.dtype)
    Qf, Kf, Vf = to_f64(Q), to_f64(K), to_f64(V)
    S = O.block_summary(Kf, c.B)
    idx, cnt, sc = O.route(Qf, S, c.B, c.topk, c.Hkv)
    out, lse = O.sparse_attention(Qf, Kf, Vf, idx, cnt, c.B)
    doc = {
        "what": "tiny workload (1x2q/1kv, N=1024, d=64, fp32, B=64, top-k=4, seed 0): "
                "oracle block selection and sampled outputs",
        "idx": idx[0, 0].tolist(),
        "cnt": cnt[0, 0].tolist(),
        "rows": ROWS,
        "O_head0": [out[0, 0, r].tolist() for r in ROWS],
        "O_head1": [out[0, 1, r].tolist() for r in ROWS],
        "LSE": [[float(lse[0, h, r]) for r in ROWS] for h in range(2)],
        "S_block1_first8": S[0, 0, 1, :8].tolist(),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json")
    with open(path, "w") as f:
        json.dump(doc, f, indent=0)
    print("wrote", path)


if __name__ == "__main__":
    main()
