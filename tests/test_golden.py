"""The oracle reproduces the committed tiny-workload fixture (regression guard)."""
import json
import os

import numpy as np

import oracle as O
from workloads import CONFIGS, planted_prefill, to_f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.json")


def test_tiny_fixture_reproduces():
    doc = json.load(open(GOLDEN))
    c = CONFIGS["tiny"]
    Q, K, V = planted_prefill(c.batch, c.Hq, c.Hkv, c.N, c.d, c.B, c.clusters, c.seed, c.dtype)
    Qf, Kf, Vf = to_f64(Q), to_f64(K), to_f64(V)
    S = O.block_summary(Kf, c.B)
    idx, cnt, _ = O.route(Qf, S, c.B, c.topk, c.Hkv)
    assert idx[0, 0].tolist() == doc["idx"]
    assert cnt[0, 0].tolist() == doc["cnt"]
    out, lse = O.sparse_attention(Qf, Kf, Vf, idx, cnt, c.B)
    rows = doc["rows"]
    np.testing.assert_allclose(out[0, 0, rows], doc["O_head0"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(out[0, 1, rows], doc["O_head1"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(S[0, 0, 1, :8], doc["S_block1_first8"], rtol=0, atol=1e-14)
