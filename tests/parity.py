"""Comparison helpers for GPU-vs-oracle parity tests (test infrastructure)."""
from __future__ import annotations

import numpy as np

# Selection near-tie: the fp64 gap between a differing pair of scores, relative
# to the larger magnitude, is below this.
NEAR_TIE_REL = 1e-4

# Output tolerances.
F32_MAX_ABS = 1e-5
BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3


def _gap_is_near_tie(a: float, b: float) -> bool:
    den = max(abs(a), abs(b))
    if den == 0.0:
        return True
    return abs(a - b) / den < NEAR_TIE_REL


def compare_selection(gpu_idx, gpu_cnt, ora_idx, ora_cnt, ora_scores_fn):
    """Compare block lists row by row.

    gpu_idx / ora_idx: ``[..., width]`` arrays (ascending, -1 padded; widths may
    differ); gpu_cnt / ora_cnt: ``[...]``.  ``ora_scores_fn(row_index_tuple)``
    returns the fp64 candidate scores of that row as ``{block: score}``.
    A differing row is accepted as a near-tie when every block chosen by only
    one side scores within NEAR_TIE_REL of some block chosen by only the other
    side.  Returns ``(n_rows, n_near_tie_rows, bad_rows)``.
    """
    gpu_idx = np.asarray(gpu_idx)
    ora_idx = np.asarray(ora_idx)
    gpu_cnt = np.asarray(gpu_cnt)
    ora_cnt = np.asarray(ora_cnt)
    n_rows = int(np.prod(gpu_cnt.shape))
    near, bad = 0, []
    for row in np.ndindex(gpu_cnt.shape):
        g = gpu_idx[row][: gpu_cnt[row]].tolist()
        o = ora_idx[row][: ora_cnt[row]].tolist()
        if g == o:
            continue
        gs, os_ = set(g), set(o)
        only_g, only_o = sorted(gs - os_), sorted(os_ - gs)
        ok = (len(g) == len(o) and len(only_g) == len(only_o) and g == sorted(g)
              and -1 not in g)
        if ok:
            sc = ora_scores_fn(row)
            for x in only_g:
                if not any(_gap_is_near_tie(sc[x], sc[y]) for y in only_o):
                    ok = False
                    break
        if ok:
            near += 1
        else:
            bad.append((row, g, o))
    return n_rows, near, bad


def out_errors(gpu, ref):
    """(max-abs, relative-L2) of gpu vs ref (both float64 arrays)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = gpu - ref
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(diff) / den) if den > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


# Per-workload parity counts of this test session (selection rows, near-ties,
# mismatches, output errors), printed at the end of the run by conftest.py.
REPORT: dict = {}


def record(name: str, doc: dict):
    """Add one workload's parity counts to the session report."""
    REPORT[name] = doc
    print(name, doc)
