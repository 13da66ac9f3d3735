import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built library")
    config.addinivalue_line("markers", "slow: long-running test")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print the parity counts of the full-size workloads (selection rows,
    near-ties, mismatches, output errors) and, when SSA_PARITY_REPORT names a
    directory, write them there as JSON."""
    import json

    try:
        from parity import REPORT
    except ImportError:
        return
    if not REPORT:
        return
    terminalreporter.write_sep("=", "parity report (near-ties are counted, not failures)")
    for name, doc in REPORT.items():
        keys = ("selection_rows", "near_ties", "mismatches", "output_units", "output_units_total",
                "sequences_checked", "sequences_total", "out_max_abs", "out_rel_l2")
        parts = [f"{k}={doc[k]:.3g}" if isinstance(doc[k], float) else f"{k}={doc[k]}"
                 for k in keys if k in doc]
        terminalreporter.write_line(f"{name}: " + " ".join(parts))
    d = os.environ.get("SSA_PARITY_REPORT")
    if d:
        os.makedirs(d, exist_ok=True)
        with open(os.path.join(d, "parity_report.json"), "w") as f:
            json.dump(REPORT, f, indent=1)
