import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workloads")


def pytest_terminal_summary(terminalreporter):
    """Near-tie report of the session's block-index comparisons: the oracle flags a row
    when its k-th and (k+1)-th pooled scores agree to 1e-5 relative, and a GPU row may
    differ from the oracle only there."""
    try:
        from tests.parity import NEAR_TIE_LOG
    except Exception:
        return
    if not NEAR_TIE_LOG:
        return
    tr = terminalreporter
    tr.write_sep("-", "block selection: oracle near-ties and GPU rows that differ")
    tot = [0, 0, 0, 0]
    for label, rows, near, bad, bad_near in NEAR_TIE_LOG:
        tr.write_line(f"{label or '(unlabelled)':<40} rows {rows:>6}  near-ties {near:>4}  "
                      f"differ {bad:>4}  (at near-ties {bad_near:>4})")
        for i, v in enumerate((rows, near, bad, bad_near)):
            tot[i] += v
    tr.write_line(f"{'total':<40} rows {tot[0]:>6}  near-ties {tot[1]:>4}  differ {tot[2]:>4}  "
                  f"(at near-ties {tot[3]:>4})")
