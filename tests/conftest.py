import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


@pytest.fixture(scope="session")
def oracle_lib():
    from oracle import oracle
    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter):
    """Margins of every bf16 output comparison against the oracle: per test
    the largest |dO|, the largest |dO| / bar (the bar is 1e-2, or half a bf16
    step + 1e-3 where |O| >= 4), the largest |dLSE| (bar 1e-3) and the largest
    |O| of the oracle; the overall worst last."""
    from tests import _helpers
    rows = _helpers.MARGINS
    if not rows:
        return
    tr = terminalreporter
    tr.write_sep("-", "parity margins (bf16 outputs against the fp64 oracle)")
    for test, n, d_o, ratio, d_l, o_max in rows:
        tr.write_line(f"{test}  n={n}  max|dO|={d_o:.5f}  worst |dO|/bar={ratio:.3f}  "
                      f"max|dLSE|={d_l:.2e}  max|O|={o_max:.3f}")
    out = os.environ.get("VA_PARITY_MARGINS")
    if out:
        import json
        with open(out, "w") as f:
            json.dump(rows, f)
    worst = max(rows, key=lambda r: r[3])
    worst_l = max(rows, key=lambda r: r[4])
    tr.write_line(f"parity margins: {len(rows)} comparisons, {sum(r[1] for r in rows)} elements; "
                  f"max |dO| {max(r[2] for r in rows):.5f}; worst |dO|/bar {worst[3]:.3f} "
                  f"({worst[0]}); max |dLSE| {worst_l[4]:.2e} (bar 1e-3)")
