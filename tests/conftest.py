import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running parity case")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """One line per attention parity check (tests/parity.py), so the error
    figures reach the log when everything passes too."""
    try:
        from tests.parity import RECORDS
    except Exception:
        return
    if not RECORDS:
        return
    tr = terminalreporter
    tr.section("attention parity (gated = |err| - tie allowance - half bf16 ulp; gate max 1e-2, mean 1e-3)")
    small = [r for r in RECORDS if r["what"].startswith(("fp8 [", "bf16 ["))]
    rest = [r for r in RECORDS if r not in small]
    if small:
        tr.write_line(
            f"{len(small)} small-shape checks: gated max {max(r['max'] for r in small):.2e}, "
            f"worst mean {max(r['mean'] for r in small):.2e}, plain max "
            f"{max(r['plain_max'] for r in small):.2e}, excluded "
            f"{sum(r['n_excluded'] for r in small)} of {sum(r['n'] for r in small)}")
    for r in rest:
        line = (f"{r['what']}: gated {r['max']:.2e}/{r['mean']:.2e} plain {r['plain_max']:.2e}/"
                f"{r['plain_mean']:.2e} n={r['n']} tie={r['n_tie']} alt={r.get('n_alt', 0)} "
                f"excl={r['n_excluded']}")
        if r.get("uq"):
            line += f" vs-unquantised {r['uq'][0]:.2e}/{r['uq'][1]:.2e}"
        tr.write_line(line)
