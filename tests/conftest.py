import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running (full-size workloads)")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter):
    """Per comparison of the GPU parity tests: cosine, max abs error, max |ref|,
    elements that needed more than the absolute bound (the bf16 output
    rounding term), and the smallest margin to the bound."""
    mod = sys.modules.get("parity_util")   # imported by the GPU parity tests only
    REPORT = getattr(mod, "REPORT", None)
    if not REPORT:
        return
    tr = terminalreporter
    tr.write_sep("-", "parity margins (cos, max|err|, max|ref|, n>abs, worst margin)")
    for r in REPORT:
        tr.write_line(f"{r['test'][-60:]:60s} {r['name'][:22]:22s} cos={r['cos']:.6f} err={r['max_abs']:.3e} "
                      f"ref={r['max_ref']:.3e} n>abs={r['n_over_abs']}/{r['n']} margin={r['worst_margin']:.3e}")
    path = os.environ.get("MSA_PARITY_REPORT")
    if path:
        import json
        with open(path, "w") as f:
            json.dump(REPORT, f, indent=1)
