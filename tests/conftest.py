import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


@pytest.fixture(scope="session")
def cuda_available():
    import torch
    return torch.cuda.is_available()


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Reports the tolerated near-tie swaps of the parity tests (selections that
    differ from the oracle's only between blocks whose oracle scores lie within
    1e-4 relative): one line per test that compared selections, also written to
    gpurun_out/tie_report.json when that folder exists."""
    try:
        from parity import TIE_REPORT
    except ImportError:
        return
    if not TIE_REPORT:
        return
    import json
    tr = terminalreporter
    tr.write_sep("-", "near-tie swaps tolerated by the selection parity checks")
    total = 0
    for name, e in sorted(TIE_REPORT.items()):
        total += e["swaps"]
        tr.write_line(f"{name}: {e['swaps']} swaps in {e['selections_compared']} selections"
                      f" (largest oracle gap {e['largest_gap']:.2e})")
    tr.write_line(f"total: {total} swaps")
    out = os.path.join(ROOT, "gpurun_out")
    if os.path.isdir(out):
        with open(os.path.join(out, "tie_report.json"), "w") as f:
            json.dump(TIE_REPORT, f, indent=1)
