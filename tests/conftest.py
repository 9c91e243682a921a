import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")


def cuda_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def cuda():
    if not cuda_available():
        pytest.skip("no CUDA device")
    return True


def pytest_terminal_summary(terminalreporter):
    """One line per parity check: rows compared, rows equal to the oracle's,
    rows that differ only inside the fp32 tie band, percentile-gate tiles
    inside their band, and output errors against the oracle."""
    try:
        import parity
    except Exception:
        return
    if not parity.REPORT:
        return
    terminalreporter.write_sep("-", "parity against the oracle (tie band counted)")
    for r in parity.REPORT:
        rest = " ".join(f"{k}={v:.3g}" if isinstance(v, float) else f"{k}={v}"
                        for k, v in r.items() if k not in ("test", "workload"))
        terminalreporter.write_line(f"PARITY {r['test']} {r['workload']} {rest}")
