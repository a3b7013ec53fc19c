import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 GPU (runs the CUDA library)")
    config.addinivalue_line("markers", "slow: large oracle workloads (minutes of CPU)")


def pytest_collection_modifyitems(config, items):
    import torch
    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """One line per greedy-pick comparison: rows compared, near-ties excluded."""
    from tests._util import PARITY_LOG
    if not PARITY_LOG:
        return
    tot = sum(e["rows"] for e in PARITY_LOG)
    exc = sum(e["excluded"] for e in PARITY_LOG)
    terminalreporter.write_line(
        f"draft parity: {len(PARITY_LOG)} comparisons, {exc} of {tot} rows excluded as "
        f"near-ties ({100.0 * exc / max(tot, 1):.2f}%)")
    for e in PARITY_LOG:
        extra = "".join(f" {k}={v}" for k, v in e.items()
                        if k not in ("name", "rows", "excluded", "rule"))
        terminalreporter.write_line(
            f"  {e['name']}: {e['excluded']}/{e['rows']} excluded ({e['rule']}){extra}")
