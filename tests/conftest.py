import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built libaxr.so")
    config.addinivalue_line("markers", "slow: CPU test that takes more than a few seconds")


def pytest_collection_modifyitems(config, items):
    # GPU tests are skipped (not failed) on a machine without CUDA when they are selected anyway.
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Scores failing the strict |s|-relative reading of the score tolerance, per test (tests/parity.py)."""
    try:
        from tests import parity
    except Exception:  # pragma: no cover
        return
    if not parity.STRICT_LOG:
        return
    tr = terminalreporter
    tr.section("scores outside the strict |s|-relative reading (1e-6 + 1e-5 |s|)")
    tot = [0, 0]
    for key, (ns, n) in sorted(parity.STRICT_LOG.items()):
        tr.write_line(f"{ns:8d} of {n:10d}  ({ns / max(n, 1):.2e})  {key}")
        tot[0] += ns
        tot[1] += n
    tr.write_line(f"{tot[0]:8d} of {tot[1]:10d}  ({tot[0] / max(tot[1], 1):.2e})  all tests")
