import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture
def golden():
    """Loader of the hand-worked fixtures under tests/golden (strings '-inf'/'inf'/'nan'
    stand for the non-finite values JSON cannot hold)."""
    import json

    def fix(v):
        if isinstance(v, list):
            return [fix(u) for u in v]
        if isinstance(v, dict):
            return {k: fix(u) for k, u in v.items()}
        if v in ("-inf", "inf", "nan"):
            return float(v)
        return v

    def load(name):
        with open(os.path.join(ROOT, "tests", "golden", name)) as f:
            return fix(json.load(f))

    return load


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """The parity report (level-2 errors, near-tie counts) of the tests that ran."""
    try:
        from helpers import REPORT
    except Exception:  # pragma: no cover
        return
    if REPORT:
        terminalreporter.write_sep("-", "parity report")
        for line in REPORT:
            terminalreporter.write_line(line)
