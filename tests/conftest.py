import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU case")


def gpu_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:  # pragma: no cover
        return False


def pytest_collection_modifyitems(config, items):
    if gpu_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device here")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Per-head parity diagnostic: the worst per-(b, h) error of every GPU test
    (each head divided by its own largest oracle value) next to the
    whole-tensor metric, largest first."""
    try:
        from tests.parity import WORST
    except Exception:  # pragma: no cover
        return
    if not WORST:
        return
    tr = terminalreporter
    tr.write_sep("-", "per-head parity (worst per-(b,h) rel | whole-tensor rel), largest first")
    rows = sorted(WORST.items(), key=lambda kv: -kv[1][0])
    for name, (worst, whole) in rows[:12]:
        tr.write_line(f"{worst:.2e} | {whole:.2e}  {name.split('::', 1)[-1]}")
    full = [kv for kv in rows if "fullsize" in kv[0]]
    for name, (worst, whole) in full:
        tr.write_line(f"full size: {worst:.2e} | {whole:.2e}  {name.split('::', 1)[-1]}")
    tr.write_line(f"{len(rows)} tests recorded; max per-head rel {rows[0][1][0]:.2e}")
