import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running full-size case")


def pytest_collection_modifyitems(config, items):
    # GPU tests are skipped cleanly (not failed) on a machine without a device
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """Worst state errors of the run, normwise (asserted) and per element (reported)."""
    mod = sys.modules.get("tests.gpu_util")
    log = getattr(mod, "STATE_LOG", None) if mod else None
    if not log:
        return
    tr = terminalreporter
    tr.section("state checks: normwise (asserted) and per-element ratio (reported)")
    tr.write_line(f"{len(log)} checks; worst normwise {max(r[1] for r in log):.3g} of tolerance, "
                  f"worst per-element {max(r[2] for r in log):.3g} of tolerance")
    for what, nw, pe in sorted(log, key=lambda r: -r[2])[:8]:
        tr.write_line(f"  {what}: normwise {nw:.3g}, per-element {pe:.3g}")
