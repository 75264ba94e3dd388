import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running")


def pytest_collection_modifyitems(config, items):
    # A GPU test on a machine without a device is a skip, never a silent CPU path.
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


def pytest_terminal_summary(terminalreporter):
    try:
        from tests import harness
    except Exception:
        return
    if harness.ERRORS:
        worst = max(e for _, e in harness.ERRORS)
        terminalreporter.write_line(
            f"attention parity: {len(harness.ERRORS)} comparisons, worst max|err|/max|ref| = {worst:.3e} "
            f"(bound {harness.ATTN_RTOL})")
        out = os.environ.get("KVQ_PARITY_REPORT")
        if out:
            import json
            with open(out, "w") as fh:
                json.dump(harness.ERRORS, fh, indent=0)
