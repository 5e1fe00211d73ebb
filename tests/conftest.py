import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long CPU-side oracle work")


def pytest_collection_modifyitems(config, items):
    """Skip GPU tests on a machine without CUDA instead of failing them, unless
    CP_REQUIRE_GPU=1 asks for a hard failure."""
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu or os.environ.get("CP_REQUIRE_GPU") == "1":
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_sessionfinish(session, exitstatus):
    """With CP_PARITY_REPORT=<path>, write every bf16 comparison the tests made
    (name, max / mean error, elements beyond the plain 2e-2, worst element in
    bf16 ulps) as JSON: the per-configuration error table."""
    path = os.environ.get("CP_PARITY_REPORT")
    if not path:
        return
    try:
        import helpers
    except Exception:  # pragma: no cover
        return
    import json
    with open(path, "w") as f:
        json.dump(helpers.PARITY_LOG, f, indent=1)
