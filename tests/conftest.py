import os
import sys

import pytest

_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
for p in (_ROOT, os.path.join(_ROOT, "tests")):
    if p not in sys.path:
        sys.path.insert(0, p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a); runs the CUDA path through the C ABI")


def pytest_collection_modifyitems(config, items):
    import torch

    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_sessionfinish(session, exitstatus):
    """With PKV_PARITY_LOG=<file>, write the largest normalised errors each parity check saw."""
    path = os.environ.get("PKV_PARITY_LOG")
    if not path:
        return
    import json

    from helpers import PARITY_LOG
    with open(path, "w") as f:
        for rec in PARITY_LOG:
            f.write(json.dumps(rec) + "\n")
