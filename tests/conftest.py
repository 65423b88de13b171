import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a); parity against the oracle")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("gpu test collected but no CUDA device is visible")
    return torch.device("cuda:0")


def pytest_sessionfinish(session, exitstatus):
    """With QMOE_PARITY_REPORT set, write the GPU parity figures (per-tensor
    max relative error and the element-wise error over |ref| >= 0.1 rms) of
    every case that ran to that JSON file."""
    path = os.environ.get("QMOE_PARITY_REPORT")
    if not path:
        return
    mod = sys.modules.get("gpu_helpers")
    if mod is None or not mod.REPORT:
        return
    import json
    os.makedirs(os.path.dirname(os.path.abspath(path)), exist_ok=True)
    with open(path, "w") as f:
        json.dump(mod.REPORT, f, indent=1)
