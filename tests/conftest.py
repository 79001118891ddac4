import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


@pytest.fixture(scope="session")
def cuda_dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def pytest_sessionfinish(session, exitstatus):
    """With M3_PARITY_REPORT set, write the errors of every GPU comparison to that file."""
    path = os.environ.get("M3_PARITY_REPORT")
    gc = sys.modules.get("gpu_common")
    if path and gc is not None and gc.ERRORS:
        import json
        with open(path, "w") as f:
            json.dump(gc.ERRORS, f, indent=1, sort_keys=True)
