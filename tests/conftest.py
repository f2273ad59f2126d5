import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workloads")


@pytest.fixture(scope="session")
def cuda_ok():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return True


def pytest_sessionfinish(session, exitstatus):
    # parity records (strict-bound ratios, envelope use, FP8 code agreement)
    path = os.environ.get("MOE_PARITY_LOG")
    if not path:
        return
    try:
        import json

        from helpers import PARITY_LOG
    except Exception:
        return
    with open(path, "w") as f:
        json.dump(PARITY_LOG, f, indent=1)
