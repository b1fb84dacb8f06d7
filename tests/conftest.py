import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size configuration")


@pytest.fixture(scope="session")
def cuda_ok():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return True


def pytest_sessionfinish(session, exitstatus):
    """With PARITY_RECORD=<path>, write the errors the parity tests measured."""
    path = os.environ.get("PARITY_RECORD")
    if not path:
        return
    try:
        import json

        import parity_util
        with open(path, "w") as f:
            json.dump(parity_util.records(), f, indent=1, sort_keys=True)
    except Exception:       # the record is a by-product; never fail the run on it
        pass
