import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
# tests/test_oracle_mutations.py runs the oracle pins against a mutated copy of the oracle
_ORACLE_OVERRIDE = os.environ.get("RRA_ORACLE_OVERRIDE")
if _ORACLE_OVERRIDE:
    sys.path.insert(0, _ORACLE_OVERRIDE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")
