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


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print the GPU parity records (rows checked, mass error, kept-list mismatches excused by
    the 1e-4 boundary rule, attention error) so they reach the log without -s."""
    mod = sys.modules.get("parity")
    recs = getattr(mod, "RECORDS", None) if mod else None
    if not recs:
        return
    tr = terminalreporter
    tr.section("parity against the fp64 oracle")
    for r in recs:
        fields = " ".join(f"{k}={v:.3g}" if isinstance(v, float) else f"{k}={v}"
                          for k, v in r.items() if k not in ("label", "when"))
        tr.write_line(f"{r['label']}: {fields}")
