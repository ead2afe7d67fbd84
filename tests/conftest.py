import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# A child run of tests/test_oracle_mutants.py: plant the named mistake in the
# oracle before any test module imports it.
_MUTANT = os.environ.get("VELOX_ORACLE_MUTANT")
if _MUTANT is not None:
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    from oracle_mutants import apply_mutant
    apply_mutant(int(_MUTANT))


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity case")


def gpu_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def lib():
    """The CUDA library binding; GPU tests fail loudly if it cannot load."""
    import routed_block_sparse_b200 as rbs
    return rbs
