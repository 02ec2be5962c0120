import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


import pytest  # noqa: E402


@pytest.fixture(scope="session")
def calibatt_lib():
    """Builds libcalibatt.so if a source is newer than it, then loads the binding."""
    from calibrated_block_sparse_calibatt_b200 import build as b

    b.build()
    from calibrated_block_sparse_calibatt_b200 import calibatt

    return calibatt
