import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload (minutes of CPU time for the oracle)")


def build_library():
    """Compile libsgd.so if needed (by path: the package import needs the library) and import it."""
    import runpy
    runpy.run_path(os.path.join(ROOT, "sparse_gqa_decode_b200", "build.py"), run_name="sgd_build")["build"]()
    import sparse_gqa_decode_b200
    return sparse_gqa_decode_b200


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")
