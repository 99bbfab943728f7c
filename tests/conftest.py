import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (run with -m gpu)")
    config.addinivalue_line("markers", "slow: long CPU test")


@pytest.fixture(scope="session", autouse=True)
def _built_cpu_libs():
    """The CPU-side helpers (generator, oracle) are built here if a build has not run yet."""
    import oracle
    import synth

    if not os.path.exists(os.path.join(ROOT, "synth", "libhqsynth.so")):
        synth.build()
    if not os.path.exists(os.path.join(ROOT, "oracle", "libhq_oracle.so")):
        oracle.build()
    yield
