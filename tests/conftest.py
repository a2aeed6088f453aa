import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session", autouse=True)
def _built_libraries():
    """Make sure the CPU-side libraries exist (cheap when they are already built)."""
    import oracle.build
    import synth.build
    if not os.path.exists(os.path.join(ROOT, "synth", "libsynth.so")):
        synth.build.build(cuda=False)
    if not os.path.exists(os.path.join(ROOT, "oracle", "liboracle.so")):
        oracle.build.build()
