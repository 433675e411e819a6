import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def tiny_cfg():
    from persistent_megakernel_interpreter_b200.config import TINY
    return TINY


@pytest.fixture(scope="session")
def tiny_weights(tiny_cfg):
    from persistent_megakernel_interpreter_b200.inputs import make_weights
    return make_weights(tiny_cfg, seed=0)


@pytest.fixture(scope="session", autouse=True)
def _built_libraries():
    """Compile libmk.so (nvcc, sm_100a) and the oracle if their sources changed."""
    from persistent_megakernel_interpreter_b200.build import build_library
    import oracle
    build_library()
    oracle.build()
