import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built engine library")
    config.addinivalue_line("markers", "slow: long CPU oracle run")


@pytest.fixture(scope="session")
def tiny_weights():
    from synth import TINY, make_weights
    return make_weights(TINY, seed=0)


@pytest.fixture(scope="session")
def tiny_weights_xavier():
    from synth import TINY, make_weights
    return make_weights(TINY, seed=0, xavier=True)
