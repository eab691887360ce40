import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on CPU")


def pytest_collection_modifyitems(config, items):
    # a GPU test on a machine without a GPU is an error, not a skip: the
    # product path has no CPU fallback.
    pass


@pytest.fixture(scope="session")
def tiny_weights():
    import synth
    return synth.make_weights(synth.TINY, 0)


@pytest.fixture(scope="session")
def tiny_prompt():
    import synth
    return synth.make_prompt(synth.TINY, 16, 0)
