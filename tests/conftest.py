import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on CPU")


@pytest.fixture(scope="session")
def libmla():
    """Builds libmla.so in-tree if needed and returns the binding module."""
    from mla_latent_kv_26_b200 import build

    build.build()
    from mla_latent_kv_26_b200 import binding

    return binding
