import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))
for p in (ROOT, HERE):
    if p not in sys.path:
        sys.path.insert(0, p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    # GPU tests fail loudly on a machine without a GPU rather than pass silently;
    # on such a machine they are selected out with -m "not gpu".
    pass


@pytest.fixture(scope="session")
def lib():
    """The CUDA C-ABI library, loaded through the Python binding."""
    from compressed_latent_grouped_b200 import binding
    return binding.load()
