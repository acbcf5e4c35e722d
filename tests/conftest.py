import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    # A GPU test run on a machine without a GPU is a setup error, not a skip:
    # the product path has no CPU fallback.  Tests select with -m gpu / -m "not gpu".
    pass
