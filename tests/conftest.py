import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built libasp.so")


def pytest_collection_modifyitems(config, items):
    # GPU tests fail loudly rather than skip when selected without a device:
    # a silent skip would read as a pass on the GPU run.
    pass
