import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built libsa.so")
    config.addinivalue_line(
        "markers", "slow: full-size workload; needs a B200 with the full workload resident")
