import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200) and the built liblsa.so")


@pytest.fixture(scope="session")
def lib():
    from sparse_attention_03_b200 import lsa
    return lsa.load()
