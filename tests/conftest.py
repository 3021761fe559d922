import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def golden():
    import json
    with open(os.path.join(ROOT, "tests", "golden",
                           "worked_examples.json")) as f:
        return json.load(f)


@pytest.fixture(scope="session")
def pkv():
    """The package with libpagedkv.so built (nvcc works without a GPU)."""
    from paged_kv_cache_383_b200 import build_lib
    build_lib.build()
    import paged_kv_cache_383_b200 as pkv_mod
    from paged_kv_cache_383_b200 import _lib
    _lib.load()
    return pkv_mod
