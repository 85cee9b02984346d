import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workload; minutes of CPU oracle time")


def _stale(lib_path, src_dir):
    import glob
    if not os.path.exists(lib_path):
        return True
    t = os.path.getmtime(lib_path)
    srcs = glob.glob(os.path.join(src_dir, "*.cu")) + glob.glob(os.path.join(src_dir, "*.cuh")) + \
        glob.glob(os.path.join(src_dir, "*.h")) + [os.path.join(ROOT, "include", "la.h")]
    return any(os.path.getmtime(s) > t for s in srcs)


@pytest.fixture(scope="session")
def lib_path():
    """Path of the CUDA library, (re)built in-tree if missing or older than its sources."""
    from linear_attention_11_b200 import build as b
    if _stale(b.OUT, b.CSRC):
        b.build()
    return b.OUT


@pytest.fixture(scope="session")
def la(lib_path):
    """The Python binding with the library loaded."""
    import linear_attention_11_b200 as la_mod
    la_mod.load_library(lib_path)
    return la_mod
