import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session", autouse=True)
def _device_index_checks():
    """When the session runs on the build with device index checks
    (MOE_LIB_PATH names libmoedc_debug.so), no kernel may have recorded an
    out-of-range index by the end of it."""
    yield
    if os.path.basename(os.environ.get("MOE_LIB_PATH", "")) != "libmoedc_debug.so":
        return
    from combine_topk_ids_scan_b200 import binding as B
    if B._lib is None:
        return
    v = B.debug_violations(reset=True)
    assert v == 0, f"device index checks recorded violations {v:#x} (-1: not a debug build)"
