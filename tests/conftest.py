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


def _trace_build_loaded() -> bool:
    return os.path.basename(os.environ.get("MOE_LIB_PATH", "")) == "libmoedc_trace.so"


@pytest.fixture(autouse=True)
def _trace_every_test():
    """When MOE_TRACE_EVERY_TEST=1 and the session runs on the build with
    trace records (MOE_LIB_PATH names libmoedc_trace.so), every test runs
    with a record buffer attached, and afterwards its launches must be
    consistent: each CTA of a launch recorded exactly once, start <= end,
    and stream order kept (no CTA of a launch starts before every CTA of the
    previous one has started, none ends before the previous one ended)."""
    if os.environ.get("MOE_TRACE_EVERY_TEST") != "1" or not _trace_build_loaded():
        yield
        return
    import torch
    if not torch.cuda.is_available():
        yield
        return
    from trace_checks import check_launches
    from combine_topk_ids_scan_b200 import trace as T
    with T.Tracer(capacity=1 << 20) as tr:
        yield
    check_launches(tr)
