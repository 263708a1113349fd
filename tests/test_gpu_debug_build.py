"""The build with device index checks (libmoedc_debug.so, -DMOE_DEBUG_CHECKS):
its kernels check every computed row index and block-scale offset before use
and record an out-of-range one instead of touching memory.  The parity
suite's layout, payload, padding, random, SwiGLU and backward cases run on
that build in a child process (MOE_LIB_PATH selects it); every result must
still match the oracle and, at the end of the session, no check may have
fired (tests/conftest.py asserts moe_debug_violations() == 0)."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
SUBSET = ("edge_case or padding or random or cluster_sizes or swizzled or workload_full "
          "or backward or swiglu_quant_parity")


def test_parity_cases_on_the_debug_build():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from combine_topk_ids_scan_b200 import build
    path = build.build(debug=True)
    env = dict(os.environ, MOE_LIB_PATH=path)
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           os.path.join(HERE, "test_gpu_parity.py"), "-k", SUBSET]
    r = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "error" not in r.stdout.splitlines()[-1]
