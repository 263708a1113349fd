"""The build with per-CTA trace records (libmoedc_trace.so, -DMOE_TRACE),
in child processes whose MOE_LIB_PATH names it: the trace cases
(tests/trace_child_cases.py), then the parity suite's layout, payload,
padding, random, cluster-size, atom-layout, workload, backward, SwiGLU and
peer-store cases with a record buffer attached around every test -- every
result must still match the oracle, and every test's records must be
consistent (tests/trace_checks.py)."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
SUBSET = ("edge_case or padding or random or cluster_sizes or swizzled or workload_full "
          "or backward or swiglu_quant_parity or permute_to_peers or grouped_gemm")


def _run(args, env):
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           *args]
    r = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    last = r.stdout.strip().splitlines()[-1]
    assert " passed" in last and "error" not in last and "skipped" not in last, last


def test_trace_build_cases_and_parity_with_records():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from combine_topk_ids_scan_b200 import build
    env = dict(os.environ, MOE_LIB_PATH=build.build(trace=True))
    _run([os.path.join(HERE, "trace_child_cases.py")], env)
    _run([os.path.join(HERE, "test_gpu_parity.py"), "-k", SUBSET],
         dict(env, MOE_TRACE_EVERY_TEST="1"))
