"""Planted mistakes in the oracle (CPU only).

Each case copies the oracle and the pin tests into a scratch directory,
makes one plausible mistake in the copy of oracle.c -- a dropped term, a
wrong sign, index, bound or constant, a transposed operand, a swapped nibble
or bit order -- rebuilds it there and runs the pin tests of the function it
touches: they must fail.  A control copy with no change must pass the same
tests, so a failure is the planted mistake's and not the harness's.  Nothing
here touches the oracle in place or the CUDA library.
"""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (what the mistake is, text in oracle.c, replacement, pin test file)
CASES = [
    ("bf16: ties away from zero instead of to even",
     "u += 0x7FFFu + ((u >> 16) & 1u);", "u += 0x7FFFu;", "test_oracle_formats.py"),
    ("E4M3: subnormal step 2^-8 instead of 2^-9",
     "code = (uint32_t)rne_int(a * 512.0);", "code = (uint32_t)rne_int(a * 256.0);",
     "test_oracle_formats.py"),
    ("E4M3: exponent bias 8 instead of 7",
     "code = (uint32_t)(((e + 7) << 3) | (int)m);", "code = (uint32_t)(((e + 8) << 3) | (int)m);",
     "test_oracle_formats.py"),
    ("layout: rows of an expert in reverse pair order",
     "row = off[e] + r;", "row = off[e + 1] - 1 - r;", "test_oracle_layout.py"),
    ("layout: segment displacement is the inclusive cumsum",
     "start = off[s * L];", "start = off[(s + 1) * L];", "test_oracle_layout.py"),
    ("layout: id E accepted as an expert",
     "if (e < 0 || e >= E) {", "if (e < 0 || e > E) {", "test_oracle_layout.py"),
    ("layout: capacity mode keeps Ce + 1 pairs",
     "row = (r < Ce) ? (int64_t)e * Ce + r : -1;", "row = (r <= Ce) ? (int64_t)e * Ce + r : -1;",
     "test_oracle_layout.py"),
    ("FP8: block scale from the E4M3 max of another variant (240)",
     "float sc = amax / 448.0f;", "float sc = amax / 240.0f;", "test_oracle_permute_combine.py"),
    ("NVFP4 dispatch: nibble order swapped",
     "        qd[m] = (uint8_t)(lo | (hi << 4));", "        qd[m] = (uint8_t)(hi | (lo << 4));",
     "test_oracle_permute_combine.py"),
    ("MXFP4 dispatch: nibble order swapped",
     "qd[i / 2] |= (uint8_t)(i % 2 ? c << 4 : c);", "qd[i / 2] |= (uint8_t)(i % 2 ? c : c << 4);",
     "test_oracle_mx_fp6.py"),
    ("MXFP4 dispatch: emax 3 instead of 2",
     "const uint8_t sc = mx_scale_code(amax, 2);", "const uint8_t sc = mx_scale_code(amax, 3);",
     "test_oracle_mx_fp6.py"),
    ("combine: gate index transposed",
     "acc = fmaf(gates[(int64_t)t * k + j], x, acc);",
     "acc = fmaf(gates[(int64_t)j * N + t], x, acc);", "test_oracle_permute_combine.py"),
    ("dispatch backward: wrong sign",
     "acc = acc + orc_bf16_to_f32(grad_out[(int64_t)s * H + h]);",
     "acc = acc - orc_bf16_to_f32(grad_out[(int64_t)s * H + h]);", "test_oracle_backward.py"),
    ("combine backward: gate dropped from the row gradient",
     "orc_bf16_from_f32(gates[p] * g);", "orc_bf16_from_f32(g);", "test_oracle_backward.py"),
    ("exp: the r^5/5! term dropped",
     "p = fmaf(p, r, 8.33333333e-03f);", "p = fmaf(p, r, 0.0f);", "test_oracle_swiglu.py"),
    ("silu: e^g instead of e^-g",
     "return g / (1.0f + orc_exp(-g));", "return g / (1.0f + orc_exp(g));", "test_oracle_swiglu.py"),
    ("SwiGLU MXFP8: emax 7 instead of 8",
     "const int32_t emax = format == 1 ? 8 : 2;", "const int32_t emax = format == 1 ? 7 : 2;",
     "test_oracle_swiglu.py"),
    ("atom layout: row index terms transposed",
     "int64_t inner = (m % 32) * row_stride + ((m / 32) % 4) * 4 + c % atom_cols;",
     "int64_t inner = ((m / 32) % 4) * row_stride + (m % 32) * 4 + c % atom_cols;",
     "test_oracle_scale_layout.py"),
    ("pre-multiplied dispatch: the next pair's gate",
     "out[(int64_t)s * H + h] = orc_bf16_from_f32(gates[p] * x);",
     "out[(int64_t)s * H + h] = orc_bf16_from_f32(gates[(p + 1) % ((int64_t)N * k)] * x);",
     "test_oracle_premultiplied.py"),
    ("FP6 packing: codes in reverse bit order",
     "w |= (uint32_t)(codes[4 * g + i] & 0x3F) << (6 * i);",
     "w |= (uint32_t)(codes[4 * g + i] & 0x3F) << (18 - 6 * i);", "test_oracle_mx_fp6.py"),
]


def _sandbox(dst, old=None, new=None):
    ign = shutil.ignore_patterns("*.so", "*.so.tmp*", "__pycache__")
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(dst, "oracle"), ignore=ign)
    shutil.copytree(os.path.join(ROOT, "tests"), os.path.join(dst, "tests"), ignore=ign)
    pkg = os.path.join(dst, "combine_topk_ids_scan_b200")
    os.makedirs(pkg)
    for f in ("__init__.py", "inputs.py"):
        shutil.copy(os.path.join(ROOT, "combine_topk_ids_scan_b200", f), pkg)
    if old is not None:
        path = os.path.join(dst, "oracle", "oracle.c")
        src = open(path).read()
        assert src.count(old) == 1, f"planted text must occur once: {old!r}"
        open(path, "w").write(src.replace(old, new))


def _run_pins(dst, test_file):
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
           "-m", "not gpu", os.path.join("tests", test_file)]
    r = subprocess.run(cmd, cwd=dst, capture_output=True, text=True, timeout=600)
    return r.returncode, (r.stdout.strip().splitlines() or [""])[-1]


@pytest.mark.slow
def test_pins_catch_planted_mistakes(tmp_path):
    files = sorted({c[3] for c in CASES})
    jobs = [("control", None, None, f) for f in files] + CASES
    dirs = []
    for i, (_, old, new, _) in enumerate(jobs):
        d = str(tmp_path / f"case{i}")
        _sandbox(d, old, new)
        dirs.append(d)
    with cf.ThreadPoolExecutor(max_workers=min(6, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda a: _run_pins(*a), [(d, j[3]) for d, j in zip(dirs, jobs)]))
    bad = []
    for (what, old, _, f), (rc, tail) in zip(jobs, results):
        if old is None and rc != 0:
            bad.append(f"control copy fails {f}: {tail}")
        if old is not None and rc == 0:
            bad.append(f"not caught by {f}: {what}")
    assert not bad, "\n".join(bad)


def test_output_guard_reports_overruns_and_keeps_poison(orc):
    """The poisoned, guarded output buffers themselves: a call that writes
    past the end of an output (here 8 bf16 values into room for 4, i.e.
    into the 64-byte guard that follows it) raises, and an element the call
    does not write keeps the poison byte."""
    import numpy as np
    x = np.arange(8, dtype=np.float32)
    o = orc._Outs()
    out = o(4, np.uint16)
    orc.lib().orc_bf16_from_f32_n(orc._p(x), orc._p(out), 8)
    with pytest.raises(RuntimeError, match="past the end"):
        o.check("overrun")
    o = orc._Outs()
    out = o(4, np.uint16)
    orc.lib().orc_bf16_from_f32_n(orc._p(x), orc._p(out), 3)
    o.check("short write")
    assert int(out[3]) == orc._POISON * 0x101 and int(out[2]) == 0x4000
