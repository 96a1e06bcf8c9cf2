"""The index-checked build (libm3_debug.so, compiled with
-DM3_DEBUG_BOUNDS=1) on a B200.

* The check itself: with index >= limit the self-test's store is skipped
  and recorded (site 9001, the index and the limit); with index < limit it
  goes through and nothing is recorded.
* The small-shape parity tests of every path -- the tile and persistent
  tensor-core prefills (ranks 1, 2, 4, 8, segments, hand-offs, carries), the
  float32 SIMT prefill and the segment combine, the decode step, rope, the
  backward pass, the phase interventions, the transition variants and the
  allocation-free entry point -- run again under the checked library, each
  against the fp64 oracle as usual; the conftest fixture fails any test whose
  kernels recorded a failed check.  The full-size sampled cases are left to
  the release runs.

Both run as child processes (the package picks the library at import).
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ENV = dict(os.environ, M3_DEBUG_BOUNDS="1", PYTHONPATH=ROOT)


def _child(args, timeout):
    return subprocess.run([sys.executable, *args], capture_output=True, text=True, env=ENV, cwd=ROOT,
                          timeout=timeout)


def test_failed_check_skips_the_access_and_is_recorded():
    code = (
        "import torch, selective_state_space_m3_b200 as m3\n"
        "assert m3.LIB_PATH.endswith('libm3_debug.so')\n"
        "r = m3.m3_debug_bounds_report(clear=True)\n"
        "assert r['enabled'] == 1 and r['failures'] == 0, r\n"
        "buf = torch.zeros(64, device='cuda')\n"
        "m3.m3_selftest_bounds_check(buf, 40, 32)\n"
        "r = m3.m3_debug_bounds_report(clear=True)\n"
        "assert r == {'enabled': 1, 'failures': 1, 'site': 9001, 'index': 40, 'limit': 32}, r\n"
        "assert float(buf.abs().sum()) == 0.0, 'the checked store was not skipped'\n"
        "m3.m3_selftest_bounds_check(buf, 5, 32)\n"
        "r = m3.m3_debug_bounds_report(clear=True)\n"
        "assert r['failures'] == 0, r\n"
        "assert float(buf[5]) == 1.0 and float(buf.sum()) == 1.0\n"
        "print('selftest ok')\n")
    r = _child(["-c", code], 300)
    assert r.returncode == 0 and "selftest ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]


SMALL_TESTS = [
    "tests/test_parity_gpu.py", "tests/test_degenerate_gpu.py", "tests/test_bwd_gpu.py",
    "tests/test_phase_gpu.py", "tests/test_variants_gpu.py", "tests/test_scan_ws_gpu.py",
    "tests/test_zz_no_alloc.py",
]
# full-size cases, and the graph-timed decode loops, stay with the release runs
DESELECT = "not full_size and not sampled and not 1000_steps and not decode_workload and not bounded_wait"


def test_small_parity_suite_under_index_checks():
    r = _child(["-m", "pytest", *SMALL_TESTS, "-q", "-x", "-m", "gpu", "-k", DESELECT, "-p", "no:cacheprovider"],
               1500)
    tail = r.stdout[-3000:] + r.stderr[-3000:]
    print(tail)
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "failed" not in r.stdout.splitlines()[-1], tail
