"""The bounds-checking debug build (libstq1_debug.so) on the GPU (needs a B200).

The debug build checks the indices its kernels read (routing tables, pair
ids, shared-memory windows and copy destinations, gather and combine rows)
and records STQ1_DEV_BOUNDS instead of accessing out of range.  A process of
its own imports the package with STQ1_DEBUG=1, so the debug build is the one
loaded.  It then runs tests/debug_build_cases.py:
- the bounds self-test (a failed check is reported, the context survives);
- small parity cases against the CPU oracle on every kernel path, each of
  which must leave the device error word at zero, so no check fires on valid
  input.
"""

import os
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_build_passes_the_parity_cases_without_a_bounds_report():
    from sub_bit_sparse_b200 import build as b
    b.build(debug=True)                                # no-op when up to date
    env = dict(os.environ, STQ1_DEBUG="1", PYTHONPATH=ROOT)
    res = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_build_cases.py")], cwd=ROOT, env=env,
                         capture_output=True, text=True, timeout=900)
    assert res.returncode == 0 and res.stdout.strip().endswith("OK"), res.stdout[-3000:] + res.stderr[-3000:]


def test_release_build_reports_nothing_from_the_bounds_self_test():
    import sub_bit_sparse_b200 as stq1
    if stq1.DEBUG_BUILD:
        pytest.skip("this process loaded the debug build")
    assert stq1.build_flags() == 0
    assert stq1.selftest_bounds(12, 10) == 0           # no checks in the release build
    assert stq1.status() == 0
