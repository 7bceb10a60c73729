"""GPU: the bounds-checked build (libmla_debug.so, MLA_DEBUG) on the small and ragged workloads.

Runs, in a child process that loads the debug build through MLA_LIBRARY: the parity tests of the
small, wrapped, ragged, sink and batched workloads and the commit tests - every sync there also
checks the guard bands after each buffer and the status word that the bounds checks write - and
tests/debug_build_checks.py, which shows that a write into a guard band and an out-of-range row
in a kernel are both reported (neither faults: the row is caught before any access).
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_build_parity_and_checks():
    from mla_latent_kv_window_b200 import build
    lib = build.build(debug=True)
    env = dict(os.environ, MLA_LIBRARY=lib)
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
           os.path.join(ROOT, "tests", "debug_build_checks.py"),
           os.path.join(ROOT, "tests", "test_gpu_commit.py"),
           os.path.join(ROOT, "tests", "test_gpu_parity.py"),
           "-k", "(debug or commit or tiny or wrap or empty or partial or ragged or batched or repeated or invalid)"
           " and not 30_layers and not full_size and not sampled"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
