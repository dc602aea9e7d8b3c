"""The diagnostic build (index checks on every kernel write, guard words around every engine
buffer) runs both kernels in parity with the oracle and reports a changed guard word (GPU
test; the checks run in a child process, since a process loads one build of the library)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_build_parity_and_guard_words():
    from bandwidth_bound_stream_b200 import build
    build.build_kie(variant="debug")
    env = dict(os.environ, KIE_VARIANT="debug")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_variant_run.py")], env=env, cwd=ROOT,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "guard words: a changed word is reported" in r.stdout
