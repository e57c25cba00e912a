"""The bounds-checked build of the library (-DNVFP4HS_CHECKS: every global
address of the per-step kernels checked against its buffer's extent) runs the
edge-case and small parity tests green with no failed check.  Needs a B200."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_checked_build_runs_the_edge_cases_clean():
    from block_scale_search_b200 import _build
    lib = _build.build(checked=True)
    env = dict(os.environ, NVFP4HS_LIB=lib)
    cmd = [sys.executable, "-m", "pytest", "-q", "-m", "gpu and not slow", "-p", "no:cacheprovider",
           os.path.join(ROOT, "tests", "test_gpu_edges.py"),
           os.path.join(ROOT, "tests", "test_gpu_parity.py")]
    out = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    tail = out.stdout[-3000:] + out.stderr[-2000:]
    assert out.returncode == 0, tail
    assert "bounds checks: 0 failed" in out.stdout, tail
