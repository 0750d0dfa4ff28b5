"""The checked build (libjsv_checked.so, every computed global index compared
with its buffer's extent, a miss written to the status word as
JSV_ERR_BOUNDS) runs the edge, parity and f-row GPU tests green: on valid
inputs no check fires (the tests assert a zero status word after their
calls) and the results still match the oracle."""
import os
import subprocess
import sys
from pathlib import Path

import pytest

from tree_verification_jsv_b200 import build as jbuild

ROOT = Path(__file__).resolve().parents[1]

pytestmark = pytest.mark.gpu


def test_checked_build_runs_the_gpu_tests_clean():
    jbuild.build(checked=True)
    env = dict(os.environ, JSV_LIBRARY="checked")
    probe = subprocess.run([sys.executable, "-c",
                            "from tree_verification_jsv_b200 import jsv; print(jsv.jsv_build_flags())"],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert probe.returncode == 0 and probe.stdout.strip() == "1", probe.stdout + probe.stderr
    files = ["tests/test_gpu_edge.py", "tests/test_gpu_parity.py", "tests/test_gpu_qkv_rope.py",
             "tests/test_gpu_tree_build.py"]
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-p", "no:cacheprovider", *files],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
