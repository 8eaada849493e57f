"""The bounds-checked build (libgs_check.so, compiled with GS_CHECK) on the
parity cases that reach every binning and blend path at small sizes: the tiny
and ragged scenes, a splat covering every tile, saturating stacks, both
binning strategies over 1 to 66 049 tiles, lists past 8 192 entries, depth
ties and the capacity error.  Its kernels test every gather and scatter
index against its array's bound and record GS_ERR_BOUNDS in the status word
instead of accessing out of range; the parity tests assert that the status
word stays clear and that results still match the oracle.  compute-sanitizer
is not available, so this stands in for it.

The cases run in a child process that loads the checked library
(GS_LIBRARY=libgs_check.so)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CASES = "tiny or ragged or huge or saturating or bin_and_sort"


def _child_env():
    return dict(os.environ, GS_LIBRARY="libgs_check.so")


def test_checked_library_is_the_one_loaded():
    from gaussian_splatting_differentiable_tile_b200 import build as B
    B.build(check=True)
    r = subprocess.run([sys.executable, "-c", "import gaussian_splatting_differentiable_tile_b200 as G; "
                        "print(G.lib()._name)"], cwd=ROOT, env=_child_env(), capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip().endswith("libgs_check.so"), r.stdout


def test_checked_build_passes_the_parity_cases():
    from gaussian_splatting_differentiable_tile_b200 import build as B
    B.build(check=True)
    cmd = [sys.executable, "-m", "pytest", "-m", "gpu", "-x", "-q", "-p", "no:cacheprovider",
           "tests/test_gpu_parity.py", "-k", CASES]
    r = subprocess.run(cmd, cwd=ROOT, env=_child_env(), capture_output=True, text=True, timeout=1200)
    tail = r.stdout[-3000:] + r.stderr[-2000:]
    print(tail)
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and " failed" not in r.stdout, tail
