"""The bounds-check build of the library (libmoe_debug.so, compiled with
-DMOE_DEBUG_BOUNDS and selected by MOE_BOUNDS_CHECK=1).

Its kernels check the indices they take from other kernels or from the caller
and, where one fails, set MOE_STATUS_BOUNDS and skip the access.  The checks
must not change a result: the same layer calls through both builds give
bit-identical outputs and a clean status word.  And one invalid input (a
combine row past the rows it is given) is caught: the status word says so and
the row adds nothing.  Each build runs in its own process (tests/bounds_child.py).
"""
import os
import subprocess
import sys

import pytest
import torch

import sparse_mixture_experts_10_b200 as moe
from sparse_mixture_experts_10_b200 import build as moe_build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _child(tmp_path, bounds_check: bool):
    out = tmp_path / ("debug.pt" if bounds_check else "release.pt")
    env = dict(os.environ, MOE_BOUNDS_CHECK="1" if bounds_check else "0")
    r = subprocess.run([sys.executable, "-m", "tests.bounds_child", str(out)], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    return torch.load(out)


@pytest.fixture(scope="module")
def runs(tmp_path_factory):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    moe_build.build()
    moe_build.build(bounds_check=True)
    tmp = tmp_path_factory.mktemp("bounds")
    return _child(tmp, False), _child(tmp, True)


def test_each_build_was_loaded(runs):
    rel, dbg = runs
    assert rel["lib"].endswith("libmoe.so") and dbg["lib"].endswith("libmoe_debug.so")


def test_checks_change_no_result(runs):
    rel, dbg = runs
    names = [k for k in rel if k != "lib"]
    assert len(names) >= 9 and set(names) <= set(dbg)
    for k in names:
        (y_r, st_r), (y_d, st_d) = rel[k], dbg[k]
        assert st_r == 0 and st_d == 0, (k, st_r, st_d)
        assert torch.isfinite(y_r).all(), k
        assert torch.equal(y_r, y_d), (k, float((y_r - y_d).abs().max()))


def test_out_of_range_combine_row_is_caught(runs):
    _, dbg = runs
    y, st = dbg["combine_bad_row"]
    assert st & moe.MOE_STATUS_BOUNDS
    # the bad row (whose entries are 1e6) was skipped: every output stays small
    assert float(y.abs().max()) < 100.0
    assert torch.isfinite(y).all()
