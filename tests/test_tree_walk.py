"""The tensor-core epilogue's storage plan for the tree (CPU only): the
library's own per-leaf operation codes, compiled for the host from
device_common.cuh, replayed on symbolic values for every leaf count up to
1100 (tests/tree_walk_check.cu).  The replay must rebuild the halving tree (and
the baseline's left-to-right chain) exactly, with at most one pending single
leaf (taken by the next leaf), one pending 2-leaf and one 3-4-leaf value, and
an L2 stack no deeper than the bound the host sizes the scratch with."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def _nvcc():
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    return None


@pytest.mark.skipif(_nvcc() is None, reason="needs nvcc")
def test_epilogue_storage_plan_rebuilds_the_tree(tmp_path):
    exe = str(tmp_path / "tree_walk_check")
    subprocess.check_call([_nvcc(), "-std=c++17", "-O1", "-I", os.path.join(ROOT, "include"),
                           "-I", os.path.join(ROOT, "invariant_tree_ordered_b200", "csrc"),
                           os.path.join(HERE, "tree_walk_check.cu"), "-o", exe])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "tree walk ok" in r.stdout
