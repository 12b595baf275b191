"""Host logic the kernels rely on, checked without a GPU: the heaviest-first grid order of
the attention kernels (grid_item) covers every (batch, head) tile exactly once, keeps each
group of heads contiguous and puts every head's heaviest tile first; the workspace layout
(ws_layout) is aligned and disjoint and does not wrap at the largest accepted problems.
tests/csrc/host_layout_check.cpp includes csrc/common.h and runs on the host compiler."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs a host C++ compiler")
def test_grid_order_and_workspace_layout(tmp_path):
    exe = tmp_path / "host_layout_check"
    subprocess.run(["g++", "-std=c++17", "-O1", "-D__host__=", "-D__device__=",
                    "-I" + os.path.join(ROOT, "rope_attention_fwd_b200", "csrc"),
                    os.path.join(ROOT, "tests", "csrc", "host_layout_check.cpp"),
                    "-o", str(exe)], check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr
