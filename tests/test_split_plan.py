"""The decode kernel's split-mode plan (csrc/q4_0_split_plan.h), checked on
the CPU: tests/split_plan_check.cpp walks each plan the way the kernel's CTAs
walk it and checks that every stage of every item is worked exactly once, that
the split items open every list of their cluster in the same order, and that
the busiest CTA's load stays within greedy list scheduling's bound.  It runs
the decoder-layer, flow-head and GEMV shape sets at the cluster sizes the
launcher uses, edge cases, and 400 seeded random problem sets."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_weight_only_matmul_b200", "csrc")


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_split_plan_walk(tmp_path):
    exe = str(tmp_path / "split_plan_check")
    subprocess.run(["g++", "-std=c++17", "-O1", "-Wall", "-Werror", f"-I{CSRC}",
                    os.path.join(ROOT, "tests", "split_plan_check.cpp"), "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok ") and int(r.stdout.split()[1]) >= 400, r.stdout
