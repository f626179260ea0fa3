"""The prefill kernel's pair builder re-cuts block-sparse KV lists into tiles
of up to 128 keys made of at most two contiguous segments.  This compiles the
host planner with a small C++ checker (tests/plan_recut_check.cpp) and runs it
over random block maps and the 24 x 1040 frame map: every pair's tiles must
cover exactly the keys of the original plan, each allowed by the map."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_io_aware_sm_b200", "csrc")


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_two_segment_recut_covers_the_plan(tmp_path):
    exe = tmp_path / "recut_check"
    subprocess.run(["g++", "-O2", "-std=c++17", "-I", CSRC, os.path.join(ROOT, "tests", "plan_recut_check.cpp"),
                    os.path.join(CSRC, "plan.cpp"), "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "bad 0" in r.stdout


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_pair_plans_keep_the_kernel_invariants(tmp_path):
    """tests/plan_pairs_check.cpp: over random shapes of every mask kind and
    both pairing modes, each Q tile runs exactly once, each slot visits
    exactly its own keys (slot A a prefix of the shared list), partial flags
    are per slot, and the visit order is longest first."""
    exe = tmp_path / "pairs_check"
    subprocess.run(["g++", "-O2", "-std=c++17", "-I", CSRC, os.path.join(ROOT, "tests", "plan_pairs_check.cpp"),
                    os.path.join(CSRC, "plan.cpp"), "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("bad 0")
