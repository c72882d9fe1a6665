"""The lane plan of packed sequences (csrc/lanes.h) and the item order built from it, checked by a
host program compiled with g++ (see tests/lanes_check.cpp for what it checks)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "gated_delta_rule_82_b200", "csrc")


def test_lane_plan_and_item_order(tmp_path):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not available")
    exe = str(tmp_path / "lanes_check")
    subprocess.run([gxx, "-O2", "-std=c++17", "-I", CSRC, os.path.join(HERE, "lanes_check.cpp"),
                    "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "failures 0" in r.stdout
