"""Host test of the decode engine's ring schedule (csrc/engine_sched.h, plain C++).

The producer warp and the consumer groups of the decode engine must agree exactly on
which tile and K-chunk every ring stage holds: a disagreement would pair a consumer with
the wrong weights or leave a barrier waiting.  tests/engine_sched_check.cpp enumerates
the producer's sequence and each group's closed-form stage list for 49 x 16 shapes and
checks them against each other; this test builds and runs it with the host compiler.
"""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "ternary_bitlinear_quantized_b200", "csrc")


def test_engine_schedule_covers_every_stage_once_and_groups_agree(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    exe = str(tmp_path / "sched_check")
    subprocess.run([cxx, "-std=c++17", "-O1", "-Wall", "-I", CSRC, os.path.join(HERE, "engine_sched_check.cpp"),
                    "-o", exe], check=True, capture_output=True, text=True)
    res = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stdout + res.stderr
    assert res.stdout.startswith("OK"), res.stdout
