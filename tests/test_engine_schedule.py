"""Host test of the decode engine's stage geometry (csrc/engine_sched.h, plain C++).

The producer warp and the consumer warps of the decode engine walk the same stage order;
a stage that does not fit its slot, a chunk that is not whole steps, or a read past a
buffer would pair consumers with the wrong bytes.  tests/engine_sched_check.cpp plans
every row length up to 49152 for 1..16 tokens and walks the stage order for 0..40 tiles;
this test builds and runs it with the host compiler.
"""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "ternary_bitlinear_quantized_b200", "csrc")


def test_engine_stage_geometry_fits_and_covers_every_stage_once(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    exe = str(tmp_path / "sched_check")
    subprocess.run([cxx, "-std=c++17", "-O1", "-Wall", "-I", CSRC, os.path.join(HERE, "engine_sched_check.cpp"),
                    "-o", exe], check=True, capture_output=True, text=True)
    res = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stdout + res.stderr
    assert res.stdout.startswith("OK"), res.stdout
