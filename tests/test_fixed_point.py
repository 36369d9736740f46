"""Host test of the integer fixed-point terms (csrc/fixed_point.h, plain C++): every term of
the exact sums behind RMSNorm's mean(x^2) and the absmean scale must equal the fp64 route
rint(ldexp(v * v, e)) bit for bit.  tests/fixed_point_check.cpp checks millions of random
fp32 values (all exponents, subnormals included), exact .5 ties and every grid exponent that
keeps a term below 2^62; this test builds and runs it with the host compiler."""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "ternary_bitlinear_quantized_b200", "csrc")


def test_integer_fixed_point_terms_equal_the_fp64_route(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    exe = str(tmp_path / "fixed_point_check")
    subprocess.run([cxx, "-std=c++17", "-O2", "-Wall", "-I", CSRC, os.path.join(HERE, "fixed_point_check.cpp"),
                    "-o", exe], check=True, capture_output=True, text=True)
    res = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stdout + res.stderr
    assert res.stdout.startswith("OK"), res.stdout
