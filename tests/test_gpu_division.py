"""The exact-division helpers of the CUDA kernels equal IEEE division.

The kernels decide q_scale = fp16(RN(m / 7)) and the stored codes
rint(RN(ws / q_scale)) with cheaper FMA sequences (common.cuh: div7_rn,
div_rn_rcp, div15_rn, quot_rcp1_2), and the duo weight mean divides fp16
magnitudes by their row maximum in fp64 with one Markstein correction
(ddiv_rn_rcp, on operands scaled by 2^-896).  This test compiles a small
check library from tests/cuda/division_check.cu and compares them bit for
bit with __fdiv_rn / __ddiv_rn: div7_rn and div15_rn over every non-negative
finite fp32 value, div_rn_rcp and the one-correction code decision over
every positive finite fp16 divisor with numerators at and around every
half-integer multiple of it (the rounding decisions) plus a sweep, and
ddiv_rn_rcp over every pair of non-negative finite fp16 values.
"""
import ctypes
import os
import subprocess
import tempfile

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_division_helpers_equal_ieee_division():
    src = os.path.join(ROOT, "tests", "cuda", "division_check.cu")
    inc = os.path.join(ROOT, "post_int4_weight_b200", "csrc")
    with tempfile.TemporaryDirectory() as d:
        so = os.path.join(d, "division_check.so")
        subprocess.run(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-I" + inc,
                        src, "-o", so], check=True)
        lib = ctypes.CDLL(so)
        out = (ctypes.c_ulonglong * 10)()
        assert lib.run_checks(out) == 0
    assert out[0] == 0, f"div7_rn differs from IEEE for {out[0]} values, first bits {out[1]:#x}"
    assert out[2] == 0, f"div_rn_rcp differs for {out[2]} pairs, first fp16 divisor {out[3]:#x}"
    assert out[4] == 0, (f"ddiv_rn_rcp (plain or scaled by 2^-896) differs for {out[4]} fp16 "
                         f"pairs, first fp16 divisor {out[5]:#x}")
    assert out[6] == 0, f"div15_rn differs from IEEE for {out[6]} values, first bits {out[7]:#x}"
    assert out[8] == 0, (f"one-correction code decision differs for {out[8]} pairs, "
                         f"first fp16 divisor {out[9]:#x}")
