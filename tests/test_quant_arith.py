"""Host checks of the GPU quantizer's divide-free arithmetic against the IEEE definition.

The quantizer (rotate_quantize.cu) computes scale = (max - min) / 15 by a divide-by-constant
correction step and each code from one fused multiply-add on a 2^-16 grid with an exact
remainder test at half-way grid values; both are claimed bit-identical to the IEEE divide of the
definition ("SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM Serving",
Research Findings: token-wise asymmetric INT4).  tests/arith/quant_arith_check.c restates the two
shortcuts in C and compares them with the IEEE operations: the scale step for every
non-negative finite fp32 dividend, the codes on a few million tie-heavy vectors.  The GPU parity
tests then compare the kernel itself with the oracle.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "arith", "quant_arith_check.c")


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path_factory.mktemp("arith") / "quant_arith_check")
    subprocess.run([cc, "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                    "-o", exe, SRC, "-lm"], check=True)
    return exe


def test_scale_division_by_15_exhaustive(checker):
    r = subprocess.run([checker, "div15"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert " 0 mismatches" in r.stdout


def test_grid_codes_match_ieee_divide(checker):
    r = subprocess.run([checker, "codes", "300000"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert " 0 mismatches" in r.stdout
    # the half-way branch must actually be exercised
    flagged = int(r.stdout.split(",")[1].split()[0])
    assert flagged > 1_000_000
