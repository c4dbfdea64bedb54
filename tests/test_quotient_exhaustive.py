"""The row quantizers and the Q8_0 -> int8 re-quantization compute fl(x / s)
without a division (a refined quotient, see quantize.cuh and q8_0.cuh).
These run the exhaustive proofs of that step on the GPU: every fp32 scale
significand against every bf16 significand over all binades the codes
depend on (about 2.5e10 pairs), and every value a Q8_0 block can hold
against every scale such values give, for the int8 and the e4m3 scales
(about 4.7e10 and 8.6e10 pairs); a few seconds each."""
import os
import subprocess
import tempfile

import pytest

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def _run_check(source, *args):
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from w8a8_quantized_linear_b200 import _build
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "check")
        subprocess.run([_build.nvcc(), *_build.ARCH, "-O3", "-o", exe, os.path.join(HERE, source)],
                       check=True, capture_output=True, text=True)
        res = subprocess.run([exe, *args], capture_output=True, text=True, timeout=600)
    line = res.stdout.strip()
    assert res.returncode == 0, line + res.stderr
    return line


def test_refined_quotient_is_ieee_division_for_every_bf16_input():
    line = _run_check("quotient_check.cu")
    assert "quotient mismatches 0, int8 code mismatches 0, e4m3 code mismatches 0" in line, line
    assert int(line.split()[1]) == (1 << 23) * 23 * 128


def test_refined_quotient_is_ieee_division_for_every_q8_0_value():
    line = _run_check("requant_quotient_check.cu", "127")
    assert "quotient mismatches 0, int8 code mismatches 0, e4m3 code mismatches 0" in line, line
    assert int(line.split()[1]) == 65537 * 65536 * 11


def test_refined_quotient_is_ieee_division_for_every_q8_0_value_e4m3_scale():
    """The e4m3 re-quantization: scales fl(a / 448), quotients down to the
    e4m3 rounding threshold 2^-10 and up to 448."""
    line = _run_check("requant_quotient_check.cu", "448")
    assert "quotient mismatches 0, int8 code mismatches 0, e4m3 code mismatches 0" in line, line
    assert int(line.split()[1]) == 65537 * 65536 * 20
