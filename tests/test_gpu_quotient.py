"""The division-free quotient of the append kernels against IEEE division.

The 8-bit and KIVI quantizers compute RN(x / s) with one multiply by RN(1/s) and one fma
correction. The check program compiles the library's own device helper and compares it with
the correctly rounded division over significand pairs: every bf16 significand against every
fp32 significand of the scale, a slice of all fp32 pairs here, and all 2^46 pairs in the slow
test (about a minute on one B200).
"""
import os
import subprocess

import pytest

from decode_attention_quantize_b200 import build as B

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    exe = str(tmp_path_factory.mktemp("quot") / "gpu_quotient_check")
    subprocess.check_call([B.nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                           "-prec-div=true", "-ftz=false", "-fmad=true", "-I", B.INCLUDE, "-I", B.CSRC,
                           "-o", exe, os.path.join(HERE, "gpu_quotient_check.cu")])
    return exe


def _run(exe, *args, timeout=600):
    out = subprocess.run([exe, *args], capture_output=True, text=True, timeout=timeout)
    assert out.returncode == 0, out.stdout + out.stderr
    assert " mismatches 0" in out.stdout, out.stdout
    return out.stdout


def test_every_bf16_significand_against_every_scale(checker):
    _run(checker, "bf16")


def test_all_fp32_significands_one_slice(checker):
    _run(checker, "slice", "64", "37")


@pytest.mark.slow
def test_all_fp32_significand_pairs(checker):
    _run(checker, "slice", "1", "0", timeout=1800)
