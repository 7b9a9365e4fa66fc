"""The refit's reciprocal and division (Newton-Raphson with Markstein's correction) are
correctly rounded: exhaustive over every significand at the exponents the refit meets,
and randomised over wide exponent ranges, against CUDA's __frcp_rn / __fdiv_rn."""
import ctypes
import os
import subprocess
import tempfile

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "quantized_linear_attention_02_b200", "csrc")


@pytest.fixture(scope="module")
def checker():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    out = os.path.join(tempfile.mkdtemp(), "fastdiv_check.so")
    subprocess.run(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                    "--fmad=false", "-shared", "-Xcompiler", "-fPIC", "-I", CSRC, "-o", out,
                    os.path.join(HERE, "cuda", "fastdiv_check.cu")], check=True)
    return ctypes.CDLL(out)


def test_reciprocal_exhaustive(checker):
    bad = ctypes.c_ulonglong(0)
    first = ctypes.c_uint32(0)
    # every significand, both signs, exponents -40..40 plus the range ends
    for lo, hi in ((-40, 40), (-126, -120), (120, 127)):
        assert checker.fastdiv_check_rcp(lo, hi, ctypes.byref(bad), ctypes.byref(first)) == 0
        assert bad.value == 0, f"reciprocal differs for 0x{first.value:08x}"


@pytest.mark.parametrize("span", [20, 60, 126])
def test_division_random(checker, span):
    bad = ctypes.c_ulonglong(0)
    n = ctypes.c_uint32(0)
    d = ctypes.c_uint32(0)
    assert checker.fastdiv_check_div(1234 + span, 64, span, ctypes.byref(bad), ctypes.byref(n), ctypes.byref(d)) == 0
    assert bad.value == 0, f"{bad.value} quotients differ, e.g. 0x{n.value:08x} / 0x{d.value:08x}"
