"""The quantizer's division-free amax / 6 (div6 in quant.cuh), checked on
the host for every non-negative fp32 input by tests/div6_check.c: the E4M3
scale code it leads to equals the one of the IEEE quotient."""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _body(text: str) -> str:
    m = re.search(r"float div6\(float x\) \{(.*?)\n\}", text, re.S)
    assert m, "div6 not found"
    return re.sub(r"\s+", " ", m.group(1)).strip()


def test_the_check_restates_the_kernel_formula():
    with open(os.path.join(ROOT, "bit_quantized_attention_sa3_b200", "csrc", "quant.cuh")) as f:
        kernel = _body(f.read())
    with open(os.path.join(ROOT, "tests", "div6_check.c")) as f:
        check = _body(f.read())
    assert kernel == check


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_div6_gives_the_scale_code_of_the_ieee_quotient(tmp_path):
    exe = str(tmp_path / "div6_check")
    flags = ["-O3", "-ffp-contract=off", "-fno-fast-math"]
    src = os.path.join(ROOT, "tests", "div6_check.c")
    b = subprocess.run(["gcc", *flags, "-mfma", src, "-o", exe, "-lm"], capture_output=True, text=True)
    if b.returncode != 0:  # no FMA instructions on this host: libm's fmaf
        b = subprocess.run(["gcc", *flags, src, "-o", exe, "-lm"], capture_output=True, text=True)
    assert b.returncode == 0, b.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok ")
