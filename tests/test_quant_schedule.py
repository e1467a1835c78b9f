"""The quantizer's static work schedule, checked on the host: the real
SchedA of quant.cuh is compiled (nvcc, host code only; no GPU needed) into
tests/quant_schedule_check.cu and run over 3840 shape / grid / mode
combinations, equal and unequal query lengths and V smoothing included."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="needs nvcc")
def test_every_tile_is_scheduled_exactly_once(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = str(tmp_path / "quant_schedule_check")
    b = subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O2",
                        "-I", os.path.join(ROOT, "bit_quantized_attention_sa3_b200", "csrc"),
                        "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "quant_schedule_check.cu"), "-o", exe],
                       capture_output=True, text=True, timeout=600)
    assert b.returncode == 0, b.stderr[-3000:]
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip() == "ok 3840 cases"
