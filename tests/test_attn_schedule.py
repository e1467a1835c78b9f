"""The FP4 attention kernel's persistent work list, checked on the host:
the real Sched of attn.cuh is compiled (nvcc, host code only; no GPU
needed) into tests/attn_schedule_check.cu and run over shapes with equal
and unequal query lengths, both masks and several grid sizes."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="needs nvcc")
def test_every_q_tile_is_scheduled_exactly_once(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = str(tmp_path / "attn_schedule_check")
    b = subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O2",
                        "-I", os.path.join(ROOT, "bit_quantized_attention_sa3_b200", "csrc"),
                        "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "attn_schedule_check.cu"), "-o", exe],
                       capture_output=True, text=True, timeout=600)
    assert b.returncode == 0, b.stderr[-3000:]
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip().startswith("ok ") and int(r.stdout.split()[1]) > 2000
