"""Build libsa3.so in-tree with nvcc for sm_100a.

    python -m bit_quantized_attention_sa3_b200.build [--force]
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libsa3.so")
SOURCES = [os.path.join(HERE, "csrc", "sa3.cu")]
DEPS = sorted(glob.glob(os.path.join(HERE, "csrc", "*")) + [os.path.join(ROOT, "include", "sa3.h")])
GENCODE = "arch=compute_100a,code=sm_100a"


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str = LIB) -> list[str]:
    return [nvcc_path(), "-gencode", GENCODE, "-lineinfo", "-O3", "-std=c++17",
            "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-warn-spills",
            "-I", os.path.join(ROOT, "include"), "-o", out] + SOURCES


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = command(tmp)
    if verbose:
        print(" ".join(cmd))
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed ({r.returncode}):\n{r.stdout}\n{r.stderr}")
    if "spill" in r.stderr:
        print(r.stderr, file=sys.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
