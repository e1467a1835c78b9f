"""The oracle's C under the host address and undefined-behaviour sanitizers.

oracle/sanitize_main.c calls every oracle entry point on small seeded
shapes (ragged tails, single-token and decode-sized queries, more queries
than keys, both masks, d 64 / 128, the optional terms); built with
-fsanitize=address,undefined and no recovery, any out-of-range access,
use after free, leak, signed overflow or other undefined behaviour ends
the run with a report and a non-zero status.  OpenMP is left out so the
sanitizers see one thread."""
import os
import shutil
import subprocess

import pytest

ORACLE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_oracle_runs_clean_under_asan_and_ubsan(tmp_path):
    exe = str(tmp_path / "oracle_sanitize")
    cmd = ["gcc", "-O1", "-g", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-Wall", "-Wno-unknown-pragmas",
           "-fsanitize=address,undefined", "-fno-sanitize-recover=all", "-fno-omit-frame-pointer",
           os.path.join(ORACLE, "sa3_oracle.c"), os.path.join(ORACLE, "sanitize_main.c"), "-o", exe, "-lm"]
    b = subprocess.run(cmd, capture_output=True, text=True)
    if b.returncode != 0 and "asan" in b.stderr.lower():
        pytest.skip("the host toolchain has no sanitizer runtime: " + b.stderr.strip().splitlines()[-1])
    assert b.returncode == 0, b.stderr
    env = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:abort_on_error=0", UBSAN_OPTIONS="print_stacktrace=1")
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "runtime error" not in r.stderr and "ERROR: AddressSanitizer" not in r.stderr, r.stderr
    assert r.stdout.strip() == "ok"
