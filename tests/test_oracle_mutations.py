"""The oracle's pins are strong enough to catch plausible mistakes: each
case below plants one single-line mistake in a copy of oracle/sa3_oracle.c
(on the CPU, in a temporary directory), builds it with the oracle's own
compiler command, and runs the pin suite against it (SA3_ORACLE_LIB); at
least one pin must fail.  The in-tree source and library are never touched."""
import concurrent.futures
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "sa3_oracle.c")
PINS = ["tests/test_oracle_attention.py", "tests/test_oracle_codecs.py", "tests/test_oracle_cross.py",
        "tests/test_oracle_i8.py", "tests/test_oracle_two_level.py", "tests/test_oracle_heads.py"]

TIES = "if (dist < bestd || (dist == bestd && (c & 1) == 0)) {"
C_LOG2 = "const float c_log2 = (float)((double)sm_scale * 1.4426950408889634);"
# (what the mistake is, text, replacement, which occurrence)
MUTATIONS = [
    ("alpha with the wrong sign", "alpha = exp2f(m - m_new);", "alpha = exp2f(m_new - m);", 0),
    ("P against the previous maximum", "p[i] = exp2f(t[i] - m_new);",
     "p[i] = exp2f(t[i] - (m > -INFINITY ? m : m_new));", 0),
    ("row sum not rescaled", "l = alpha * l + rowsum;", "l = l + rowsum;", 0),
    ("O not rescaled", "O[c] = alpha * O[c] + (float)acc;", "O[c] = O[c] + (float)acc;", 0),
    ("block scale amax / 4", "float ratio = amax / 6.0f;", "float ratio = amax / 4.0f;", 0),
    ("E2M1 ties to the larger code", TIES, "if (dist < bestd || dist == bestd) {", 0),
    ("E4M3 ties to the larger code", TIES, "if (dist < bestd || dist == bestd) {", 1),
    ("K smoothing adds the mean", "x[i] = sub ? xv - sub[b * VEC + i] : xv;",
     "x[i] = sub ? xv + sub[b * VEC + i] : xv;", 0),
    ("V smoothing adds the mean", "vv - v_mean[bh * d + c]", "vv + v_mean[bh * d + c]", 0),
    ("causal mask off by one", "if (col >= Nkv || (causal && col > row + off))",
     "if (col >= Nkv || (causal && col >= row + off))", 0),
    ("log2(e) left out", C_LOG2, "const float c_log2 = (float)((double)sm_scale);", 0),
    ("K mean over the padded length", "mean[bh * d + c] = (float)(acc / (double)N);",
     "mean[bh * d + c] = (float)(acc / (double)((N + 127) / 128 * 128));", 0),
    ("V^T nibbles swapped", "(uint8_t)(codes[i] | (codes[i + 1] << 4));\n            }\n        }\n    }\n}",
     "(uint8_t)(codes[i + 1] | (codes[i] << 4));\n            }\n        }\n    }\n}", 0),
    ("two-level factor 2^10", "o * (1.0f / 2048.0f)", "o * (1.0f / 1024.0f)", 0),
    ("8-bit: alpha with the wrong sign", "alpha = exp2f(m - m_new);", "alpha = exp2f(m_new - m);", 1),
    ("8-bit: row sum not rescaled", "l = alpha * l + (float)psum;", "l = l + (float)psum;", 0),
    ("8-bit: log2(e) left out", C_LOG2, "const float c_log2 = (float)((double)sm_scale);", 1),
]


def _nth_replace(s, old, new, n):
    i = -1
    for _ in range(n + 1):
        i = s.index(old, i + 1)
    return s[:i] + new + s[i + len(old):]


def _run(case, tmp):
    name, old, new, n = case
    src = open(SRC).read()
    mutated = _nth_replace(src, old, new, n)
    assert mutated != src
    d = os.path.join(tmp, str(MUTATIONS.index(case)))
    os.makedirs(d)
    c_file, lib = os.path.join(d, "sa3_oracle.c"), os.path.join(d, "liboracle.so")
    open(c_file, "w").write(mutated)
    subprocess.run(oracle.gcc_command(c_file, lib), check=True, capture_output=True)
    env = dict(os.environ, SA3_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", *PINS],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, r.returncode


def test_every_planted_mistake_fails_a_pin(tmp_path):
    oracle.build()
    with concurrent.futures.ThreadPoolExecutor(max_workers=4) as ex:
        results = list(ex.map(lambda c: _run(c, str(tmp_path)), MUTATIONS))
    missed = [name for name, rc in results if rc == 0]
    assert not missed, f"pins passed with these mistakes planted: {missed}"


def test_the_unmutated_copy_passes(tmp_path):
    """The same route with the source unchanged passes every pin, so a
    failure above comes from the planted mistake, not from the route."""
    lib = str(tmp_path / "liboracle.so")
    subprocess.run(oracle.gcc_command(SRC, lib), check=True, capture_output=True)
    env = dict(os.environ, SA3_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", *PINS],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:]
