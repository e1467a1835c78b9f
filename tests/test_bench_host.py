"""Host-side logic of bench.py that needs no GPU: the operation count for
unequal query / key lengths (4*d per (query, key) pair the mask leaves,
checked against a brute-force count of the mask), the input shapes, and
the tiles behind the exp2 ceiling (against a brute-force tile count)."""
import dataclasses
import importlib.util
import os

import numpy as np
import pytest

import sa3_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _pairs(Nq, Nkv, causal):
    r = np.arange(Nq)[:, None]
    c = np.arange(Nkv)[None, :]
    vis = np.ones((Nq, Nkv), bool) if not causal else (c <= r + (Nkv - Nq))
    return int(vis.sum())


@pytest.mark.parametrize("Nq,Nkv,causal", [(300, 300, True), (77, 1000, True), (1000, 130, True),
                                           (1, 300, True), (77, 1000, False), (300, 17, False)])
def test_attn_ops_counts_the_pairs_the_mask_leaves(bench, Nq, Nkv, causal):
    w = dataclasses.replace(sa3_inputs.WORKLOADS["tiny_b1h2n256d64"], N=Nkv, causal=causal)
    ops = bench.attn_ops(w, Nq)
    if Nq == Nkv:
        assert ops == w.ops  # the workload's own convention: 4*B*H*N^2*d, halved when causal
    else:
        assert ops == 4.0 * w.B * w.H * w.d * _pairs(Nq, Nkv, causal)


@pytest.mark.parametrize("Nq", [100, 256, 300])
def test_make_inputs_shapes_and_prefix(bench, Nq):
    w = sa3_inputs.WORKLOADS["tiny_b1h2n256d64"]
    q, k, v = bench.make_inputs(w, Nq, seed=0)
    assert q.shape[2] == Nq and k.shape[2] == w.N and v.shape[2] == w.N
    if Nq <= w.N:
        q0, k0, v0 = sa3_inputs.make_qkv(w, seed=0)
        assert (q == q0[:, :, :Nq]).all() and (k == k0).all() and (v == v0).all()


REQUIRED = {"metric": str, "value": (int, float), "unit": str, "n_gpus": int, "steps": int, "warmup": int,
            "ms_per_step": (int, float), "higher_is_better": bool, "scaling": str, "dtype": str, "data": str,
            "config": dict, "e2e": dict}


def _check_line(line):
    for k, t in REQUIRED.items():
        assert k in line and isinstance(line[k], t), k
    assert "vs_baseline" in line and line["vs_baseline"] is None
    assert line["config"]["workload"] and line["value"] > 0
    for k in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"):
        assert k in line["e2e"], k


def test_reference_arm_prints_the_contract_line():
    import json
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny_b1h2n256d64", "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    _check_line(line)
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["cores"] >= 1 and line["cpu_baseline"]["sample"]


@pytest.mark.gpu
def test_gpu_arm_prints_the_contract_line():
    """The benchmark's own arm on the headline workload, briefly: every key of
    the line, the roofline object, clocks and the launch count."""
    import json
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "3", "--warmup", "3",
                        "--skip-cpu-baseline"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    _check_line(line)
    roof = line["roofline"]
    assert roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s" and 0 < roof["frac"] < 1.5
    assert abs(roof["achieved"] / roof["peak"] - roof["frac"]) < 1e-3
    assert line["gpu_launches"] == 3 * line["steps"]
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(line["clocks"])
    assert line["e2e"]["h2d_bytes_per_step"] == 3 * 2 * 16 * 4096 * 128 * 2


def _tiles_brute(Nq, N, causal):
    """Q tile t computes KV block b when some row of t sees some key of b."""
    n = 0
    for t in range((Nq + 127) // 128):
        for b in range((N + 127) // 128):
            if not causal:
                n += 1
                continue
            last_row = t * 128 + 127            # rows past Nq still belong to the tile
            if b * 128 <= last_row + (N - Nq):  # the block's first key is visible to the last row
                n += 1
    return n


@pytest.mark.parametrize("Nq,N,causal", [(4096, 4096, False), (256, 256, True), (300, 300, True), (77, 1000, True),
                                         (1000, 130, True), (1, 300, True), (17776, 17776, False),
                                         (8192, 8192, True), (130, 1000, False)])
def test_processed_s_elements_counts_the_kernels_tiles(bench, Nq, N, causal):
    assert bench.processed_s_elements(2, 3, Nq, N, causal) == 2 * 3 * _tiles_brute(Nq, N, causal) * 128 * 128


def test_exp2_ceiling_of_the_headline_shape(bench):
    # 2*16*4096^2 S elements x (1 + 1/16 + 1/64) exp2 / (16 per SM-clock x 148 SMs x 1.965 GHz)
    us = bench.exp2_ceiling_us(2, 16, 4096, 4096, False, 1965.0, 148)
    assert abs(us - 2 * 16 * 4096 * 4096 * 1.078125 / (16 * 148 * 1965e6) * 1e6) < 1e-6
    assert 124.0 < us < 125.0
