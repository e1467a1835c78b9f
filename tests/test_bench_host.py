"""Host-side logic of bench.py that needs no GPU: the operation count for
unequal query / key lengths (4*d per (query, key) pair the mask leaves,
checked against a brute-force count of the mask) and the input shapes."""
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
