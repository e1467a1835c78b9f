"""The 8-bit variant (sa3_quantize_qkv_i8 / sa3_attn_fwd_i8) on the GPU
against the oracle's 8-bit recipe.

Bars: INT8 codes, per-tile scales, FP16 V^T and the K mean bit-exact; the
attention output rel-L2 <= 2e-3 in every (head, Q block) against the
oracle attending on its own quantized operands, after those have been
checked equal to the GPU's (ex2.approx against exp2f and tensor-core
accumulation order), and its cosine to fp64 exact attention within 1e-3 of
the oracle's.  Rows that
see no key (causal, Nq > Nkv) are exactly 0."""
import numpy as np
import pytest
import torch

import oracle
import sa3_inputs
from sa3_testutil import bits_to_f32, blockwise_rel_l2, cosine, fp64_sum_is_exact

sa3 = pytest.importorskip("bit_quantized_attention_sa3_b200")

TOL = 2e-3

CASES = [
    ("tiny_b1h2n256d64", 256, 256, None),
    ("tiny_b1h2n256d64", 300, 300, {"H": 3}),
    ("tiny_b1h2n256d64", 1, 300, None),
    ("noncausal_b2h16n4096d128", 640, 640, {"B": 2, "H": 2}),
    ("noncausal_b2h16n4096d128", 77, 1000, {"B": 1, "H": 2}),
    ("noncausal_b2h16n4096d128", 1000, 130, {"B": 1, "H": 2}),
    ("videodit_b1h30n17776d64", 1000, 1000, {"H": 2}),
    ("prefill_b4h32n8192d128_causal", 2048, 2048, {"B": 1, "H": 4}),
]


def _ids(c):
    return f"{c[0]}-q{c[1]}-kv{c[2]}"


def _qkv(name, Nq, Nkv, over):
    o = dict(over or {})
    o["N"] = max(Nq, Nkv)
    q, k, v = sa3_inputs.make_qkv(name, shape_override=o)
    return q[:, :, :Nq].contiguous(), k[:, :, :Nkv].contiguous(), v[:, :, :Nkv].contiguous()


def assert_i8_equal(g, r):
    """The GPU's 8-bit operands (canonical) equal the oracle's bit for bit."""
    for f in ("q_i8", "k_i8", "vt_f16"):
        if not np.array_equal(g[f], r[f]):
            bad = np.argwhere(g[f] != r[f])
            pytest.fail(f"{f}: {len(bad)} mismatches, first {bad[:5].tolist()}")
    for f in ("q_scale", "k_scale", "k_mean"):
        assert np.array_equal(g[f].view(np.uint32), r[f].view(np.uint32)), f


def _canon(qz):
    return dict(q_i8=qz.q_i8.cpu().numpy(), q_scale=qz.q_scale.cpu().numpy(), k_i8=qz.k_i8.cpu().numpy(),
                k_scale=qz.k_scale.cpu().numpy(), vt_f16=qz.vt_f16.cpu().view(torch.int16).numpy().view(np.uint16),
                k_mean=qz.k_mean.cpu().numpy(), n_kv=qz.N)


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_quantize_i8_matches_oracle_bit_exact(case):
    name, Nq, Nkv, over = case
    q, k, v = _qkv(name, Nq, Nkv, over)
    assert fp64_sum_is_exact(k)
    qz = sa3.quantize_qkv_i8(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    assert_i8_equal(_canon(qz), oracle.quantize_qkv_i8(q, k, v))


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True], ids=["noncausal", "causal"])
@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_attn_i8_matches_oracle(case, causal):
    name, Nq, Nkv, over = case
    q, k, v = _qkv(name, Nq, Nkv, over)
    qz = sa3.quantize_qkv_i8(q.cuda(), k.cuda(), v.cuda())
    out = sa3.attn_fwd_i8(qz, causal=causal)
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    r_q = oracle.quantize_qkv_i8(q, k, v)
    assert_i8_equal(_canon(qz), r_q)
    ref = bits_to_f32(oracle.attn_fwd_i8(r_q, Nq, causal, n_kv=Nkv))
    ex = oracle.attn_exact(q, k, v, causal)
    live = (np.arange(Nq) + (Nkv - Nq) >= 0) if causal else np.ones(Nq, bool)
    if causal:
        assert not got[:, :, ~live].any() and not ref[:, :, ~live].any()
    B, H, _, d = q.shape
    blocks = [(h, qb) for h in range(B * H) for qb in range((Nq + 127) // 128)]
    blockwise_rel_l2(got.reshape(B * H, Nq, d), ref.reshape(B * H, Nq, d), blocks, TOL, live=live,
                     label=_ids(case))
    g, r, e = got[:, :, live], ref[:, :, live], ex[:, :, live]
    assert cosine(g, e) >= cosine(r, e) - 1e-3


@pytest.mark.gpu
def test_causal_row0_returns_its_value_i8():
    """Row 0 sees key 0 only, so P = 1 there and the output is V's row 0,
    whatever its logit: on the prefill workload (outlier channels) some
    heads' row-0 logit is far below zero, which a wrong running maximum
    turns into P = 0, l = 0 and NaN."""
    q, k, v = sa3_inputs.make_qkv("prefill_b4h32n8192d128_causal", shape_override={"B": 1, "H": 32, "N": 1024})
    qz = sa3.quantize_qkv_i8(q.cuda(), k.cuda(), v.cuda())
    out = sa3.attn_fwd_i8(qz, causal=True)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    assert torch.equal(out[:, :, 0].cpu(), v[:, :, 0])
