"""Pins of the oracle when Q has a different token count (Nq) than K and V
(Nkv): readings R11 (the causal mask aligns the last query with the last
key, so row r sees keys 0 .. r + Nkv - Nq) and R12 (a row that sees no key
outputs 0).

Independent references: closed forms for a single key (every visible row
returns that key's value: exactly in fp64, and as bf16(1.03125 * v^) under
the method's P recipe, tests/golden/causal_row0.txt); the identity "causal
row r == non-causal attention over the first r + Nkv - Nq + 1 keys",
checked on the same quantized buffers; brute-force fp64 attention on the
dequantized operands; and the untiled formula when there is one KV block.
"""
import numpy as np
import pytest
import torch

import oracle
import sa3_inputs
from test_oracle_attention import _bf16_to_f64, _golden_kv, _p_quant_ref, cosine, dequant, rel_l2


def _qkv(Nq, Nkv, d=64, H=2, seed=0):
    """Seeded tiny-workload draws, Q cut to Nq tokens and K, V to Nkv."""
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64", seed=seed,
                                  shape_override={"N": max(Nq, Nkv), "d": d, "H": H})
    return q[:, :, :Nq].contiguous(), k[:, :, :Nkv].contiguous(), v[:, :, :Nkv].contiguous()


def test_quantize_lengths_follow_q_and_kv():
    q, k, v = _qkv(70, 300)
    qz = oracle.quantize_qkv(q, k, v)
    assert qz["q_codes"].shape[2] == 128 and qz["k_codes"].shape[2] == 384
    assert qz["vt_codes"].shape[-1] == 384 // 2 and (qz["n_q"], qz["n_kv"]) == (70, 300)
    # Q alone is unchanged by the length of K and V; K's mean runs over Nkv
    qz_self = oracle.quantize_qkv(q, q, q)
    assert np.array_equal(qz["q_codes"], qz_self["q_codes"]) and np.array_equal(qz["q_sf"], qz_self["q_sf"])
    assert np.array_equal(qz["k_mean"], oracle.kmean(k))
    # padding tokens of K and V carry code 0 and scale 0
    assert not qz["k_codes"][:, :, 300:].any() and not qz["k_sf"][:, :, 300:].any()


@pytest.mark.parametrize("causal", [False, True])
def test_exact_single_key_returns_its_value(causal):
    Nq = 5
    q, k, v = _qkv(Nq, 1)
    out = oracle.attn_exact(q, k, v, causal)
    v0 = oracle.bf16_bits_to_f32(oracle._as_u16(v))[:, :, 0, :].astype(np.float64)
    for r in range(Nq):
        if causal and r < Nq - 1:   # sees no key (R12)
            assert not out[:, :, r].any()
        else:
            assert np.array_equal(out[:, :, r], v0)


@pytest.mark.parametrize("causal", [False, True])
def test_fp4_single_key_closed_form(causal):
    """One key: P = [1, 0, ...] in its block, so every row that sees it
    returns bf16(1.03125 * v^[0]); with the causal mask and Nq = 200 only
    the last row sees it and the others return 0."""
    Nq = 200
    q, k, v = _qkv(Nq, 1)
    qz = oracle.quantize_qkv(q, k, v)
    out = oracle.bf16_bits_to_f32(oracle.attn_fwd(qz, Nq, causal))
    _, _, vh = dequant(qz)
    g = _golden_kv("causal_row0.txt")
    want = torch.from_numpy((g["p_hat"] / g["row_sum"]) * vh[:, :, 0, :]).to(torch.float32)
    want = want.to(torch.bfloat16).float().numpy()
    for r in range(Nq):
        if causal and r < Nq - 1:
            assert not out[:, :, r].any(), r
        else:
            assert np.array_equal(out[:, :, r], want), r


def _prefix(qz, nkv):
    """The quantized K and V buffers of the first nkv keys (a slice of the
    token dimension, padded length included), Q unchanged."""
    npk = oracle.padded_len(nkv)
    return dict(q_codes=qz["q_codes"], q_sf=qz["q_sf"],
                k_codes=np.ascontiguousarray(qz["k_codes"][:, :, :npk]),
                k_sf=np.ascontiguousarray(qz["k_sf"][:, :, :npk]),
                vt_codes=np.ascontiguousarray(qz["vt_codes"][..., :npk // 2]),
                vt_sf=np.ascontiguousarray(qz["vt_sf"][..., :npk // 16]), n_kv=nkv)


@pytest.mark.parametrize("Nq,Nkv", [(150, 400), (300, 300), (260, 130)])
def test_causal_row_is_noncausal_over_its_prefix(Nq, Nkv):
    q, k, v = _qkv(Nq, Nkv)
    qz = oracle.quantize_qkv(q, k, v)
    full = oracle.attn_fwd(qz, Nq, True)
    off = Nkv - Nq
    rows = [r for r in (0, 1, 63, 127, 128, 129, 149, 200, 255, 259, 299) if r < Nq]
    for r in rows:
        n = r + off + 1
        if n <= 0:
            assert not full[:, :, r].any(), r
            continue
        n = min(n, Nkv)
        part = oracle.attn_fwd(_prefix(qz, n), Nq, False, units=[(bh, r // 128) for bh in range(2)])
        assert np.array_equal(full[:, :, r], part[:, :, r]), r


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nkv", [(200, 333), (333, 200)])
def test_agrees_with_bruteforce_on_dequantized_operands(Nq, Nkv, causal):
    d = 64
    q, k, v = _qkv(Nq, Nkv, d=d)
    qz = oracle.quantize_qkv(q, k, v)
    out = _bf16_to_f64(oracle.attn_fwd(qz, Nq, causal))
    qh, kh, vh = dequant(qz)
    s = qh[:, :, :Nq] @ np.swapaxes(kh[:, :, :Nkv], -1, -2) / np.sqrt(d)
    seen = np.ones((Nq, Nkv), bool)
    if causal:
        seen = np.arange(Nkv)[None, :] <= np.arange(Nq)[:, None] + (Nkv - Nq)
    s = np.where(seen, s, -np.inf)
    live = seen.any(-1)
    s = s - np.where(live[:, None], s.max(-1, keepdims=True), 0)
    p = np.exp(s)
    ref = (p @ vh[:, :, :Nkv]) / np.where(live[:, None], p.sum(-1, keepdims=True), 1)
    assert not out[:, :, ~live].any()
    assert cosine(out[:, :, live], ref[:, :, live]) >= 0.99
    assert rel_l2(out[:, :, live], ref[:, :, live]) <= 0.1


def test_exact_causal_row_is_noncausal_over_its_prefix():
    Nq, Nkv = 40, 90
    q, k, v = _qkv(Nq, Nkv)
    full = oracle.attn_exact(q, k, v, True)
    for r in (0, 17, 39):
        n = r + Nkv - Nq + 1
        part = oracle.attn_exact(q, k[:, :, :n].contiguous(), v[:, :, :n].contiguous(), False)
        assert np.array_equal(full[:, :, r], part[:, :, r]), r


def test_decode_rows_match_untiled_formula():
    """A few query rows against one KV block (Nkv <= 128): the tiled oracle
    must equal softmax with P microscaled once against the row maximum."""
    Nq, Nkv, d = 3, 100, 64
    q, k, v = _qkv(Nq, Nkv, d=d)
    qz = oracle.quantize_qkv(q, k, v)
    out = _bf16_to_f64(oracle.attn_fwd(qz, Nq, False))
    qh, kh, vh = dequant(qz)
    c = np.float32(np.float64(np.float32(1 / np.sqrt(d))) * 1.4426950408889634)
    t = ((qh[:, :, :Nq] @ np.swapaxes(kh[:, :, :Nkv], -1, -2)).astype(np.float32) * c).astype(np.float32)
    p = np.exp2((t - t.max(-1, keepdims=True)).astype(np.float32)).astype(np.float32)
    l = p.astype(np.float64).sum(-1, keepdims=True)
    pp = np.concatenate([p, np.zeros(p.shape[:-1] + (128 - Nkv,), np.float32)], -1)
    ref = (_p_quant_ref(pp)[..., :Nkv] @ vh[:, :, :Nkv]) / l
    assert rel_l2(out, ref) <= 2e-3
