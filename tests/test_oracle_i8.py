"""Pins of the oracle's 8-bit variant ("SageAttention" summary, "Approach":
INT8 Q and K with per-block scales after K smoothing, P and V in FP16;
readings I1-I5 in oracle/sa3_oracle.c).

Independent references: numpy's float16 conversion (round to nearest even)
and numpy's half-even rint; lossless blocks built as code x power-of-two
scale; the causal row-0 closed form (one visible key, P = 1 exactly, so the
output is that key's value); brute-force fp64 attention on the dequantized
operands; the untiled formula when there is one KV block.
"""
import numpy as np
import pytest
import torch

import oracle
import sa3_inputs


def test_f16_conversion_matches_numpy():
    rng = np.random.default_rng(0)
    xs = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-9, 6, 20000),
                         np.float32([0.0, -0.0, 65504.0, 65519.0, 65520.0, 1e30, -1e30, 2.0 ** -24, 2.0 ** -25,
                                     3 * 2.0 ** -26, 2.0 ** -14, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11])])
    xs = xs.astype(np.float32)
    got = np.array([oracle.f32_to_f16(float(x)) for x in xs], np.uint16)
    with np.errstate(over="ignore"):  # overflow to inf is part of the rule
        want = xs.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)


def _blocks(q):
    """Quantize q as the Q operand (no smoothing) with K, V dummies."""
    z = torch.zeros_like(q)
    return oracle.quantize_qkv_i8(q, z, z)


def test_int8_block_is_lossless_for_code_times_power_of_two():
    rng = np.random.default_rng(1)
    codes = rng.integers(-127, 128, (1, 1, 128, 64)).astype(np.float32)
    codes[0, 0, 5, 7] = 127.0
    s = 2.0 ** -7
    q = torch.from_numpy(codes * s).to(torch.bfloat16)  # |x| <= 127/128: exact in bf16 (8 bits)
    r = _blocks(q)
    assert r["q_scale"][0, 0, 0] == np.float32(s)
    assert np.array_equal(r["q_i8"][0, 0].astype(np.float32), codes[0, 0])


def test_int8_rounding_is_half_even_and_clamped():
    # amax 127 * 2^-4 -> s = 2^-4 exactly, r = 16: x * r lands on the ties below
    vals = np.zeros((1, 1, 128, 64), np.float32)
    vals[0, 0, 0, 0] = 127 * 2.0 ** -4
    ties = np.array([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5], np.float32) * 2.0 ** -4
    vals[0, 0, 1, :7] = ties
    r = _blocks(torch.from_numpy(vals).to(torch.bfloat16))
    assert r["q_scale"][0, 0, 0] == np.float32(2.0 ** -4)
    assert list(r["q_i8"][0, 0, 1, :7]) == list(np.rint(ties * 16).astype(np.int8)) == [0, 2, 2, 0, -2, -2, 126]


def test_causal_row0_returns_its_value():
    """Row 0 sees key 0 only: P = [1] (exactly 1 in FP16), l = 1, so the
    output is V's row 0 (bf16 -> fp16 exact in range -> bf16)."""
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64")
    out = oracle.attn_fwd_i8(oracle.quantize_qkv_i8(q, k, v), 256, True)
    v0 = v[:, :, 0, :].contiguous().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(out[:, :, 0, :], v0)


def _dequant(qz):
    qh = qz["q_i8"].astype(np.float64) * np.repeat(qz["q_scale"].astype(np.float64), 128, axis=-1)[..., None]
    kh = qz["k_i8"].astype(np.float64) * np.repeat(qz["k_scale"].astype(np.float64), 128, axis=-1)[..., None]
    vh = np.swapaxes(qz["vt_f16"].view(np.float16).astype(np.float64), -1, -2)
    return qh, kh, vh


@pytest.mark.parametrize("causal", [False, True])
def test_agrees_with_bruteforce_on_dequantized_operands(causal):
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"N": 300})
    N, d = 300, 64
    qz = oracle.quantize_qkv_i8(q, k, v)
    out = oracle.bf16_bits_to_f32(oracle.attn_fwd_i8(qz, N, causal)).astype(np.float64)
    qh, kh, vh = _dequant(qz)
    s = qh[:, :, :N] @ np.swapaxes(kh[:, :, :N], -1, -2) / np.sqrt(d)
    if causal:
        s = s + np.triu(np.full((N, N), -np.inf), 1)
    p = np.exp(s - s.max(-1, keepdims=True))
    ref = (p @ vh[:, :, :N]) / p.sum(-1, keepdims=True)
    err = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert err <= 2e-3, err


def test_single_kv_block_matches_untiled_formula():
    Nq, N, d = 70, 100, 64
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"N": N})
    q = q[:, :, :Nq].contiguous()
    qz = oracle.quantize_qkv_i8(q, k, v)
    out = oracle.bf16_bits_to_f32(oracle.attn_fwd_i8(qz, Nq, False)).astype(np.float64)
    si = qz["q_i8"][:, :, :Nq].astype(np.int64) @ np.swapaxes(qz["k_i8"][:, :, :N].astype(np.int64), -1, -2)
    c = np.float32(np.float64(np.float32(1 / np.sqrt(d))) * 1.4426950408889634)
    f = (qz["q_scale"][:, :, :1, None] * qz["k_scale"][:, :, None, :1]).astype(np.float32) * c
    t = (si.astype(np.float32) * f.astype(np.float32)).astype(np.float32)
    p = np.exp2((t - t.max(-1, keepdims=True)).astype(np.float32)).astype(np.float32)
    l = p.astype(np.float64).sum(-1, keepdims=True)
    p16 = p.astype(np.float16).astype(np.float64)
    vh = np.swapaxes(qz["vt_f16"].view(np.float16).astype(np.float64), -1, -2)[:, :, :N]
    ref = (p16 @ vh) / l
    assert np.linalg.norm(out - ref) / np.linalg.norm(ref) <= 2e-3
    exact_frac = np.mean(torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16).float().numpy() == out)
    assert exact_frac >= 0.95


def test_int8_variant_is_more_accurate_than_fp4():
    """The pages' claim for 8-bit attention: cosine to full precision well
    above the FP4 path's on the same inputs."""
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64")
    ex = oracle.attn_exact(q, k, v, False).ravel()
    i8 = oracle.bf16_bits_to_f32(oracle.attn_fwd_i8(oracle.quantize_qkv_i8(q, k, v), 256, False)).astype(np.float64).ravel()
    fp4 = oracle.bf16_bits_to_f32(oracle.attn_fwd(oracle.quantize_qkv(q, k, v), 256, False)).astype(np.float64).ravel()
    cos = lambda a, b: a @ b / np.sqrt((a @ a) * (b @ b))
    assert cos(i8, ex) >= 0.999 and cos(i8, ex) > cos(fp4, ex)


# ---- log-sum-exp of the training forward (reading I6)

@pytest.mark.parametrize("Nq,Nkv,causal", [(300, 300, False), (300, 300, True), (70, 300, True),
                                           (300, 70, True), (70, 300, False)])
def test_lse_with_zero_scale_is_log_of_visible_count(Nq, Nkv, causal):
    """sm_scale = 0 makes every visible logit 0, so P = 1 on each visible
    key and lse = ln(number of keys the row sees); a row that sees none
    gets +inf."""
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"N": max(Nq, Nkv)})
    q, k, v = q[:, :, :Nq].contiguous(), k[:, :, :Nkv].contiguous(), v[:, :, :Nkv].contiguous()
    _, lse = oracle.attn_fwd_i8(oracle.quantize_qkv_i8(q, k, v), Nq, causal, sm_scale=0.0, return_lse=True)
    rows = np.arange(Nq)
    count = np.minimum(rows + 1 + (Nkv - Nq), Nkv) if causal else np.full(Nq, Nkv)
    want = np.where(count > 0, np.log(np.maximum(count, 1)), np.inf).astype(np.float32)
    assert np.array_equal(np.isinf(lse[0, 0]), count <= 0)
    np.testing.assert_allclose(lse[..., count > 0], np.broadcast_to(want[count > 0], lse[..., count > 0].shape),
                               rtol=2e-7, atol=0)


@pytest.mark.parametrize("Nq,Nkv,causal", [(300, 300, False), (300, 300, True), (70, 300, True), (300, 70, True)])
def test_lse_agrees_with_bruteforce_logsumexp(Nq, Nkv, causal):
    """fp64 logsumexp of sm_scale * (Q^ K^T) on the dequantized INT8
    operands.  The oracle's t is fp32 (a few roundings of a product whose
    magnitude stays below 64 here) and l an fp32 sum, so 1e-5 absolute."""
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"N": max(Nq, Nkv)})
    q, k, v = q[:, :, :Nq].contiguous(), k[:, :, :Nkv].contiguous(), v[:, :, :Nkv].contiguous()
    d = q.shape[-1]
    qz = oracle.quantize_qkv_i8(q, k, v)
    _, lse = oracle.attn_fwd_i8(qz, Nq, causal, return_lse=True)
    qh, kh, _ = _dequant(qz)
    s = qh[:, :, :Nq] @ np.swapaxes(kh[:, :, :Nkv], -1, -2) / np.sqrt(d)
    assert np.abs(s).max() < 64
    if causal:
        vis = np.arange(Nkv)[None, :] <= np.arange(Nq)[:, None] + (Nkv - Nq)
        s = np.where(vis, s, -np.inf)
    with np.errstate(divide="ignore"):
        mx = s.max(-1, keepdims=True)
        ref = (mx + np.log(np.exp(s - np.where(np.isfinite(mx), mx, 0)).sum(-1, keepdims=True)))[..., 0]
    live = np.isfinite(ref)
    assert np.array_equal(np.isinf(lse), ~live) and (lse[~live] > 0).all()
    assert np.abs(lse[live] - ref[live]).max() <= 1e-5


def test_lse_reconstructs_the_output():
    """What a backward pass does with lse: P = exp(s - lse) has rows that sum
    to 1 and P V^ gives the forward's output (to the FP16 rounding of P)."""
    N, d = 260, 64
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"N": N})
    qz = oracle.quantize_qkv_i8(q, k, v)
    out, lse = oracle.attn_fwd_i8(qz, N, True, return_lse=True)
    qh, kh, vh = _dequant(qz)
    s = qh[:, :, :N] @ np.swapaxes(kh[:, :, :N], -1, -2) / np.sqrt(d) + np.triu(np.full((N, N), -np.inf), 1)
    pr = np.exp(s - lse[..., None].astype(np.float64))
    np.testing.assert_allclose(pr.sum(-1), 1.0, rtol=0, atol=2e-5)
    o = oracle.bf16_bits_to_f32(out).astype(np.float64)
    ref = pr @ vh[:, :, :N]
    assert np.linalg.norm(o - ref) / np.linalg.norm(ref) <= 2e-3


def test_lse_is_optional_and_leaves_the_output_unchanged():
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64")
    qz = oracle.quantize_qkv_i8(q, k, v)
    a = oracle.attn_fwd_i8(qz, 256, True)
    b, _ = oracle.attn_fwd_i8(qz, 256, True, return_lse=True)
    assert np.array_equal(a, b)
