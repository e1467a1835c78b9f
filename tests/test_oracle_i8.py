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
