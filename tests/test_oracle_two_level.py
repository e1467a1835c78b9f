"""Pins of the oracle's optional two-level P (reading R14): P is scaled by
2^11 before it is microscaled and O / l by 2^-11 after; and of its optional
V smoothing (reading R13): V - mean(V) is quantized and the mean added back
after O / l.

Independent references: the scale invariance of power-of-two factors (with
every block scale in the E4M3 normal range, the option changes nothing),
and a hand-derived closed form for a row whose second 16-column block of P
holds 16 keys at exactly 2^-9: the direct recipe rounds that block's scale
to 0 (2^-9 / 6 is below half the smallest E4M3 subnormal), two-level keeps
it with scale 0.6875 and code 6, which adds w / 32 to the output.
"""
import numpy as np
import pytest
import torch

import oracle
import sa3_inputs
from test_oracle_attention import _e2m1_table, _e4m3, _unpack, dequant


def test_no_change_when_every_block_scale_is_normal():
    """sm_scale 1e-3 keeps every logit within 0.02 of the row maximum, so
    every 16-block of P has amax > 0.9 and a normal E4M3 scale."""
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"N": 300})
    qz = oracle.quantize_qkv(q, k, v)
    for causal in (False, True):
        a = oracle.attn_fwd(qz, 300, causal, sm_scale=1e-3)
        b = oracle.attn_fwd(qz, 300, causal, sm_scale=1e-3, p_two_level=True)
        assert np.array_equal(a, b)


def _far_block_operands(d=64, N=128, seed=3):
    """Every query row: q^ = 6 on channel 0 (scale 1).  Keys: token 0 has
    k^ = 3 on channel 0 (logit 18), tokens 16..31 have 1.5 (logit 9), every
    other token -6 * 32 (logit -1152).  V^ random, except that tokens
    16..31 share one value w per channel (code 4 = 2.0 times the block
    scale).  With sm_scale = 1/log2(e) the logits in base 2 are exact."""
    rng = np.random.default_rng(seed)
    Np = oracle.padded_len(N)
    z = lambda *s: np.zeros(s, np.uint8)
    qz = dict(q_codes=z(1, 1, Np, d // 2), q_sf=z(1, 1, Np, d // 16), k_codes=z(1, 1, Np, d // 2),
              k_sf=z(1, 1, Np, d // 16),
              vt_codes=rng.integers(0, 256, (1, 1, d, Np // 2)).astype(np.uint8),
              vt_sf=rng.integers(40, 60, (1, 1, d, Np // 16)).astype(np.uint8))
    qz["q_codes"][0, 0, :N, 0] = 7      # 6.0
    qz["q_sf"][0, 0, :N, 0] = 56        # 1.0
    qz["k_codes"][0, 0, :N, 0] = 15     # -6.0
    qz["k_sf"][0, 0, :N, 0] = 96        # 32.0
    qz["k_codes"][0, 0, 0, 0] = 5       # 3.0
    qz["k_sf"][0, 0, 0, 0] = 56
    qz["k_codes"][0, 0, 16:32, 0] = 3   # 1.5
    qz["k_sf"][0, 0, 16:32, 0] = 56
    qz["vt_codes"][0, 0, :, 8:16] = 0x44  # tokens 16..31: code 4 (2.0) in both nibbles
    return qz


def test_two_level_closed_form():
    d, N = 64, 128
    qz = _far_block_operands(d, N)
    sm = float(np.float32(1 / np.log2(np.e)))
    direct = oracle.bf16_bits_to_f32(oracle.attn_fwd(qz, N, False, sm_scale=sm))
    two = oracle.bf16_bits_to_f32(oracle.attn_fwd(qz, N, False, sm_scale=sm, p_two_level=True))
    vt = _e2m1_table()[_unpack(qz["vt_codes"])] * np.repeat(_e4m3(qz["vt_sf"]), 16, axis=-1)
    v_hot = vt[0, 0, :, 0]
    w = 2.0 * _e4m3(qz["vt_sf"])[0, 0, :, 1]
    assert np.array_equal(vt[0, 0, :, 16], w)
    bf = lambda x: torch.from_numpy(np.asarray(x, np.float64)).to(torch.float32).to(torch.bfloat16).float().numpy()
    # direct: the far block is lost (scale 0); p^_hot = 1.03125 = l
    assert np.array_equal(direct[0, 0], np.broadcast_to(bf(v_hot), (N, d)))
    # two-level: P' = 4 there, scale E4M3(4/6) = 0.6875, code 6, p^' = 4.125;
    # (2112 v + 66 w) / 1.03125 * 2^-11 = v + w / 32
    assert np.array_equal(two[0, 0], np.broadcast_to(bf(v_hot + w / 32), (N, d)))


# ---- V smoothing (reading R13): V - mean(V) quantized, the mean added after O / l

def test_v_mean_matches_numpy_fp64_mean():
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"N": 300})
    r = oracle.quantize_qkv(q, k, v, smooth_v=True)
    want = v.double().mean(dim=2).float().numpy()
    assert np.array_equal(r["v_mean"].view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_is_returned_exactly_with_v_smoothing(causal):
    """V constant over tokens: V - mean is exactly 0, so every V code is 0,
    O = 0, and out = bf16(0 + mean) = V's row bit for bit, whatever P is.
    Without smoothing the same inputs give v times a row factor near 1."""
    q, k, _ = sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"N": 300})
    B, H, N, d = q.shape
    row = torch.randn((B, H, 1, d), generator=torch.Generator().manual_seed(11)).to(torch.bfloat16)
    v = row.expand(B, H, N, d).contiguous()
    r = oracle.quantize_qkv(q, k, v, smooth_v=True)
    assert not r["vt_codes"].any() and not r["vt_sf"].any()
    out = oracle.attn_fwd(r, N, causal)
    want = np.broadcast_to(row.view(torch.int16).numpy().view(np.uint16), out.shape)
    assert np.array_equal(out, want)
    plain = oracle.attn_fwd(oracle.quantize_qkv(q, k, v), N, causal)
    assert not np.array_equal(plain, want)


def test_v_smoothing_helps_when_v_has_a_channel_offset():
    """A per-channel offset of 8 on V (standard normal otherwise): each
    16-token block's scale is set by the offset, so the variation around it
    is coarsely quantized; subtracting the mean first restores it.  Cosine
    of the centred outputs to exact attention: 0.64 without, 0.97 with
    (Q/K quantization alone keeps this config near 0.98).  A missing or
    wrong-signed add-back of the mean is caught exactly by the constant-V
    closed form above."""
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"N": 300})
    v = (v.float() + 8.0).to(torch.bfloat16)
    ex = oracle.attn_exact(q, k, v, False).ravel()
    cos = lambda a, b: a @ b / np.sqrt((a @ a) * (b @ b))
    centred = lambda x: x - x.mean()
    res = {}
    for sv in (False, True):
        out = oracle.bf16_bits_to_f32(oracle.attn_fwd(oracle.quantize_qkv(q, k, v, smooth_v=sv), 300, False))
        res[sv] = cos(centred(out.astype(np.float64).ravel()), centred(ex))
    assert res[True] >= res[False] + 0.2 and res[True] >= 0.95, res
