"""Pins of the oracle's K smoothing and tiled FP4 attention.

Independent references used here: the exact-arithmetic invariance of
softmax attention under K mean subtraction ("SageAttention" summary,
"Approach"); a closed form for causal row 0 (tests/golden/causal_row0.txt);
one-hot rows whose answer is fixed by the recurrence; and brute-force fp64
attention on the dequantized operands, decoded here with torch's E4M3 view
and the golden E2M1 table rather than with the oracle's own decoder.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import sa3_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
E2M1 = None


def _e2m1_table():
    global E2M1
    if E2M1 is None:
        vals = {}
        for line in open(os.path.join(GOLDEN, "e2m1_values.txt")):
            line = line.strip()
            if line and not line.startswith("#"):
                c, v = line.split()
                vals[int(c)] = float(v)
        E2M1 = np.array([vals[c] for c in range(16)], np.float64)
    return E2M1


def _golden_kv(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            out[k] = float(v)
    return out


def _e4m3(sf: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(sf)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _unpack(codes: np.ndarray) -> np.ndarray:
    return np.stack([codes & 15, codes >> 4], -1).reshape(*codes.shape[:-1], codes.shape[-1] * 2)


def dequant(qz):
    """Q^, K^ [B,H,Np,d] and V^ [B,H,Np,d] (untransposed) in fp64."""
    t = _e2m1_table()
    qh = t[_unpack(qz["q_codes"])] * np.repeat(_e4m3(qz["q_sf"]), 16, axis=-1)
    kh = t[_unpack(qz["k_codes"])] * np.repeat(_e4m3(qz["k_sf"]), 16, axis=-1)
    vth = t[_unpack(qz["vt_codes"])] * np.repeat(_e4m3(qz["vt_sf"]), 16, axis=-1)
    return qh, kh, np.swapaxes(vth, -1, -2)


def _bf16_to_f64(a):
    return oracle.bf16_bits_to_f32(a).astype(np.float64)


def cosine(a, b):
    a = a.ravel().astype(np.float64)
    b = b.ravel().astype(np.float64)
    return float(a @ b / np.sqrt((a @ a) * (b @ b)))


def rel_l2(a, b):
    a = a.astype(np.float64)
    b = b.astype(np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.fixture(scope="module")
def tiny():
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64")
    return q, k, v, oracle.quantize_qkv(q, k, v)


def test_smoothing_leaves_exact_attention_unchanged(tiny):
    q, k, v, qz = tiny
    for causal in (False, True):
        a = oracle.attn_exact(q, k, v, causal)
        b = oracle.attn_exact(q, k, v, causal, k_sub=qz["k_mean"])
        assert np.abs(a - b).max() <= 1e-12 * np.abs(a).max()


def test_smoothing_improves_fp4_accuracy(tiny):
    """The pages' ablation: smoothing K raises cosine similarity of
    quantized attention against full precision."""
    q, k, v, qz = tiny
    ex = oracle.attn_exact(q, k, v, False)
    with_s = _bf16_to_f64(oracle.attn_fwd(qz, 256, False))
    without = _bf16_to_f64(oracle.attn_fwd(oracle.quantize_qkv(q, k, v, smooth_k=False), 256, False))
    assert cosine(with_s, ex) > cosine(without, ex) + 0.01


def test_causal_row0_closed_form(tiny):
    q, k, v, qz = tiny
    g = _golden_kv("causal_row0.txt")
    out = oracle.attn_fwd(qz, 256, True)
    _, _, vh = dequant(qz)
    want = torch.from_numpy((g["p_hat"] / g["row_sum"]) * vh[:, :, 0, :]).to(torch.float32)
    want = want.to(torch.bfloat16).float().numpy()
    # compared by value: the sum that forms O starts at +0, so a -0 input
    # product may come out as +0
    assert np.array_equal(oracle.bf16_bits_to_f32(out[:, :, 0, :]), want)


def _onehot_operands(B, H, N, d, hot):
    """Quantized operands where row r of Q attends overwhelmingly to token
    hot[bh]: q^ = 6 on channel 0 (scale 1), k^[hot] = 6*64 on channel 0,
    every other key 0 there; V^ random."""
    rng = np.random.default_rng(5)
    Np = oracle.padded_len(N)
    qz = dict(
        q_codes=np.zeros((B, H, Np, d // 2), np.uint8), q_sf=np.zeros((B, H, Np, d // 16), np.uint8),
        k_codes=np.zeros((B, H, Np, d // 2), np.uint8), k_sf=np.zeros((B, H, Np, d // 16), np.uint8),
        vt_codes=rng.integers(0, 256, (B, H, d, Np // 2)).astype(np.uint8),
        vt_sf=rng.integers(40, 60, (B, H, d, Np // 16)).astype(np.uint8))
    qz["q_codes"][:, :, :N, 0] = 7
    qz["q_sf"][:, :, :N, 0] = 56  # 1.0
    for bh, t in enumerate(hot):
        b, h = divmod(bh, H)
        qz["k_codes"][b, h, t, 0] = 7
        qz["k_sf"][b, h, t, 0] = 120  # 256.0
    Npad = qz["vt_codes"].shape[-1] * 2
    # padded tokens carry code 0
    vt = _unpack(qz["vt_codes"])
    vt[..., N:] = 0
    qz["vt_codes"] = (vt[..., 0::2] | (vt[..., 1::2] << 4)).astype(np.uint8)
    assert Npad == Np
    return qz


def test_onehot_rows_follow_the_recurrence():
    """Logit gap 6*6*256/sqrt(d)*log2(e) >> 150: every other p underflows
    to 0, so each row returns bf16(1.03125 * v^[hot]) whichever KV block
    holds the hot key (earlier blocks must be wiped by alpha = 0)."""
    B, H, N, d = 1, 3, 300, 64
    hot = [5, 200, 299]
    qz = _onehot_operands(B, H, N, d, hot)
    out = oracle.attn_fwd(qz, N, False)
    _, _, vh = dequant(qz)
    g = _golden_kv("causal_row0.txt")
    for bh, t in enumerate(hot):
        want = torch.from_numpy(g["p_hat"] * vh[0, bh, t, :]).to(torch.float32).to(torch.bfloat16)
        want = want.float().numpy()
        assert np.array_equal(oracle.bf16_bits_to_f32(out[0, bh]), np.broadcast_to(want, (N, d))), bh


def _brute(qh, kh, vh, N, causal, sm_scale):
    """fp64 softmax attention on dequantized operands (P not quantized)."""
    qh, kh, vh = qh[:, :, :N], kh[:, :, :N], vh[:, :, :N]
    s = qh @ np.swapaxes(kh, -1, -2) * sm_scale
    if causal:
        s = s + np.triu(np.full((N, N), -np.inf), 1)
    s = s - s.max(-1, keepdims=True)
    p = np.exp(s)
    return (p @ vh) / p.sum(-1, keepdims=True)


@pytest.mark.parametrize("causal", [False, True])
def test_oracle_agrees_with_bruteforce_on_dequantized_operands(tiny, causal):
    q, k, v, qz = tiny
    N, d = 256, 64
    out = _bf16_to_f64(oracle.attn_fwd(qz, N, causal))
    qh, kh, vh = dequant(qz)
    ref = _brute(qh, kh, vh, N, causal, 1 / np.sqrt(d))
    assert cosine(out, ref) >= 0.99
    assert rel_l2(out, ref) <= 0.1


def _p_quant_ref(p: np.ndarray) -> np.ndarray:
    """Per-16 microscaling of P, written with torch's E4M3 conversion for
    the scale and numpy's half-even rounding per E2M1 binade."""
    pb = p.astype(np.float32).reshape(*p.shape[:-1], -1, 16)
    amax = pb.max(-1)
    sc = torch.from_numpy((amax / np.float32(6)).astype(np.float32)).to(torch.float8_e4m3fn)
    s = sc.to(torch.float32).numpy()
    r = np.where(s > 0, np.float32(1) / np.where(s > 0, s, 1), 0).astype(np.float32)
    y = (pb * r[..., None]).astype(np.float32)
    mag = np.where(y < 2, np.round(y * 2) / 2, np.where(y < 4, np.round(y), np.round(y / 2) * 2))
    mag = np.minimum(mag, 6.0)
    return (mag * s[..., None]).reshape(p.shape)


def test_single_kv_block_matches_untiled_formula():
    """With N <= 128 there is one KV block: the oracle must equal
    softmax with the running max = row max and P microscaled once."""
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"N": 100})
    qz = oracle.quantize_qkv(q, k, v)
    N, d = 100, 64
    out = _bf16_to_f64(oracle.attn_fwd(qz, N, False))
    qh, kh, vh = dequant(qz)
    c = np.float32(np.float64(np.float32(1 / np.sqrt(d))) * 1.4426950408889634)
    s = (qh[:, :, :N] @ np.swapaxes(kh[:, :, :N], -1, -2)).astype(np.float32)
    t = (s * c).astype(np.float32)
    m = t.max(-1, keepdims=True)
    p = np.exp2((t - m).astype(np.float32)).astype(np.float32)
    l = p.astype(np.float64).sum(-1, keepdims=True)
    pp = np.concatenate([p, np.zeros(p.shape[:-1] + (128 - N,), np.float32)], -1)
    ph = _p_quant_ref(pp)[..., :N]
    ref = (ph @ vh[:, :, :N]) / l
    assert rel_l2(out, ref) <= 2e-3
    exact_frac = np.mean(torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16).float().numpy() == out)
    assert exact_frac >= 0.95


def test_max_in_first_block_matches_untiled_formula():
    """For rows whose maximum logit sits in KV block 0, alpha stays 1 after
    that block, so the tiled result must equal the untiled formula with P
    microscaled per block against the row maximum."""
    B, H, N, d = 1, 2, 384, 64
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"N": N})
    qz = oracle.quantize_qkv(q, k, v)
    out = _bf16_to_f64(oracle.attn_fwd(qz, N, False))
    qh, kh, vh = dequant(qz)
    c = np.float32(np.float64(np.float32(1 / np.sqrt(d))) * 1.4426950408889634)
    s = (qh[:, :, :N] @ np.swapaxes(kh[:, :, :N], -1, -2)).astype(np.float32)
    t = (s * c).astype(np.float32)
    m = t.max(-1, keepdims=True)
    p = np.exp2((t - m).astype(np.float32)).astype(np.float32)
    l = p.astype(np.float64).sum(-1, keepdims=True)
    ref = (_p_quant_ref(p) @ vh[:, :, :N]) / l
    rows = t.argmax(-1) < 128
    assert rows.sum() >= 100
    assert rel_l2(out[rows], ref[rows]) <= 2e-3
    # rows whose maximum comes later see a different running max in block 0
    assert rel_l2(out[~rows], ref[~rows]) > 1e-3


def _constant_v(q, seed=5):
    """V constant over tokens, v_c = +-6 * 2^k_c per (b, h, channel): every
    16-token block of V^T quantizes exactly (scale 2^k_c, code 6)."""
    B, H, N, d = q.shape
    g = np.random.default_rng(seed)
    vc = g.choice([-1.0, 1.0], (B, H, 1, d)) * 6.0 * 2.0 ** g.integers(-3, 3, (B, H, 1, d))
    return torch.from_numpy(np.broadcast_to(vc, (B, H, N, d)).copy()).to(torch.bfloat16), vc


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_rows_are_v_times_one_factor(causal):
    """With V^ = V constant over tokens, O_c = v_c * sum(P^) / sum(P): one
    factor per row, and since the channels differ only by a sign and a power
    of two, every rounding scales with them, so out / v is bit-identical
    across channels.  Causal row 0 sees one key: P = 1, P^ = 6 * E4M3(1/6) =
    1.03125.  The factor stays near 1 (P's FP4 rounding, averaged over the
    row: between 0.92 and 1.09 on these inputs; bound 0.75 .. 1.25)."""
    q, k, _ = sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"N": 300})
    v, vc = _constant_v(q)
    out = oracle.bf16_bits_to_f32(oracle.attn_fwd(oracle.quantize_qkv(q, k, v), 300, causal)).astype(np.float64)
    ratio = out / vc
    assert np.array_equal(ratio, np.broadcast_to(ratio[..., :1], ratio.shape))
    assert (ratio > 0.75).all() and (ratio < 1.25).all()
    if causal:
        assert (ratio[:, :, 0] == 1.03125).all()


@pytest.mark.parametrize("Nq,Nkv,causal,sm", [(300, 300, False, None), (300, 300, True, None), (77, 300, True, 0.3),
                                              (300, 77, False, None), (129, 1, True, None)])
def test_exact_attention_matches_torch_sdpa(Nq, Nkv, causal, sm):
    """The fp64 reference against PyTorch's scaled_dot_product_attention in
    float64 on the same bf16 inputs.  The causal mask is passed explicitly,
    bottom-right aligned (query r sees keys 0 .. r + Nkv - Nq); rows that see
    no key are left out (the oracle gives them 0, the library routine NaN)."""
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"N": max(Nq, Nkv)})
    q, k, v = q[:, :, :Nq].contiguous(), k[:, :, :Nkv].contiguous(), v[:, :, :Nkv].contiguous()
    d = q.shape[-1]
    got = oracle.attn_exact(q, k, v, causal, sm_scale=sm)
    vis = torch.ones((Nq, Nkv), dtype=torch.bool)
    if causal:
        vis = torch.arange(Nkv)[None, :] <= torch.arange(Nq)[:, None] + (Nkv - Nq)
    scale = float(np.float32((1.0 / np.sqrt(d)) if sm is None else sm))  # the oracle takes sm_scale as fp32
    want = torch.nn.functional.scaled_dot_product_attention(
        q.double(), k.double(), v.double(), attn_mask=vis, scale=scale).numpy()
    live = vis.any(dim=1).numpy()
    np.testing.assert_allclose(got[:, :, live], want[:, :, live], rtol=1e-12, atol=1e-12)
    assert not got[:, :, ~live].any()


@pytest.mark.parametrize("causal", [False, True])
def test_sampled_units_equal_the_full_computation(causal):
    """The full-size GPU tests compare only sampled (head, Q block) units
    against the oracle, so the unit path must give exactly the rows of the
    full computation and leave every other row untouched: FP4, 8-bit (with
    the log-sum-exp) and exact attention."""
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"N": 300, "H": 3})
    B, H, N, d = q.shape
    units = [(0, 2), (2, 0), (1, 1)]
    rows = np.zeros((B * H, N), bool)
    for bh, qb in units:
        rows[bh, qb * 128: min(N, qb * 128 + 128)] = True
    rows = rows.reshape(B, H, N)

    qz = oracle.quantize_qkv(q, k, v)
    full, part = oracle.attn_fwd(qz, N, causal), oracle.attn_fwd(qz, N, causal, units=units)
    assert np.array_equal(part[rows], full[rows]) and not part[~rows].any()

    q8 = oracle.quantize_qkv_i8(q, k, v)
    f8, fl = oracle.attn_fwd_i8(q8, N, causal, return_lse=True)
    p8, pl = oracle.attn_fwd_i8(q8, N, causal, units=units, return_lse=True)
    assert np.array_equal(p8[rows], f8[rows]) and not p8[~rows].any()
    assert np.array_equal(pl[rows], fl[rows]) and np.isnan(pl[~rows]).all()

    ex, pe = oracle.attn_exact(q, k, v, causal), oracle.attn_exact(q, k, v, causal, units=units)
    assert np.array_equal(pe[rows], ex[rows]) and not pe[~rows].any()
