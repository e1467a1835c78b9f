"""Degenerate and extreme inputs on the GPU against the oracle.

Quantization (bit-exact, as for the seeded workloads):
  * all-zero Q, K, V: every scale 0, every code 0, K mean +0;
  * -0.0 inside non-zero blocks (sign-preserving code 0x8) and whole -0.0
    blocks (scale 0, codes 0);
  * constant K per (b, h): smoothing leaves exact zeros, so K codes and
    scales are all 0;
  * 16-element blocks whose magnitudes spread from far below the smallest
    E4M3 scale (scale rounds to 0) through subnormal scales to saturation
    at 448 (codes clip at +-6).
Attention (rel-L2 <= 2e-3 against the oracle on the same operands, finite):
  * zero Q and K, and constant K: every logit is 0, so each visible key gets
    the same P;
  * the spread inputs with Q and K kept at moderate magnitudes (the kernel
    folds log2(1/s) into the exp2 argument, rounded at the size of the row
    maximum, so logits in the tens of thousands are outside its accuracy
    bar by design)."""
import numpy as np
import pytest
import torch

import oracle
from sa3_testutil import (bits_to_f32, blockwise_rel_l2, fp64_sum_is_exact, qk_sf_to_canonical, vt_sf_to_canonical)

sa3 = pytest.importorskip("bit_quantized_attention_sa3_b200")

E4M3_MAX = 0x7E  # 448


def _spread(B, H, N, d, lo, hi, along, seed):
    """Normal values times 2^e, e drawn per 16-element block: along "d" for
    Q and K (blocks of channels), "tok" for V (blocks of 16 tokens)."""
    g = torch.Generator().manual_seed(seed)
    z = torch.randn((B, H, N, d), generator=g, dtype=torch.float32)
    if along == "d":
        e = torch.randint(lo, hi + 1, (B, H, N, d // 16, 1), generator=g).expand(B, H, N, d // 16, 16)
        e = e.reshape(B, H, N, d)
    else:
        nb = (N + 15) // 16
        e = torch.randint(lo, hi + 1, (B, H, nb, 1, d), generator=g).expand(B, H, nb, 16, d)
        e = e.reshape(B, H, nb * 16, d)[:, :, :N]
    return (z * torch.pow(2.0, e.float())).to(torch.bfloat16)


def _quantized(q, k, v):
    B, H, N, d = q.shape
    Np = sa3.padded_len(N)
    qz = sa3.quantize_qkv(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    g = dict(q_codes=qz.q_fp4.cpu().numpy(), k_codes=qz.k_fp4.cpu().numpy(), vt_codes=qz.vt_fp4.cpu().numpy(),
             q_sf=qk_sf_to_canonical(qz.q_sf.cpu().numpy(), B, H, Np, d),
             k_sf=qk_sf_to_canonical(qz.k_sf.cpu().numpy(), B, H, Np, d),
             vt_sf=vt_sf_to_canonical(qz.vt_sf.cpu().numpy(), B, H, Np, d),
             k_mean=qz.k_mean.cpu().numpy())
    return qz, g


def _assert_same(g, r):
    for f in ("q_codes", "q_sf", "k_codes", "k_sf", "vt_codes", "vt_sf"):
        if not np.array_equal(g[f], r[f]):
            bad = np.argwhere(g[f] != r[f])
            pytest.fail(f"{f}: {len(bad)} mismatches, first {bad[:3].tolist()}")
    assert np.array_equal(g["k_mean"].view(np.uint32), r["k_mean"].view(np.uint32))


def _cases():
    B, H, N = 1, 2, 300
    out = []
    for d in (64, 128):
        zero = torch.zeros((B, H, N, d), dtype=torch.bfloat16)
        out.append((f"zeros-d{d}", zero, zero, zero))
        g = torch.Generator().manual_seed(d)
        q = torch.randn((B, H, N, d), generator=g).to(torch.bfloat16)
        k = torch.randn((B, H, N, d), generator=g).to(torch.bfloat16)
        v = torch.randn((B, H, N, d), generator=g).to(torch.bfloat16)
        for t in (q, k, v):  # scattered -0.0, and whole 16-blocks of -0.0
            t[..., ::7, ::5] = -0.0
        q[..., 3, :16] = -0.0
        v[..., 32:48, 5] = -0.0
        out.append((f"negzero-d{d}", q, k, v))
        row = torch.randn((B, H, 1, d), generator=g).to(torch.bfloat16)
        out.append((f"constk-d{d}", q, row.expand(B, H, N, d).contiguous(), v))
        out.append((f"spread-d{d}", _spread(B, H, N, d, -40, 14, "d", 10 + d),
                    _spread(B, H, N, d, -8, 15, "d", 20 + d), _spread(B, H, N, d, -40, 14, "tok", 30 + d)))
    return out


CASES = _cases()


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_quantize_special_values_bit_exact(case):
    name, q, k, v = case
    assert fp64_sum_is_exact(k)
    _, g = _quantized(q, k, v)
    r = oracle.quantize_qkv(q, k, v)
    _assert_same(g, r)
    if name.startswith("zeros"):
        assert not any(g[f].any() for f in ("q_codes", "q_sf", "k_codes", "k_sf", "vt_codes", "vt_sf"))
        assert not g["k_mean"].view(np.uint32).any()  # +0, not -0
    if name.startswith("constk"):
        assert not g["k_codes"].any() and not g["k_sf"].any()
    if name.startswith("negzero"):
        assert (g["q_codes"] & 0x0F == 0x08).any() or (g["q_codes"] >> 4 == 0x08).any()
    if name.startswith("spread"):
        for f in ("q_sf", "vt_sf"):
            s = g[f]
            assert (s == 0).any() and ((s > 0) & (s < 8)).any() and (s == E4M3_MAX).any(), f


ATTN = [c for c in CASES if c[0].split("-")[0] in ("zeros", "constk", "negzero")]
ATTN += [(f"spread-moderate-d{d}", _spread(1, 2, 300, d, -40, 1, "d", 40 + d), _spread(1, 2, 300, d, -8, 1, "d", 50 + d),
          _spread(1, 2, 300, d, -40, 14, "tok", 60 + d)) for d in (64, 128)]


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True], ids=["noncausal", "causal"])
@pytest.mark.parametrize("case", ATTN, ids=[c[0] for c in ATTN])
def test_attn_special_values_match_oracle(case, causal):
    name, q, k, v = case
    qz, g = _quantized(q, k, v)
    B, H, N, d = q.shape
    out = sa3.attn_fwd(qz, causal=causal)
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    r = oracle.quantize_qkv(q, k, v)  # the oracle attends on its own operands
    _assert_same(g, r)
    o32 = np.zeros((B, H, N, d), np.float32)
    ref = bits_to_f32(oracle.attn_fwd(r, N, causal, out32=o32))
    if name.startswith("zeros"):
        assert not got.any() and not ref.any()
    else:
        blocks = [(h, qb) for h in range(B * H) for qb in range((N + 127) // 128)]
        blockwise_rel_l2(got.reshape(B * H, N, d), ref.reshape(B * H, N, d), blocks, 2e-3, label=name,
                         ref32=o32.reshape(B * H, N, d))


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_quantize_i8_special_values_bit_exact(case):
    """The 8-bit quantizer on the same inputs: zero tiles give scale 0 and
    codes 0; V values beyond the FP16 range become inf on both sides."""
    from test_i8_gpu import _canon
    name, q, k, v = case
    qz = sa3.quantize_qkv_i8(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    g = _canon(qz)
    r = oracle.quantize_qkv_i8(q, k, v)
    for f in ("q_i8", "k_i8", "vt_f16"):
        assert np.array_equal(g[f], r[f]), f
    for f in ("q_scale", "k_scale", "k_mean"):
        assert np.array_equal(g[f].view(np.uint32), r[f].view(np.uint32)), f
    if name.startswith("zeros"):
        assert not g["q_scale"].any() and not g["q_i8"].any() and not g["k_i8"].any()


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True], ids=["noncausal", "causal"])
@pytest.mark.parametrize("d", [64, 128])
def test_attn_constant_v_rows_are_v_times_one_factor(d, causal):
    """V constant over tokens with v_c = +-6 * 2^k_c (exact in FP4): each
    output row is v times one factor, bit-identical across channels (the
    tensor core sums every channel in the same order, and the channels
    differ by a sign and a power of two), and equal to the oracle's."""
    g = torch.Generator().manual_seed(d)
    B, H, N = 1, 2, 300
    q = torch.randn((B, H, N, d), generator=g).to(torch.bfloat16)
    k = torch.randn((B, H, N, d), generator=g).to(torch.bfloat16)
    rng = np.random.default_rng(d)
    vc = rng.choice([-1.0, 1.0], (B, H, 1, d)) * 6.0 * 2.0 ** rng.integers(-3, 3, (B, H, 1, d))
    v = torch.from_numpy(np.broadcast_to(vc, (B, H, N, d)).copy()).to(torch.bfloat16)
    qz, gq = _quantized(q, k, v)
    out = sa3.attn_fwd(qz, causal=causal)
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    ratio = out.double().cpu().numpy() / vc
    assert np.array_equal(ratio, np.broadcast_to(ratio[..., :1], ratio.shape))
    if causal:
        assert (ratio[:, :, 0] == 1.03125).all()
    r = oracle.quantize_qkv(q, k, v)
    _assert_same(gq, r)
    ref = bits_to_f32(oracle.attn_fwd(r, N, causal))
    blocks = [(h, qb) for h in range(B * H) for qb in range((N + 127) // 128)]
    blockwise_rel_l2(out.float().cpu().numpy().reshape(B * H, N, d), ref.reshape(B * H, N, d), blocks, 2e-3,
                     label=f"constant V d={d}")
