"""Pins of the oracle's E2M1 / E4M3 codecs and of its block quantizer.

Each check compares the oracle with something other than itself: printed
values of the formats (tests/golden), torch's float8_e4m3fn conversion (a
library routine with round-to-nearest-even), numpy's round-half-to-even per
binade, and inputs built so that quantization must be lossless.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_pairs(name):
    out = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        a, b = line.split()
        out.append((int(a), float(b)))
    return out


def test_e2m1_table_matches_format_definition():
    for code, val in _read_pairs("e2m1_values.txt"):
        got = oracle.e2m1_value(code)
        assert got == val and math.copysign(1, got) == math.copysign(1, val), code


def test_e4m3_points_match_format_definition():
    for code, val in _read_pairs("e4m3_points.txt"):
        got = oracle.e4m3_value(code)
        if math.isnan(val):
            assert math.isnan(got), code
        else:
            assert got == val and math.copysign(1, got) == math.copysign(1, val), code


def test_e4m3_decode_agrees_with_torch_for_all_codes():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = oracle.e4m3_value(c)
        if math.isnan(ref[c]):
            assert math.isnan(got)
        else:
            assert got == ref[c], c


def _e4m3_probe_points():
    vals = sorted({oracle.e4m3_value(c) for c in range(127)})
    pts = []
    for a, b in zip(vals[:-1], vals[1:]):
        mid = (a + b) / 2
        for x in (a, b, mid):
            f = np.float32(x)
            pts += [f, np.nextafter(f, np.float32(0)), np.nextafter(f, np.float32(1e9))]
    rng = np.random.default_rng(0)
    pts += list(rng.uniform(0, 479.0, 20000).astype(np.float32))
    pts += list((2.0 ** rng.uniform(-12, 8.9, 20000)).astype(np.float32))
    # torch maps values above 464 (midpoint of 448 and 480) to NaN; the
    # saturation region is checked separately below.
    return np.array([p for p in pts if 0 <= p <= 464], np.float32)


def test_e4m3_round_nearest_even_matches_torch():
    pts = _e4m3_probe_points()
    ref = torch.from_numpy(pts).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_rn_sat(float(x)) for x in pts], np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(pts[i]), int(got[i]), int(ref[i])) for i in bad[:10]]


def test_e4m3_saturates_at_448():
    # torch turns >= 480 into NaN; the satfinite reading clamps to 448.
    for x in (448.0, 463.9, 464.0, 479.0, 480.0, 1e6, 3.0e38):
        assert oracle.e4m3_rn_sat(x) == 0x7E


def _e2m1_ref(x: float) -> float:
    """Nearest E2M1 magnitude via numpy's round-half-to-even inside each
    binade (step 0.5 below 2, 1 in [2,4), 2 in [4,8)), saturating at 6."""
    a = abs(x)
    if a < 2:
        r = float(np.round(a * 2) / 2)
    elif a < 4:
        r = float(np.round(a))
    else:
        r = float(np.round(a / 2) * 2)
    return min(r, 6.0)


def test_e2m1_round_nearest_even_matches_binade_rounding():
    mags = [0, .5, 1, 1.5, 2, 3, 4, 6]
    pts = []
    for a, b in zip(mags[:-1], mags[1:]):
        for x in (a, b, (a + b) / 2):
            f = np.float32(x)
            pts += [f, np.nextafter(f, np.float32(0)), np.nextafter(f, np.float32(100))]
    pts += list(np.linspace(0, 8, 4097, dtype=np.float32))
    pts += [np.float32(7.0), np.float32(100.0), np.float32(1e30)]
    for x in pts:
        for sx in (float(x), -float(x)):
            code = oracle.e2m1_rn(sx)
            val = oracle.e2m1_value(code)
            assert abs(val) == _e2m1_ref(sx), (sx, code)
            if abs(val) != 0:
                assert (val < 0) == (sx < 0)


def test_e2m1_ties_table():
    # ties of the grid {0,.5,1,1.5,2,3,4,6} go to the even mantissa
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for x, want in ties.items():
        assert oracle.e2m1_value(oracle.e2m1_rn(x)) == want


def test_e2m1_keeps_sign_of_zero():
    assert oracle.e2m1_rn(-0.0) == 0x8
    assert oracle.e2m1_rn(-0.1) == 0x8
    assert oracle.e2m1_rn(0.1) == 0x0


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    xs = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-8, 8, 20000),
                         np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -9, -(1 + 2 ** -8)], np.float32)])
    ref = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f32_to_bf16(float(x)) for x in xs], np.uint16)
    assert np.array_equal(got, ref)


# --------------------------------------------------------------- quantizer

def _bf16(a: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)
    assert torch.equal(t.float(), torch.from_numpy(np.ascontiguousarray(a, np.float32))), "not bf16-exact"
    return t


def _unpack(codes: np.ndarray) -> np.ndarray:
    lo = codes & 15
    hi = codes >> 4
    return np.stack([lo, hi], -1).reshape(*codes.shape[:-1], codes.shape[-1] * 2)


def test_quantize_is_lossless_on_representable_blocks():
    """Blocks built as code * scale with one element at code 6 must come back
    exactly (codes, scale), for Q and K (blocks along d) and V (along tokens).
    K gets every token paired with its negation so its mean is exactly 0."""
    rng = np.random.default_rng(2)
    B, H, N, d = 1, 2, 256, 64
    e2 = np.array([oracle.e2m1_value(c) for c in range(16)])
    scales = [c for c in range(1, 127) if 2 ** -6 <= oracle.e4m3_value(c) <= 64]

    def build(blocks_along_last):
        codes = rng.integers(0, 16, size=blocks_along_last.shape + (16,))
        codes[..., rng.integers(0, 16)] = 7  # amax code 6
        sc = rng.choice(scales, size=blocks_along_last.shape)
        sval = np.vectorize(oracle.e4m3_value)(sc)
        return codes, sc, e2[codes] * sval[..., None]

    cq, sq, xq = build(np.zeros((B, H, N, d // 16)))
    q = xq.reshape(B, H, N, d)
    ck, sk, xk = build(np.zeros((B, H, N // 2, d // 16)))
    khalf = xk.reshape(B, H, N // 2, d)
    k = np.concatenate([khalf, -khalf], axis=2)
    cv, sv, xv = build(np.zeros((B, H, d, N // 16)))
    v = np.swapaxes(xv.reshape(B, H, d, N), 2, 3)
    r = oracle.quantize_qkv(_bf16(q), _bf16(k), _bf16(v))
    assert np.all(r["k_mean"] == 0)
    assert np.array_equal(r["q_sf"], sq.astype(np.uint8))
    assert np.array_equal(_unpack(r["q_codes"]), cq.reshape(B, H, N, d))
    assert np.array_equal(r["k_sf"][:, :, : N // 2], sk.astype(np.uint8))
    assert np.array_equal(_unpack(r["k_codes"])[:, :, : N // 2], ck.reshape(B, H, N // 2, d))
    assert np.array_equal(r["vt_sf"], sv.astype(np.uint8))
    assert np.array_equal(_unpack(r["vt_codes"]), cv.reshape(B, H, d, N))


def test_quantize_nibble_order_and_padding():
    """Element 2i sits in the low nibble; tokens past N are code 0 / scale 0."""
    B, H, N, d = 1, 1, 130, 64
    q = np.zeros((B, H, N, d), np.float32)
    q[0, 0, 0, 0] = 6.0   # code 7 with scale 1
    q[0, 0, 0, 1] = 1.0   # code 2
    v = np.zeros_like(q)
    v[0, 0, 0, 3] = 6.0
    v[0, 0, 1, 3] = -3.0
    r = oracle.quantize_qkv(_bf16(q), _bf16(np.zeros_like(q)), _bf16(v))
    assert r["q_codes"][0, 0, 0, 0] == (7 | (2 << 4))
    assert oracle.e4m3_value(int(r["q_sf"][0, 0, 0, 0])) == 1.0
    assert r["vt_codes"][0, 0, 3, 0] == (7 | (0xD << 4))
    assert r["q_codes"].shape[2] == 256
    assert not r["q_codes"][0, 0, N:].any() and not r["q_sf"][0, 0, N:].any()
    assert not r["vt_codes"][0, 0, :, N // 2 + 1:].any()


def test_quantize_zero_block_and_saturation():
    B, H, N, d = 1, 1, 128, 64
    q = np.zeros((B, H, N, d), np.float32)
    q[0, 0, 1, :16] = 2.0 ** 127  # huge finite bf16: the scale saturates at 448
    q[0, 0, 2, 0] = 2.0 ** -20  # amax/6 below half the smallest subnormal scale -> s == 0
    r = oracle.quantize_qkv(_bf16(q), _bf16(np.zeros_like(q)), _bf16(np.zeros_like(q)))
    assert r["q_sf"][0, 0, 0, 0] == 0 and not r["q_codes"][0, 0, 0].any()
    assert r["q_sf"][0, 0, 1, 0] == 0x7E
    assert np.all(_unpack(r["q_codes"][0, 0, 1])[:16] == 7)
    assert r["q_sf"][0, 0, 2, 0] == 0 and not r["q_codes"][0, 0, 2].any()


def test_kmean_matches_numpy_fp64_mean():
    import sa3_inputs
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64")
    got = oracle.kmean(k)
    ref = k.to(torch.float64).mean(dim=2).to(torch.float32).numpy()
    assert np.array_equal(got, ref)


def test_kmean_closed_form_offset():
    """K = offset +/- x in token pairs has mean exactly offset."""
    rng = np.random.default_rng(3)
    B, H, N, d = 2, 3, 64, 64
    off = np.round(rng.standard_normal((B, H, 1, d)) * 4) / 4
    x = np.round(rng.standard_normal((B, H, N // 2, d)) * 8) / 8
    k = np.concatenate([off + x, off - x], axis=2)
    got = oracle.kmean(_bf16(k))
    assert np.array_equal(got, off[:, :, 0, :].astype(np.float32))
