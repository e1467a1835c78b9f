"""sa3_attn_fwd on the GPU against the CPU oracle.

Bar: output rel-L2 <= 2e-3 against the oracle on the same quantized
operands (the GPU takes its exponentials with ex2.approx and accumulates in
the tensor core, so P codes may flip at rounding boundaries; the oracle
uses exp2f and fp64 sums).  The GPU is also checked against fp64 exact
attention of the bf16 inputs: its cosine must be within 1e-3 of the
oracle's own cosine (the method's accuracy, not a kernel property).

Small shapes are compared in full; the benchmark workloads at full size
are compared on sampled Q blocks (block 0, the last block with its ragged
tail or longest causal rows, and two seeded random blocks per (b, h))."""
import numpy as np
import pytest
import torch

import oracle
import sa3_inputs
from sa3_testutil import bits_to_f32, cosine, qk_sf_to_canonical, rel_l2, sample_units, vt_sf_to_canonical

sa3 = pytest.importorskip("bit_quantized_attention_sa3_b200")

TOL = 2e-3


def _canonical(qz, B, H, N, d):
    Np = sa3.padded_len(N)
    return dict(q_codes=qz.q_fp4.cpu().numpy(), k_codes=qz.k_fp4.cpu().numpy(),
                vt_codes=qz.vt_fp4.cpu().numpy(),
                q_sf=qk_sf_to_canonical(qz.q_sf.cpu().numpy(), B, H, Np, d),
                k_sf=qk_sf_to_canonical(qz.k_sf.cpu().numpy(), B, H, Np, d),
                vt_sf=vt_sf_to_canonical(qz.vt_sf.cpu().numpy(), B, H, Np, d))


def _run(name, over, causal, units=None):
    q, k, v = sa3_inputs.make_qkv(name, shape_override=over)
    B, H, N, d = q.shape
    qz = sa3.quantize_qkv(q.cuda(), k.cuda(), v.cuda())
    out = sa3.attn_fwd(qz, causal=causal)
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    canon = _canonical(qz, B, H, N, d)
    ref = bits_to_f32(oracle.attn_fwd(canon, N, causal, units=units))
    ex = oracle.attn_exact(q, k, v, causal, units=units)
    if units is None:
        mask = np.ones((B * H, N), bool)
    else:
        mask = np.zeros((B * H, N), bool)
        for bh, qb in units:
            mask[bh, qb * 128: min(N, qb * 128 + 128)] = True
    g = got.reshape(B * H, N, d)[mask]
    r = ref.reshape(B * H, N, d)[mask]
    e = ex.reshape(B * H, N, d)[mask]
    return rel_l2(g, r), cosine(g, e), cosine(r, e)


SMALL = [
    ("tiny_b1h2n256d64", None),
    ("tiny_b1h2n256d64", {"N": 1}),
    ("tiny_b1h2n256d64", {"N": 15}),
    ("tiny_b1h2n256d64", {"N": 129}),
    ("tiny_b1h2n256d64", {"N": 300, "H": 3}),
    ("tiny_b1h2n256d64", {"N": 640}),
    ("noncausal_b2h16n4096d128", {"B": 1, "H": 2, "N": 16}),
    ("noncausal_b2h16n4096d128", {"B": 1, "H": 2, "N": 127}),
    ("noncausal_b2h16n4096d128", {"B": 2, "H": 2, "N": 640}),
    ("noncausal_b2h16n4096d128", {"B": 1, "H": 3, "N": 1000}),
]


def _ids(c):
    return c[0] + ("" if c[1] is None else "-" + "-".join(f"{k}{v}" for k, v in c[1].items()))


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True], ids=["noncausal", "causal"])
@pytest.mark.parametrize("case", SMALL, ids=[_ids(c) for c in SMALL])
def test_attn_matches_oracle_small(case, causal):
    err, cos_gpu, cos_oracle = _run(case[0], case[1], causal)
    assert err <= TOL, f"rel-L2 vs oracle {err:.3e}"
    assert cos_gpu >= cos_oracle - 1e-3


FULL = [
    ("noncausal_b2h16n4096d128", False),
    ("videodit_b1h30n17776d64", False),
    ("prefill_b4h32n8192d128_causal", True),
    ("longctx_b1h32n32768d128_causal", True),
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", FULL, ids=[c[0] for c in FULL])
def test_attn_matches_oracle_full_size_sampled(case):
    name, causal = case
    w = sa3_inputs.WORKLOADS[name]
    bh_list = None
    if w.B * w.H > 32:
        rng = np.random.default_rng(2)
        bh_list = sorted({0, w.B * w.H - 1} | set(int(x) for x in rng.choice(w.B * w.H, 14, replace=False)))
    units = sample_units(w.B, w.H, w.N, seed=3, per_bh=2, bh_list=bh_list)
    err, cos_gpu, cos_oracle = _run(name, None, causal, units=units)
    print(f"{name}: rel-L2 vs oracle {err:.3e}, cosine vs exact gpu {cos_gpu:.5f} oracle {cos_oracle:.5f}")
    assert err <= TOL
    assert cos_gpu >= cos_oracle - 1e-3


@pytest.mark.gpu
def test_attn_sm_scale_and_repeatability():
    q, k, v = [t.cuda() for t in sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"N": 384})]
    B, H, N, d = q.shape
    qz = sa3.quantize_qkv(q, k, v)
    a = sa3.attn_fwd(qz, causal=False, sm_scale=0.05)
    b = sa3.attn_fwd(qz, causal=False, sm_scale=0.05)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    canon = _canonical(qz, B, H, N, d)
    ref = bits_to_f32(oracle.attn_fwd(canon, N, False, sm_scale=0.05))
    assert rel_l2(a.float().cpu().numpy(), ref) <= TOL


@pytest.mark.gpu
def test_attn_rejects_bad_arguments():
    q, k, v = [t.cuda() for t in sa3_inputs.make_qkv("tiny_b1h2n256d64")]
    qz = sa3.quantize_qkv(q, k, v)
    bad = sa3.QuantizedQKV(**{**qz.__dict__, "d": 80})
    with pytest.raises(sa3.Sa3Error) as e:
        sa3.attn_fwd(bad)
    assert e.value.code == sa3.SA3_ERR_UNSUPPORTED
    mis = torch.empty(q.numel() + 8, dtype=torch.bfloat16, device="cuda")[1:1 + q.numel()].view(q.shape)
    with pytest.raises(sa3.Sa3Error) as e:
        sa3.attn_fwd(qz, out=mis)
    assert e.value.code == sa3.SA3_ERR_INVALID_ARG


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True], ids=["noncausal", "causal"])
def test_attn_tail_wave_single_tile_units(causal):
    """151 heads x 3 Q tiles = 302 tile pairs: the pairs of the short last
    wave run as single-tile work units; every row must still match."""
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("split point assumes 148 SMs")
    err, cos_gpu, cos_oracle = _run("tiny_b1h2n256d64", {"H": 151, "N": 300}, causal)
    assert err <= TOL, f"rel-L2 vs oracle {err:.3e}"
    assert cos_gpu >= cos_oracle - 1e-3


@pytest.mark.gpu
def test_causal_row0_matches_oracle_exactly():
    """Row 0 sees key 0 only (P = [1, 0, ...], one code and scale decision):
    the GPU must give the oracle's bf16(1.03125 * v^_0) to within one bf16
    ulp, on inputs whose row-0 logits reach far below zero.  (The GPU folds
    log2(1/s) into the exp2 argument, -m' + log2(1/s) rounded at the size of
    m', so with logits in the thousands P carries ~1e-4 relative error and
    some outputs land one ulp away.)"""
    q, k, v = sa3_inputs.make_qkv("prefill_b4h32n8192d128_causal", shape_override={"B": 1, "H": 32, "N": 1024})
    B, H, N, d = q.shape
    qz = sa3.quantize_qkv(q.cuda(), k.cuda(), v.cuda())
    out = sa3.attn_fwd(qz, causal=True)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    ref = oracle.attn_fwd(_canonical(qz, B, H, N, d), N, True, units=[(bh, 0) for bh in range(B * H)])
    got = out[:, :, 0].float().cpu().numpy()
    want = bits_to_f32(ref[:, :, 0])
    assert np.all(np.abs(got - want) <= 2.0 ** -7 * np.abs(want))


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True], ids=["noncausal", "causal"])
def test_long_sequence_131072_tokens(causal):
    """Four times the longest workload: B=1, H=2, N=131072, d=128 (its
    distribution).  Quantization bit-exact on the whole tensors; attention
    against the oracle on the first, the last and one seeded block of each
    head (the last block's causal rows see all 131072 keys)."""
    name, over = "longctx_b1h32n32768d128_causal", {"H": 2, "N": 131072}
    q, k, v = sa3_inputs.make_qkv(name, shape_override=over)
    B, H, N, d = q.shape
    qz = sa3.quantize_qkv(q.cuda(), k.cuda(), v.cuda())
    out = sa3.attn_fwd(qz, causal=causal)
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    canon = _canonical(qz, B, H, N, d)
    if not causal:  # the quantized operands do not depend on the mask: compare once
        r = oracle.quantize_qkv(q, k, v)
        for f in ("q_codes", "q_sf", "k_codes", "k_sf", "vt_codes", "vt_sf"):
            assert np.array_equal(canon[f], r[f]), f
        assert np.array_equal(qz.k_mean.cpu().numpy().view(np.uint32), r["k_mean"].view(np.uint32))
    nqb = N // 128
    units = [(bh, qb) for bh in range(B * H) for qb in (0, nqb - 1, 517)]
    ref = bits_to_f32(oracle.attn_fwd(canon, N, causal, units=units)).reshape(B * H, N, d)
    got = out.float().cpu().numpy().reshape(B * H, N, d)
    assert np.isfinite(got).all()
    for bh, qb in units:
        rows = slice(qb * 128, qb * 128 + 128)
        assert rel_l2(got[bh, rows], ref[bh, rows]) <= TOL, (bh, qb)


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True], ids=["noncausal", "causal"])
def test_many_heads_beyond_65535(causal):
    """B*H = 66000 short heads (N = 40, d = 64): grids are one-dimensional,
    so B*H is bounded only by the size limit.  Heads on both sides of
    65536 and the last one are compared with the oracle run on their slice
    (quantization and attention of one head do not depend on the others)."""
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"B": 2, "H": 33000, "N": 40})
    B, H, N, d = q.shape
    qz = sa3.quantize_qkv(q.cuda(), k.cuda(), v.cuda())
    out = sa3.attn_fwd(qz, causal=causal)
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    codes = qz.k_fp4.cpu().numpy()
    for bh in (0, 65535, 65536, B * H - 1):
        b, h = divmod(bh, H)
        sl = slice(b, b + 1), slice(h, h + 1)
        r = oracle.quantize_qkv(q[sl].contiguous(), k[sl].contiguous(), v[sl].contiguous())
        assert np.array_equal(codes[b, h], r["k_codes"][0, 0]), bh
        ref = bits_to_f32(oracle.attn_fwd(r, N, causal))[0, 0]
        assert rel_l2(bits_to_f32(got[b, h]), ref) <= TOL, bh
