"""The training forward of the 8-bit variant (sa3_attn_fwd_i8_lse) on the
GPU: the per-row log-sum-exp against the oracle (reading I6), and the
output unchanged by asking for it.

Tolerance on lse: the kernel and the oracle take the same fp32 steps for t
and for the running maximum m (the integer S is exact, f is formed in the
same order), so they differ through l: ex2.approx against exp2f (a few
2^-23 relative per term) and the order of the fp32 sums.  A relative error
e in l moves lse by about e; 3e-5 absolute leaves two orders of magnitude
over the typical sqrt(N) * 2^-24 of a 4096-term sum.  The kernel also forms
m + log2 l and its product with ln 2 in fp32 where the oracle rounds once
from fp64: up to about two fp32 ulps of |lse|, which matters where logits
are large (the prefill workload's outlier channels give lse near 600, where
an ulp is 6e-5); the bound adds four ulps, 4 * 2^-23 * |lse|.  Rows that
see no key are +inf on both sides."""
import numpy as np
import pytest
import torch

import oracle
import sa3_inputs
from sa3_testutil import heads_of
from test_i8_gpu import CASES, _canon, _ids, _qkv, assert_i8_equal

sa3 = pytest.importorskip("bit_quantized_attention_sa3_b200")

LSE_ATOL = 3e-5
LSE_ULPS = 4 * 2.0 ** -23


def _check_lse(got, ref):
    assert np.array_equal(np.isposinf(got), np.isposinf(ref))
    assert not np.isnan(got).any()
    fin = np.isfinite(ref)
    if fin.any():
        err = np.abs(got[fin].astype(np.float64) - ref[fin])
        bound = LSE_ATOL + LSE_ULPS * np.abs(ref[fin].astype(np.float64))
        assert (err <= bound).all(), f"lse error {err.max():.3e}, worst ratio to bound {(err / bound).max():.2f}"


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True], ids=["noncausal", "causal"])
@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_lse_matches_oracle(case, causal):
    name, Nq, Nkv, over = case
    q, k, v = _qkv(name, Nq, Nkv, over)
    qz = sa3.quantize_qkv_i8(q.cuda(), k.cuda(), v.cuda())
    plain = sa3.attn_fwd_i8(qz, causal=causal)
    out, lse = sa3.attn_fwd_i8(qz, causal=causal, lse=True)
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    assert torch.equal(out, plain)
    r_q = oracle.quantize_qkv_i8(q, k, v)
    assert_i8_equal(_canon(qz), r_q)
    _, ref = oracle.attn_fwd_i8(r_q, Nq, causal, n_kv=Nkv, return_lse=True)
    _check_lse(lse.cpu().numpy(), ref)
    if causal and Nq > Nkv:
        assert np.isposinf(lse[:, :, : Nq - Nkv].cpu().numpy()).all()


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True], ids=["noncausal", "causal"])
def test_lse_full_size_sampled_units(causal):
    """B=2, H=16, N=4096, d=128 in the launch the benchmark times; the
    oracle recomputes a sample of (head, 128-row tile) units, first and last
    tiles included."""
    q, k, v = sa3_inputs.make_qkv("noncausal_b2h16n4096d128")
    B, H, N, d = q.shape
    qz = sa3.quantize_qkv_i8(q.cuda(), k.cuda(), v.cuda())
    out, lse = sa3.attn_fwd_i8(qz, causal=causal, lse=True)
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    rng = np.random.default_rng(7)
    nqb = N // 128
    units = [(0, 0), (B * H - 1, nqb - 1)] + [(int(rng.integers(B * H)), int(rng.integers(nqb))) for _ in range(4)]
    heads = sorted({bh for bh, _ in units})
    pos = {bh: i for i, bh in enumerate(heads)}
    # the oracle quantizes the sampled heads itself; they must equal the GPU's
    r_q = oracle.quantize_qkv_i8(heads_of(q, heads), heads_of(k, heads), heads_of(v, heads))
    g = _canon(qz)
    for f in ("q_i8", "q_scale", "k_i8", "k_scale", "vt_f16", "k_mean"):
        gf = g[f].reshape((B * H,) + g[f].shape[2:])[heads]
        rf = r_q[f].reshape((len(heads),) + r_q[f].shape[2:])
        assert np.array_equal(gf.view(np.uint8), rf.view(np.uint8)), f
    sub = [(pos[bh], qb) for bh, qb in units]
    ref_out, ref = oracle.attn_fwd_i8(r_q, N, causal, units=sub, return_lse=True)
    got = lse.cpu().numpy().reshape(B * H, N)
    ref = ref.reshape(len(heads), N)
    o = out.view(torch.int16).cpu().numpy().view(np.uint16).reshape(B * H, N, d)
    ro = ref_out.reshape(len(heads), N, d)
    for bh, qb in units:
        rows = slice(qb * 128, qb * 128 + 128)
        _check_lse(got[bh, rows], ref[pos[bh], rows])
        a = oracle.bf16_bits_to_f32(o[bh, rows]).astype(np.float64)
        r = oracle.bf16_bits_to_f32(ro[pos[bh], rows]).astype(np.float64)
        assert np.linalg.norm(a - r) / np.linalg.norm(r) <= 2e-3


@pytest.mark.gpu
def test_lse_argument_checks():
    import ctypes
    q, k, v = [t.cuda() for t in sa3_inputs.make_qkv("tiny_b1h2n256d64")]
    qz = sa3.quantize_qkv_i8(q, k, v)
    out = torch.empty_like(q)
    buf = torch.empty(2 * 256 + 1, dtype=torch.float32, device="cuda")
    rc = sa3.lib().sa3_attn_fwd_i8_lse(ctypes.byref(qz.struct()), 1, 2, 256, 256, 64, 0, 0.0, out.data_ptr(),
                                       buf.data_ptr() + 2, torch.cuda.current_stream().cuda_stream)
    assert rc == sa3.SA3_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        sa3.attn_fwd_i8(qz, lse=torch.empty(7, dtype=torch.float32, device="cuda"))
