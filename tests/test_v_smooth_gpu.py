"""V smoothing (SA3_V_SMOOTH) on the GPU against the oracle's smooth_v
recipe (reading R13): V_s = fp32(V) - mean of V over the keys, quantized
like V; out = bf16(O / l + mean).

The inputs get a per-channel V offset (the case smoothing is for).  Bars:
codes, scales, the K mean and the V mean bit-exact; then the oracle attends
on its own operands and the GPU output must be within rel-L2 2e-3 in every
(head, 128-row Q block); rows that see no key are 0 on both sides."""
import numpy as np
import pytest
import torch

import oracle
import sa3_inputs
from sa3_testutil import assert_quantized_equal, bits_to_f32, blockwise_rel_l2, fp64_sum_is_exact, gpu_canonical

sa3 = pytest.importorskip("bit_quantized_attention_sa3_b200")

TOL = 2e-3

CASES = [
    ("tiny_b1h2n256d64", 300, 300, {"H": 3}),
    ("noncausal_b2h16n4096d128", 640, 640, {"B": 2, "H": 2}),
    ("videodit_b1h30n17776d64", 1000, 1000, {"H": 2}),
    ("noncausal_b2h16n4096d128", 77, 1000, {"B": 1, "H": 2}),
    ("prefill_b4h32n8192d128_causal", 1000, 130, {"B": 1, "H": 2}),
]


def _ids(c):
    return f"{c[0]}-q{c[1]}-kv{c[2]}"


def _qkv(name, Nq, Nkv, over):
    o = dict(over)
    o["N"] = max(Nq, Nkv)
    q, k, v = sa3_inputs.make_qkv(name, shape_override=o)
    B, H, _, d = v.shape
    g = torch.Generator().manual_seed(77)
    off = (torch.randn((B, H, 1, d), generator=g) * 8.0).to(torch.bfloat16).float()
    v = (v.float() + off).to(torch.bfloat16)  # exact in fp32, one bf16 rounding
    return q[:, :, :Nq].contiguous(), k[:, :, :Nkv].contiguous(), v[:, :, :Nkv].contiguous()


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True], ids=["noncausal", "causal"])
@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_v_smooth_matches_oracle(case, causal):
    name, Nq, Nkv, over = case
    q, k, v = _qkv(name, Nq, Nkv, over)
    B, H, _, d = q.shape
    assert fp64_sum_is_exact(k) and fp64_sum_is_exact(v)
    qz = sa3.quantize_qkv(q.cuda(), k.cuda(), v.cuda(), v_smooth=True)
    out = sa3.attn_fwd(qz, causal=causal)
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    r_q = oracle.quantize_qkv(q, k, v, smooth_v=True)
    assert_quantized_equal(gpu_canonical(qz, B, H, Nq, Nkv, d), r_q, range(B * H))
    assert np.array_equal(qz.v_mean.cpu().numpy().view(np.uint32), r_q["v_mean"].view(np.uint32))
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    o32 = np.zeros((B, H, Nq, d), np.float32)
    ref = bits_to_f32(oracle.attn_fwd(r_q, Nq, causal, n_kv=Nkv, out32=o32))
    live = (np.arange(Nq) + (Nkv - Nq) >= 0) if causal else np.ones(Nq, bool)
    if causal:
        assert not got[:, :, ~live].any() and not ref[:, :, ~live].any()
    blocks = [(h, qb) for h in range(B * H) for qb in range((Nq + 127) // 128)]
    blockwise_rel_l2(got.reshape(B * H, Nq, d), ref.reshape(B * H, Nq, d), blocks, TOL, live=live,
                     label=_ids(case), ref32=o32.reshape(B * H, Nq, d))


@pytest.mark.gpu
def test_v_smooth_helps_with_a_channel_offset():
    """What the option is for: with a large per-channel V offset, smoothing
    brings the output closer to fp64 exact attention (the oracle shows the
    same; here the GPU must reproduce the gain)."""
    q, k, v = _qkv("noncausal_b2h16n4096d128", 512, 512, {"B": 1, "H": 2})
    plain = sa3.attn_fwd(sa3.quantize_qkv(q.cuda(), k.cuda(), v.cuda()))
    smooth = sa3.attn_fwd(sa3.quantize_qkv(q.cuda(), k.cuda(), v.cuda(), v_smooth=True))
    torch.cuda.synchronize()
    ex = oracle.attn_exact(q, k, v, False)
    mean = ex.mean(axis=2, keepdims=True)  # centred: the offset itself is reproduced by both

    def centred_cos(a):
        a = a.float().cpu().numpy().astype(np.float64) - mean
        b = ex - mean
        return float((a * b).sum() / np.sqrt((a * a).sum() * (b * b).sum()))
    assert centred_cos(smooth) > centred_cos(plain) + 0.01


@pytest.mark.gpu
def test_v_smooth_argument_checks():
    import ctypes
    q, k, v = [t.cuda() for t in sa3_inputs.make_qkv("tiny_b1h2n256d64")]
    B, H, N, d = q.shape
    qz = sa3.quantize_qkv(q, k, v, v_smooth=True)
    st = qz.struct()
    stream = torch.cuda.current_stream().cuda_stream
    ws = torch.empty(sa3.quant_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")  # half of what it needs
    rc = sa3.lib().sa3_quantize_qkv_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, N, N, d, sa3.SA3_V_SMOOTH,
                                       ctypes.byref(st), qz.v_mean.data_ptr(), ws.data_ptr(), ws.numel(), stream)
    assert rc == sa3.SA3_ERR_INVALID_ARG
    rc = sa3.lib().sa3_quantize_qkv_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, N, N, d, sa3.SA3_V_SMOOTH,
                                       ctypes.byref(st), None, ws.data_ptr(), 2 * ws.numel(), stream)
    assert rc == sa3.SA3_ERR_INVALID_ARG  # no v_mean
    out = torch.empty_like(q)
    rc = sa3.lib().sa3_attn_fwd_ex(ctypes.byref(st), None, None, B, H, N, N, d, 0, 0.0, sa3.SA3_V_SMOOTH,
                                   out.data_ptr(), stream)
    assert rc == sa3.SA3_ERR_INVALID_ARG
    rc = sa3.lib().sa3_attn_fwd_ex(ctypes.byref(st), None, None, B, H, N, N, d, 0, 0.0, 16, out.data_ptr(), stream)
    assert rc == sa3.SA3_ERR_INVALID_ARG  # unknown flag
