"""SA3_P_TWO_LEVEL on the GPU against the oracle with p_two_level=True.

Bar as for the default recipe: the GPU's quantized operands equal the
oracle's, then output rel-L2 <= 2e-3 in every (head, Q block) against the
oracle attending on its own operands, cosine against fp64 exact attention
within 1e-3 of the oracle's.  Covers the self-attention and the unequal-length
kernel instances."""
import numpy as np
import pytest
import torch

import oracle
import sa3_inputs
from sa3_testutil import assert_quantized_equal, bits_to_f32, blockwise_rel_l2, cosine, gpu_canonical

sa3 = pytest.importorskip("bit_quantized_attention_sa3_b200")

TOL = 2e-3

CASES = [
    ("tiny_b1h2n256d64", 300, 300, {"H": 3}),
    ("noncausal_b2h16n4096d128", 640, 640, {"B": 2, "H": 2}),
    ("videodit_b1h30n17776d64", 1000, 1000, {"H": 2}),
    ("longctx_b1h32n32768d128_causal", 1024, 1024, {"H": 2}),
    ("noncausal_b2h16n4096d128", 77, 1000, {"B": 1, "H": 2}),
]


def _ids(c):
    return f"{c[0]}-q{c[1]}-kv{c[2]}"


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True], ids=["noncausal", "causal"])
@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_two_level_matches_oracle(case, causal):
    name, Nq, Nkv, over = case
    o = dict(over)
    o["N"] = max(Nq, Nkv)
    q, k, v = sa3_inputs.make_qkv(name, shape_override=o)
    q, k, v = q[:, :, :Nq].contiguous(), k[:, :, :Nkv].contiguous(), v[:, :, :Nkv].contiguous()
    B, H, _, d = q.shape
    qz = sa3.quantize_qkv(q.cuda(), k.cuda(), v.cuda())
    out = sa3.attn_fwd(qz, causal=causal, p_two_level=True)
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    r_q = oracle.quantize_qkv(q, k, v)
    assert_quantized_equal(gpu_canonical(qz, B, H, Nq, Nkv, d), r_q, range(B * H))
    o32 = np.zeros((B, H, Nq, d), np.float32)
    ref = bits_to_f32(oracle.attn_fwd(r_q, Nq, causal, n_kv=Nkv, p_two_level=True, out32=o32))
    ex = oracle.attn_exact(q, k, v, causal)
    live = (np.arange(Nq) + (Nkv - Nq) >= 0) if causal else np.ones(Nq, bool)
    blocks = [(h, qb) for h in range(B * H) for qb in range((Nq + 127) // 128)]
    blockwise_rel_l2(got.reshape(B * H, Nq, d), ref.reshape(B * H, Nq, d), blocks, TOL, live=live,
                     label=_ids(case), ref32=o32.reshape(B * H, Nq, d))
    g, r, e = got[:, :, live], ref[:, :, live], ex[:, :, live]
    assert cosine(g, e) >= cosine(r, e) - 1e-3


@pytest.mark.gpu
def test_unknown_flag_bits_are_rejected():
    q, k, v = [t.cuda() for t in sa3_inputs.make_qkv("tiny_b1h2n256d64")]
    qz = sa3.quantize_qkv(q, k, v)
    out = torch.empty_like(q)
    import ctypes
    rc = sa3.lib().sa3_attn_fwd_lens(ctypes.byref(qz.struct()), 1, 2, 256, 256, 64, 0, 0.0, 2, out.data_ptr(),
                                     torch.cuda.current_stream().cuda_stream)
    assert rc == sa3.SA3_ERR_INVALID_ARG
