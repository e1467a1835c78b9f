"""Q quantized on load (SA3_SKIP_Q + SA3_Q_ON_LOAD): the quantizer leaves Q
alone and the attention kernel quantizes each bf16 Q tile itself with the
quantizer's block recipe.  The codes must be the quantizer's bit for bit, so
the output must equal the two-pass path's bit for bit, on every shape and
option; at full size it is also checked against the oracle chain."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import sa3_inputs
from sa3_testutil import bits_to_f32, blockwise_rel_l2, heads_of, sample_units

sa3 = pytest.importorskip("bit_quantized_attention_sa3_b200")

CASES = [
    ("tiny_b1h2n256d64", 300, 300, {"H": 3}),
    ("tiny_b1h2n256d64", 1, 300, None),
    ("noncausal_b2h16n4096d128", 640, 640, {"B": 2, "H": 2}),
    ("noncausal_b2h16n4096d128", 77, 1000, {"B": 1, "H": 2}),
    ("noncausal_b2h16n4096d128", 1000, 130, {"B": 1, "H": 2}),
    ("videodit_b1h30n17776d64", 1000, 1000, {"H": 2}),
    ("tiny_b1h2n256d64", 300, 200, {"H": 151}),  # a last wave of single-tile units
]


def _ids(c):
    return f"{c[0]}-q{c[1]}-kv{c[2]}" + ("" if c[3] is None else "-" + "-".join(f"{k}{v}" for k, v in c[3].items()))


def _qkv(name, Nq, Nkv, over):
    o = dict(over or {})
    o["N"] = max(Nq, Nkv)
    q, k, v = sa3_inputs.make_qkv(name, shape_override=o)
    return q[:, :, :Nq].contiguous(), k[:, :, :Nkv].contiguous(), v[:, :, :Nkv].contiguous()


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_q_on_load_equals_two_pass_path(case):
    name, Nq, Nkv, over = case
    q, k, v = [t.cuda() for t in _qkv(name, Nq, Nkv, over)]
    full = sa3.quantize_qkv(q, k, v)
    kv = sa3.quantize_qkv(q, k, v, skip_q=True)
    torch.cuda.synchronize()
    assert kv.q_fp4 is None and kv.q_sf is None
    for f in ("k_fp4", "k_sf", "vt_fp4", "vt_sf", "k_mean"):
        assert torch.equal(getattr(kv, f), getattr(full, f)), f
    for causal in (False, True):
        for two in (False, True):
            ref = sa3.attn_fwd(full, causal=causal, p_two_level=two)
            got = sa3.attn_fwd(kv, causal=causal, p_two_level=two, q=q)
            again = sa3.attn_fwd(full, causal=causal, p_two_level=two, q=q)  # Q codes given but not read
            torch.cuda.synchronize()
            assert sa3.device_status() == sa3.SA3_OK
            assert torch.equal(got, ref), (causal, two)
            assert torch.equal(again, ref), (causal, two)


@pytest.mark.gpu
def test_q_on_load_with_v_smoothing():
    q, k, v = [t.cuda() for t in _qkv("noncausal_b2h16n4096d128", 500, 700, {"B": 1, "H": 2})]
    full = sa3.quantize_qkv(q, k, v, v_smooth=True)
    kv = sa3.quantize_qkv(q, k, v, v_smooth=True, skip_q=True)
    for causal in (False, True):
        ref = sa3.attn_fwd(full, causal=causal)
        got = sa3.attn_fwd(kv, causal=causal, q=q)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)


@pytest.mark.gpu
def test_q_on_load_full_size_against_the_oracle():
    """The headline workload B=2, H=16, N=4096, d=128 as the bench runs it:
    bit-identical to the two-pass path, and on sampled (head, Q block) units
    within the per-block bar of the oracle attending on its own operands."""
    name = "noncausal_b2h16n4096d128"
    w = sa3_inputs.WORKLOADS[name]
    q, k, v = sa3_inputs.make_qkv(name)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    ref = sa3.attn_fwd(sa3.quantize_qkv(qd, kd, vd))
    got = sa3.attn_fwd(sa3.quantize_qkv(qd, kd, vd, skip_q=True), q=qd)
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    assert torch.equal(got, ref)
    units = sample_units(w.B, w.H, w.N, seed=5, per_bh=1, bh_list=[0, 7, 31])
    heads = sorted({bh for bh, _ in units})
    pos = {bh: i for i, bh in enumerate(heads)}
    rq = oracle.quantize_qkv(heads_of(q, heads), heads_of(k, heads), heads_of(v, heads))
    sub = [(pos[bh], qb) for bh, qb in units]
    o32 = np.zeros((1, len(heads), w.N, w.d), np.float32)
    r = bits_to_f32(oracle.attn_fwd(rq, w.N, False, units=sub, out32=o32))[0]
    g = got.float().cpu().numpy().reshape(w.B * w.H, w.N, w.d)[heads]
    blockwise_rel_l2(g, r, sub, 2e-3, label="Q on load, full size", ref32=o32[0])


@pytest.mark.gpu
def test_q_on_load_argument_checks():
    q, k, v = [t.cuda() for t in sa3_inputs.make_qkv("tiny_b1h2n256d64")]
    B, H, N, d = q.shape
    kv = sa3.quantize_qkv(q, k, v, skip_q=True)
    with pytest.raises(ValueError):
        sa3.attn_fwd(kv)  # no Q codes and no q
    out = torch.empty_like(q)
    st = kv.struct()
    stream = torch.cuda.current_stream().cuda_stream
    rc = sa3.lib().sa3_attn_fwd_ex(ctypes.byref(st), None, None, B, H, N, N, d, 0, 0.0, sa3.SA3_Q_ON_LOAD,
                                   out.data_ptr(), stream)
    assert rc == sa3.SA3_ERR_INVALID_ARG  # Q on load without q
    rc = sa3.lib().sa3_attn_fwd_ex(ctypes.byref(st), None, None, B, H, N, N, d, 0, 0.0, 0, out.data_ptr(), stream)
    assert rc == sa3.SA3_ERR_INVALID_ARG  # no Q codes and no flag


@pytest.mark.gpu
def test_q_written_by_the_kernel_just_before():
    """The attention kernel is a programmatic dependent launch: with Q on
    load, its Q reads must still come after the preceding kernel's writes.
    Here the kernel just before the attention launch writes the Q it reads."""
    q, k, v = [t.cuda() for t in _qkv("noncausal_b2h16n4096d128", 1000, 1000, {"B": 1, "H": 4})]
    kv = sa3.quantize_qkv(q, k, v, skip_q=True)
    ref = sa3.attn_fwd(kv, q=q)
    for i in range(3):
        q2 = torch.empty_like(q)
        torch.mul(q, 1.0, out=q2)  # an elementwise kernel (x * 1 is exact), right before the attention launch
        got = sa3.attn_fwd(kv, q=q2)
        torch.cuda.synchronize()
        assert sa3.device_status() == sa3.SA3_OK
        assert torch.equal(got, ref), i
