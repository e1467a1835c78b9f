"""sa3_quantize_qkv on the GPU against the CPU oracle: codes, scales and the
K mean must be bit-identical (integer / byte work).  Full tensors for the
small cases and the headline case; for the three largest workloads a
seeded sample of (b, h) slices is compared in full (quantization of one
slice does not depend on the others)."""
import numpy as np
import pytest
import torch

import oracle
import sa3_inputs
from sa3_testutil import fp64_sum_is_exact, qk_sf_to_canonical, vt_sf_padding, vt_sf_to_canonical

sa3 = pytest.importorskip("bit_quantized_attention_sa3_b200")

CASES = [
    ("tiny_b1h2n256d64", None),
    ("tiny_b1h2n256d64", {"N": 1}),
    ("tiny_b1h2n256d64", {"N": 15}),
    ("tiny_b1h2n256d64", {"N": 129}),
    ("tiny_b1h2n256d64", {"N": 700, "H": 3}),
    ("noncausal_b2h16n4096d128", {"B": 1, "H": 2, "N": 17}),
    ("noncausal_b2h16n4096d128", {"B": 1, "H": 3, "N": 1100}),
    ("noncausal_b2h16n4096d128", None),
    ("videodit_b1h30n17776d64", None),
    ("prefill_b4h32n8192d128_causal", None),
    ("longctx_b1h32n32768d128_causal", None),
]
LARGE = {"videodit_b1h30n17776d64", "prefill_b4h32n8192d128_causal", "longctx_b1h32n32768d128_causal"}


def _ids(c):
    return c[0] + ("" if c[1] is None else "-" + "-".join(f"{k}{v}" for k, v in c[1].items()))


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_quantize_matches_oracle_bit_exact(case):
    name, over = case
    q, k, v = sa3_inputs.make_qkv(name, shape_override=over)
    B, H, N, d = q.shape
    Np = sa3.padded_len(N)
    # the K mean is order independent (hence bit-exact) only if its fp64 sum is exact
    assert fp64_sum_is_exact(k)
    qz = sa3.quantize_qkv(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    g = {f: getattr(qz, f).cpu().numpy() for f in ("q_fp4", "q_sf", "k_fp4", "k_sf", "vt_fp4", "vt_sf", "k_mean")}
    g["q_sf"] = qk_sf_to_canonical(g["q_sf"], B, H, Np, d)
    g["k_sf"] = qk_sf_to_canonical(g["k_sf"], B, H, Np, d)
    pad = vt_sf_padding(g["vt_sf"], B, H, Np, d)
    assert not pad.any()
    g["vt_sf"] = vt_sf_to_canonical(g["vt_sf"], B, H, Np, d)

    if name in LARGE and over is None:
        rng = np.random.default_rng(1)
        bhs = sorted({0, B * H - 1} | set(int(x) for x in rng.choice(B * H, 2, replace=False)))
    else:
        bhs = list(range(B * H))
    for bh in bhs:
        b, h = divmod(bh, H)
        sl = slice(b, b + 1), slice(h, h + 1)
        r = oracle.quantize_qkv(q[sl].contiguous(), k[sl].contiguous(), v[sl].contiguous())
        mapping = {"q_fp4": "q_codes", "q_sf": "q_sf", "k_fp4": "k_codes", "k_sf": "k_sf",
                   "vt_fp4": "vt_codes", "vt_sf": "vt_sf", "k_mean": "k_mean"}
        for gf, of in mapping.items():
            got = g[gf][b, h]
            want = r[of][0, 0]
            if gf == "k_mean":
                ok = np.array_equal(got.view(np.uint32), want.view(np.uint32))
            else:
                ok = np.array_equal(got, want)
            if not ok:
                bad = np.argwhere(got != want)
                pytest.fail(f"{gf} differs at bh={bh}: {len(bad)} mismatches, first {bad[:5].tolist()} "
                            f"got {got[tuple(bad[0])]} want {want[tuple(bad[0])]}")


@pytest.mark.gpu
def test_quantize_repeatable_and_ignores_workspace_contents():
    q, k, v = [t.cuda() for t in sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"N": 600})]
    B, H, N, d = q.shape
    ws = torch.full((sa3.quant_workspace_bytes(B, H, N, d),), 0xAB, dtype=torch.uint8, device="cuda")
    a = sa3.quantize_qkv(q, k, v, workspace=ws)
    b = sa3.quantize_qkv(q, k, v)
    torch.cuda.synchronize()
    for f in ("q_fp4", "q_sf", "k_fp4", "k_sf", "vt_fp4", "vt_sf", "k_mean"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f


@pytest.mark.gpu
def test_quantize_rejects_bad_arguments():
    import ctypes
    q, k, v = [t.cuda() for t in sa3_inputs.make_qkv("tiny_b1h2n256d64")]
    B, H, N, d = q.shape
    out = sa3.empty_quantized(B, H, N, d)
    small = torch.empty(8, dtype=torch.uint8, device="cuda")
    # the binding checks the workspace first; the library checks it again
    with pytest.raises(ValueError):
        sa3.quantize_qkv(q, k, v, out=out, workspace=small)
    st = out.struct()
    stream = torch.cuda.current_stream().cuda_stream
    rc = sa3.lib().sa3_quantize_qkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, N, d, ctypes.byref(st),
                                    small.data_ptr(), small.numel(), stream)
    assert rc == sa3.SA3_ERR_INVALID_ARG
    # an output or the workspace sharing bytes with an input is rejected
    rc = sa3.lib().sa3_quantize_qkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, N, d, ctypes.byref(st),
                                    k.data_ptr(), sa3.quant_workspace_bytes(B, H, N, d), stream)
    assert rc == sa3.SA3_ERR_INVALID_ARG
    alias = sa3._QKV(*[getattr(st, f) for f, _ in sa3._QKV._fields_])
    alias.vt_fp4 = v.data_ptr() + 64
    ws = torch.empty(sa3.quant_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    rc = sa3.lib().sa3_quantize_qkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, N, d, ctypes.byref(alias),
                                    ws.data_ptr(), ws.numel(), stream)
    assert rc == sa3.SA3_ERR_INVALID_ARG
    q96 = torch.zeros((1, 1, 16, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sa3.Sa3Error) as e:
        sa3.quantize_qkv(q96, q96, q96)
    assert e.value.code == sa3.SA3_ERR_UNSUPPORTED


def _offset16(t):
    """A copy of t's shape and dtype whose storage starts 16 bytes past a
    256-byte boundary: 16-byte aligned (the ABI's requirement), not 32."""
    n = t.numel() * t.element_size()
    buf = torch.empty(n + 256, dtype=torch.uint8, device=t.device)
    base = (-buf.data_ptr()) % 256 + 16
    out = buf[base:base + n].view(t.dtype).view(t.shape)
    assert out.data_ptr() % 32 == 16
    return out


@pytest.mark.gpu
@pytest.mark.parametrize("d", [64, 128])
def test_quantize_outputs_only_16_byte_aligned(d):
    """The tiles store 32-byte pieces in one instruction when every code
    output is 32-byte aligned, else in 16-byte pieces: same bytes."""
    import dataclasses
    q, k, v = [t.cuda() for t in sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"N": 300, "d": d})]
    a = sa3.quantize_qkv(q, k, v)
    b = sa3.empty_quantized(1, 2, 300, d)
    b = dataclasses.replace(b, **{f: _offset16(getattr(b, f)) for f in ("q_fp4", "k_fp4", "vt_fp4")})
    sa3.quantize_qkv(q, k, v, out=b)
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    for f in ("q_fp4", "q_sf", "k_fp4", "k_sf", "vt_fp4", "vt_sf", "k_mean"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f


@pytest.mark.gpu
@pytest.mark.parametrize("d", [64, 128])
def test_quantize_i8_outputs_only_16_byte_aligned(d):
    import dataclasses
    q, k, v = [t.cuda() for t in sa3_inputs.make_qkv("tiny_b1h2n256d64", shape_override={"N": 300, "d": d})]
    a = sa3.quantize_qkv_i8(q, k, v)
    b = sa3.empty_quantized_i8(1, 2, 300, d)
    b = dataclasses.replace(b, **{f: _offset16(getattr(b, f)) for f in ("q_i8", "k_i8", "vt_f16")})
    sa3.quantize_qkv_i8(q, k, v, out=b)
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    for f in ("q_i8", "q_scale", "k_i8", "k_scale", "vt_f16", "k_mean"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f
