"""sa3_quantize_qkv_lens / sa3_attn_fwd_lens on the GPU against the CPU
oracle: queries of length Nq, keys and values of length Nkv (Nq != Nkv).

Bars as for the self-attention calls: quantized codes, scales and the K
mean bit-exact; attention output rel-L2 <= 2e-3 against the oracle on the
oracle's own quantized operands in every (head, 128-row Q block), after
the GPU's operands have been checked equal to the oracle's; cosine against
fp64 exact attention within 1e-3 of the oracle's.  With the causal mask the last query is aligned with the
last key, and rows that see no key must be exactly 0 on both sides."""
import numpy as np
import pytest
import torch

import oracle
import sa3_inputs
from sa3_testutil import (assert_quantized_equal, bits_to_f32, blockwise_rel_l2, cosine, fp64_sum_is_exact,
                          gpu_canonical, qk_sf_to_canonical, vt_sf_padding, vt_sf_to_canonical)

sa3 = pytest.importorskip("bit_quantized_attention_sa3_b200")

TOL = 2e-3


def _qkv(name, Nq, Nkv, over=None):
    """Seeded draws of the workload's distribution, Q cut to Nq tokens and
    K, V to Nkv."""
    o = dict(over or {})
    o["N"] = max(Nq, Nkv)
    q, k, v = sa3_inputs.make_qkv(name, shape_override=o)
    return q[:, :, :Nq].contiguous(), k[:, :, :Nkv].contiguous(), v[:, :, :Nkv].contiguous()


def _canonical(qz, B, H, Nq, Nkv, d):
    Npq, Np = sa3.padded_len(Nq), sa3.padded_len(Nkv)
    g = {f: getattr(qz, f).cpu().numpy() for f in ("q_fp4", "q_sf", "k_fp4", "k_sf", "vt_fp4", "vt_sf", "k_mean")}
    assert not vt_sf_padding(g["vt_sf"], B, H, Np, d).any()
    return dict(q_codes=g["q_fp4"], k_codes=g["k_fp4"], vt_codes=g["vt_fp4"], k_mean=g["k_mean"],
                q_sf=qk_sf_to_canonical(g["q_sf"], B, H, Npq, d),
                k_sf=qk_sf_to_canonical(g["k_sf"], B, H, Np, d),
                vt_sf=vt_sf_to_canonical(g["vt_sf"], B, H, Np, d), n_kv=Nkv)


CASES = [
    ("tiny_b1h2n256d64", 1, 300, None),
    ("tiny_b1h2n256d64", 300, 17, {"H": 3}),
    ("noncausal_b2h16n4096d128", 77, 1000, {"B": 1, "H": 2}),
    ("noncausal_b2h16n4096d128", 640, 129, {"B": 2, "H": 2}),
    ("noncausal_b2h16n4096d128", 1000, 130, {"B": 1, "H": 2}),
    ("videodit_b1h30n17776d64", 200, 333, {"H": 2}),
]


def _ids(c):
    return f"{c[0]}-q{c[1]}-kv{c[2]}" + ("" if c[3] is None else "-" + "-".join(f"{k}{v}" for k, v in c[3].items()))


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_quantize_lens_matches_oracle_bit_exact(case):
    name, Nq, Nkv, over = case
    q, k, v = _qkv(name, Nq, Nkv, over)
    B, H, _, d = q.shape
    assert fp64_sum_is_exact(k)
    qz = sa3.quantize_qkv(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    assert qz.q_fp4.shape[2] == sa3.padded_len(Nq) and qz.k_fp4.shape[2] == sa3.padded_len(Nkv)
    g = _canonical(qz, B, H, Nq, Nkv, d)
    r = oracle.quantize_qkv(q, k, v)
    for gf, of in (("q_codes", "q_codes"), ("q_sf", "q_sf"), ("k_codes", "k_codes"), ("k_sf", "k_sf"),
                   ("vt_codes", "vt_codes"), ("vt_sf", "vt_sf")):
        if not np.array_equal(g[gf], r[of]):
            bad = np.argwhere(g[gf] != r[of])
            pytest.fail(f"{gf}: {len(bad)} mismatches, first {bad[:5].tolist()}")
    assert np.array_equal(g["k_mean"].view(np.uint32), r["k_mean"].view(np.uint32))


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True], ids=["noncausal", "causal"])
@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_attn_lens_matches_oracle(case, causal):
    name, Nq, Nkv, over = case
    q, k, v = _qkv(name, Nq, Nkv, over)
    B, H, _, d = q.shape
    qz = sa3.quantize_qkv(q.cuda(), k.cuda(), v.cuda())
    out = sa3.attn_fwd(qz, causal=causal)
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    assert tuple(out.shape) == (B, H, Nq, d)
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    r_q = oracle.quantize_qkv(q, k, v)
    assert_quantized_equal(gpu_canonical(qz, B, H, Nq, Nkv, d), r_q, range(B * H))
    o32 = np.zeros((B, H, Nq, d), np.float32)
    ref = bits_to_f32(oracle.attn_fwd(r_q, Nq, causal, n_kv=Nkv, out32=o32))
    ex = oracle.attn_exact(q, k, v, causal)
    live = np.ones(Nq, bool)
    if causal:
        live = np.arange(Nq) + (Nkv - Nq) >= 0  # rows that see at least one key
        assert not got[:, :, ~live].any() and not ref[:, :, ~live].any()
    blocks = [(h, qb) for h in range(B * H) for qb in range((Nq + 127) // 128)]
    blockwise_rel_l2(got.reshape(B * H, Nq, d), ref.reshape(B * H, Nq, d), blocks, TOL, live=live,
                     label=_ids(case), ref32=o32.reshape(B * H, Nq, d))
    g, r, e = got[:, :, live], ref[:, :, live], ex[:, :, live]
    assert cosine(g, e) >= cosine(r, e) - 1e-3


@pytest.mark.gpu
def test_attn_lens_many_heads_with_single_tile_units():
    """H = 151 heads of 300 queries against 200 keys: the grid has more pair
    units than SMs, so the short last wave runs single-tile units."""
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("split point assumes 148 SMs")
    Nq, Nkv = 300, 200
    q, k, v = _qkv("tiny_b1h2n256d64", Nq, Nkv, {"H": 151})
    B, H, _, d = q.shape
    qz = sa3.quantize_qkv(q.cuda(), k.cuda(), v.cuda())
    r_q = oracle.quantize_qkv(q, k, v)
    torch.cuda.synchronize()
    assert_quantized_equal(gpu_canonical(qz, B, H, Nq, Nkv, d), r_q, range(B * H))
    for causal in (False, True):
        out = sa3.attn_fwd(qz, causal=causal)
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()
        o32 = np.zeros((B, H, Nq, d), np.float32)
        ref = bits_to_f32(oracle.attn_fwd(r_q, Nq, causal, n_kv=Nkv, out32=o32))
        live = np.arange(Nq) + (Nkv - Nq) >= 0 if causal else np.ones(Nq, bool)
        assert not got[:, :, ~live].any()
        blocks = [(h, qb) for h in range(B * H) for qb in range((Nq + 127) // 128)]
        blockwise_rel_l2(got.reshape(B * H, Nq, d), ref.reshape(B * H, Nq, d), blocks, TOL, live=live,
                         label=f"151 heads causal={causal}", ref32=o32.reshape(B * H, Nq, d))


@pytest.mark.gpu
def test_lens_entry_points_reject_mismatched_buffers():
    q, k, v = [t.cuda() for t in _qkv("tiny_b1h2n256d64", 100, 200)]
    with pytest.raises(ValueError):
        sa3.quantize_qkv(q, k, v, out=sa3.empty_quantized(1, 2, 200, 64))
    with pytest.raises(ValueError):
        sa3.quantize_qkv(q, k[:, :, :150].contiguous(), v)
