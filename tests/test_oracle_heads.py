"""Pin of the oracle's batch and head indexing: every (b, h) is an
independent problem (the method smooths K per head and attends per head),
so the oracle run on a [B, H] stack must give, slice for slice, bit for bit,
what it gives on each (b, h) alone.  A wrong batch or head stride, or a mean
taken over the wrong axis, fails here.  Distinct offsets per head make the
K and V means differ from head to head."""
import numpy as np
import pytest
import torch

import oracle

B, H, D = 2, 3, 64


def _inputs(Nq, Nkv, seed=11):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, Nq, D, generator=g)
    k = torch.randn(B, H, Nkv, D, generator=g) + 3.0 * torch.randn(B, H, 1, D, generator=g)
    v = torch.randn(B, H, Nkv, D, generator=g) + 2.0 * torch.randn(B, H, 1, D, generator=g)
    return q.bfloat16(), k.bfloat16(), v.bfloat16()


def _slice(t, b, h):
    return t[b:b + 1, h:h + 1].contiguous()


@pytest.mark.parametrize("Nq,Nkv", [(200, 200), (77, 300)])
@pytest.mark.parametrize("causal", [False, True])
def test_fp4_heads_are_independent(Nq, Nkv, causal):
    q, k, v = _inputs(Nq, Nkv)
    full = oracle.quantize_qkv(q, k, v, smooth_v=True)
    out = oracle.attn_fwd(full, Nq, causal, n_kv=Nkv)
    for b in range(B):
        for h in range(H):
            one = oracle.quantize_qkv(_slice(q, b, h), _slice(k, b, h), _slice(v, b, h), smooth_v=True)
            for name in ("q_codes", "q_sf", "k_codes", "k_sf", "vt_codes", "vt_sf", "k_mean", "v_mean"):
                assert np.array_equal(full[name][b, h], one[name][0, 0]), (name, b, h)
            assert np.array_equal(out[b, h], oracle.attn_fwd(one, Nq, causal, n_kv=Nkv)[0, 0]), (b, h)
    # the heads really differ (the check above is not vacuous)
    assert not np.array_equal(full["k_mean"][0, 0], full["k_mean"][1, 2])
    assert not np.array_equal(out[0, 0], out[1, 2])


@pytest.mark.parametrize("causal", [False, True])
def test_i8_heads_are_independent(causal):
    Nq = Nkv = 200
    q, k, v = _inputs(Nq, Nkv, seed=12)
    full = oracle.quantize_qkv_i8(q, k, v)
    out, lse = oracle.attn_fwd_i8(full, Nq, causal, return_lse=True)
    for b in range(B):
        for h in range(H):
            one = oracle.quantize_qkv_i8(_slice(q, b, h), _slice(k, b, h), _slice(v, b, h))
            for name in ("q_i8", "q_scale", "k_i8", "k_scale", "vt_f16", "k_mean"):
                assert np.array_equal(full[name][b, h], one[name][0, 0]), (name, b, h)
            o1, l1 = oracle.attn_fwd_i8(one, Nq, causal, return_lse=True)
            assert np.array_equal(out[b, h], o1[0, 0]) and np.array_equal(lse[b, h], l1[0, 0]), (b, h)
