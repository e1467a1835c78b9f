"""The parity tests' bf16 tie rule (sa3_testutil._forgive_ties), pinned on
hand-built values: only a one-ulp difference whose fp32 reference sits on
the bf16 rounding midpoint is forgiven; larger or off-midpoint differences
and sign changes still count."""
import numpy as np
import torch

from sa3_testutil import _forgive_ties, blockwise_rel_l2


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def test_only_midpoint_one_ulp_differences_are_forgiven():
    u = 2.0 ** -7                                        # bf16 ulp in [1, 2)
    r32 = np.array([1 + u / 2,                           # exact tie: rounds to 1 (even)
                    1 + u / 2 + 2.0 ** -17,              # within 2^-16 of the midpoint: rounds to 1 + u
                    1 + u / 2 + 2.0 ** -10,              # far from it (rounds to 1 + u)
                    1 + u / 2,                           # tie, but got is two ulps away
                    -(1 + u / 2),                        # tie on the negative side
                    1 + u / 2], np.float32)
    ref = _bf16(r32)
    got = np.array([1 + u, 1.0, 1.0, 1 + 2 * u, -(1 + u), -1.0], np.float32)
    adj, n = _forgive_ties(got, ref, r32)
    assert n == 3
    assert adj[0] == ref[0] and adj[1] == ref[1] and adj[4] == ref[4]
    assert adj[2] == got[2] and adj[3] == got[3] and adj[5] == got[5]


def test_blockwise_check_sees_a_wrong_row_despite_ties():
    rng = np.random.default_rng(0)
    ref32 = rng.standard_normal((1, 256, 64)).astype(np.float32)
    ref = _bf16(ref32)
    got = ref.copy()
    got[0, 200, :] *= 1.05                               # one wrong row in block 1
    blockwise_rel_l2(got, ref, [(0, 0)], 1e-12, ref32=ref32)
    try:
        blockwise_rel_l2(got, ref, [(0, 0), (0, 1)], 2e-3, ref32=ref32)
    except AssertionError:
        return
    raise AssertionError("a wrong row was not caught")
