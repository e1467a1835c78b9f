"""sa3_quantize_qkv_noalloc through the C ABI.

This entry point is for callers that cannot give the library device memory
at call time (for example a plug-in layer whose host framework owns every
device allocation, or a latency-critical path that must not call
cudaMalloc).  It keeps its scratch in a fixed device array inside the
library.  Two calls in a row must each give exactly what the workspace
entry point gives for the same inputs -- the second call also shows that
whatever the first call left in the shared scratch does not leak into the
result.  The file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import sa3_inputs

sa3 = pytest.importorskip("bit_quantized_attention_sa3_b200")

FIELDS = ("q_fp4", "q_sf", "k_fp4", "k_sf", "vt_fp4", "vt_sf", "k_mean")
SCRATCH_BYTES = 4 << 20  # SA3_NOALLOC_SCRATCH_BYTES in include/sa3.h


def _noalloc_fn():
    f = sa3.lib().sa3_quantize_qkv_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    f.restype = I
    f.argtypes = [P, P, P, I, I, I, I, ctypes.POINTER(sa3._QKV), P]
    return f


def _call_noalloc(q, k, v):
    B, H, N, d = q.shape
    out = sa3.empty_quantized(B, H, N, d, q.device)
    st = out.struct()
    rc = _noalloc_fn()(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, N, d, ctypes.byref(st),
                       torch.cuda.current_stream().cuda_stream)
    return rc, out


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    cases = [("noncausal_b2h16n4096d128", {"B": 1, "H": 3, "N": 1100}, 11),
             ("tiny_b1h2n256d64", {"N": 700, "H": 3}, 12)]
    for name, over, seed in cases:
        q, k, v = [t.cuda() for t in sa3_inputs.make_qkv(name, seed=seed, shape_override=over)]
        ref = sa3.quantize_qkv(q, k, v)
        rc, got = _call_noalloc(q, k, v)
        assert rc == sa3.SA3_OK
        torch.cuda.synchronize()
        assert sa3.device_status() == sa3.SA3_OK
        for f in FIELDS:
            assert torch.equal(getattr(got, f), getattr(ref, f)), (name, f)


@pytest.mark.gpu
def test_noalloc_rejects_shapes_beyond_its_scratch():
    B, H, N, d = 64, 64, 4096, 128  # needs 64*64*8*128*8 = 32 MiB of scratch
    assert sa3.quant_workspace_bytes(B, H, N, d) > SCRATCH_BYTES
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = dummy.data_ptr()
    st = sa3._QKV(p, p, p, p, p, p, p)
    rc = _noalloc_fn()(p, p, p, B, H, N, d, ctypes.byref(st), torch.cuda.current_stream().cuda_stream)
    assert rc == sa3.SA3_ERR_UNSUPPORTED
