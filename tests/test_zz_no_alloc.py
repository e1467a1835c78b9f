"""sa3_quantize_qkv_noalloc through the C ABI.

This entry point is for callers that cannot give the library device memory
at call time (for example a plug-in layer whose host framework owns every
device allocation, or a latency-critical path that must not call
cudaMalloc).  It keeps its scratch in a fixed device array inside the
library, shared by every call.  The checks here: the same inputs quantized
twice in a row, with a call on other, large-valued inputs of the same shape
in between (so the shared scratch holds different sums each time), give
exactly what the workspace entry point gives; a shape whose scratch fills
the array exactly (16 K-mean chunks) works, and the first shape past it is
rejected.  The file is named so that pytest collects it last.
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


def _device_qkv(B, H, N, d, seed, scale=1.0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    shape = (B, H, N, d)
    q, k, v = (torch.randn(shape, generator=g, device="cuda") * scale for _ in range(3))
    k = k + torch.randn((B, H, 1, d), generator=g, device="cuda") * 2.0 * scale  # a K offset to smooth away
    return q.bfloat16(), k.bfloat16(), v.bfloat16()


def _assert_same(got, ref, what):
    for f in FIELDS:
        assert torch.equal(getattr(got, f), getattr(ref, f)), (what, f)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    cases = [("noncausal_b2h16n4096d128", {"B": 1, "H": 3, "N": 1100}, 11),
             ("tiny_b1h2n256d64", {"N": 700, "H": 3}, 12)]
    for name, over, seed in cases:
        q, k, v = [t.cuda() for t in sa3_inputs.make_qkv(name, seed=seed, shape_override=over)]
        B, H, N, d = q.shape
        ref = sa3.quantize_qkv(q, k, v)
        rc, first = _call_noalloc(q, k, v)
        assert rc == sa3.SA3_OK
        # other inputs of the same shape, values ~1000x larger: the shared
        # scratch now holds their K-mean partial sums
        qo, ko, vo = _device_qkv(B, H, N, d, seed + 100, scale=1000.0)
        rc, other = _call_noalloc(qo, ko, vo)
        assert rc == sa3.SA3_OK
        rc, second = _call_noalloc(q, k, v)
        assert rc == sa3.SA3_OK
        torch.cuda.synchronize()
        assert sa3.device_status() == sa3.SA3_OK
        _assert_same(first, ref, (name, "first call"))
        _assert_same(second, ref, (name, "second call"))
        _assert_same(other, sa3.quantize_qkv(qo, ko, vo), (name, "large-valued call"))


@pytest.mark.gpu
def test_noalloc_at_the_scratch_limit():
    """B*H = 256 heads of N = 8192 tokens, d = 128: 16 chunks of 512 tokens,
    256 * 16 * 128 fp64 sums = exactly the 4 MiB array."""
    B, H, N, d = 1, 256, 8192, 128
    assert sa3.quant_workspace_bytes(B, H, N, d) == SCRATCH_BYTES
    q, k, v = _device_qkv(B, H, N, d, seed=5)
    ref = sa3.quantize_qkv(q, k, v)
    for _ in range(2):
        rc, got = _call_noalloc(q, k, v)
        assert rc == sa3.SA3_OK
        torch.cuda.synchronize()
        assert sa3.device_status() == sa3.SA3_OK
        _assert_same(got, ref, "4 MiB of scratch")


@pytest.mark.gpu
def test_noalloc_rejects_shapes_beyond_its_scratch():
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = dummy.data_ptr()
    st = sa3._QKV(p, p, p, p, p, p, p)
    # one head past the limit, and a shape far beyond it
    for B, H, N, d in ((1, 257, 8192, 128), (64, 64, 4096, 128)):
        assert sa3.quant_workspace_bytes(B, H, N, d) > SCRATCH_BYTES
        rc = _noalloc_fn()(p, p, p, B, H, N, d, ctypes.byref(st), torch.cuda.current_stream().cuda_stream)
        assert rc == sa3.SA3_ERR_UNSUPPORTED
