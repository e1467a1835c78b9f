"""Failure detection without a GPU fault: a device wait that can never be
satisfied must give up after its limit, report SA3_ERR_TIMEOUT through
sa3_device_status, and leave the CUDA context usable."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import sa3_inputs
from sa3_testutil import assert_quantized_equal, bits_to_f32, gpu_canonical, rel_l2

sa3 = pytest.importorskip("bit_quantized_attention_sa3_b200")


@pytest.mark.gpu
def test_bounded_wait_reports_timeout_and_context_survives():
    f = sa3.lib().sa3_selftest_wait_timeout
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_uint, ctypes.c_void_p]
    assert sa3.device_status() == sa3.SA3_OK
    stream = torch.cuda.current_stream().cuda_stream
    assert f(20000, stream) == sa3.SA3_OK          # 20 ms limit
    assert sa3.device_status() == sa3.SA3_ERR_TIMEOUT
    assert sa3.device_status() == sa3.SA3_OK       # cleared by the read
    # the context still works: a normal call matches the oracle
    q, k, v = sa3_inputs.make_qkv("tiny_b1h2n256d64")
    qz = sa3.quantize_qkv(q.cuda(), k.cuda(), v.cuda())
    out = sa3.attn_fwd(qz, causal=True)
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    B, H, N, d = q.shape
    r = oracle.quantize_qkv(q, k, v)
    assert_quantized_equal(gpu_canonical(qz, B, H, N, N, d), r, range(B * H))
    ref = bits_to_f32(oracle.attn_fwd(r, N, True))
    assert rel_l2(out.float().cpu().numpy(), ref) <= 2e-3
