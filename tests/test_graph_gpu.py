"""The quantizer and attention calls recorded into a CUDA graph and replayed.

The calls only enqueue kernels on the given stream: no allocation, no host
synchronization, and after a first call on a device no attribute call
either.  So a serving loop can record quantize + attention once and replay
it for new inputs written into the same buffers.  Replays must give the
same bits as the direct calls, for the FP4 path and for the 8-bit training
forward (output and log-sum-exp)."""
import pytest
import torch

import sa3_inputs

sa3 = pytest.importorskip("bit_quantized_attention_sa3_b200")


def _inputs(seed):
    q, k, v = sa3_inputs.make_qkv("noncausal_b2h16n4096d128", seed=seed, shape_override={"B": 1, "H": 3, "N": 700})
    return q.cuda(), k.cuda(), v.cuda()


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True], ids=["noncausal", "causal"])
def test_fp4_step_replays_in_a_cuda_graph(causal):
    q, k, v = _inputs(0)
    B, H, N, d = q.shape
    qz = sa3.empty_quantized(B, H, N, d)
    ws = torch.empty(sa3.quant_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)

    def step():
        sa3.quantize_qkv(q, k, v, out=qz, workspace=ws)
        sa3.attn_fwd(qz, causal=causal, out=out)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()  # first call on this device: sets the kernels' attributes
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    direct = out.clone()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    assert torch.equal(out, direct)

    # new inputs written into the recorded buffers
    q2, k2, v2 = _inputs(1)
    q.copy_(q2), k.copy_(k2), v.copy_(v2)
    g.replay()
    torch.cuda.synchronize()
    want = sa3.attn_fwd(sa3.quantize_qkv(q2, k2, v2), causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(out, want)
    assert not torch.equal(out, direct)


@pytest.mark.gpu
def test_i8_training_forward_replays_in_a_cuda_graph():
    q, k, v = _inputs(2)
    B, H, N, d = q.shape
    qz = sa3.empty_quantized_i8(B, H, N, d)
    ws = torch.empty(sa3.quant_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")

    def step():
        sa3.quantize_qkv_i8(q, k, v, out=qz, workspace=ws)
        sa3.attn_fwd_i8(qz, causal=True, out=out, lse=lse)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    direct, direct_lse = out.clone(), lse.clone()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    out.zero_(), lse.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert sa3.device_status() == sa3.SA3_OK
    assert torch.equal(out, direct) and torch.equal(lse, direct_lse)
