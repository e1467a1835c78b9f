"""sa3_probe_fp4_mma, the block-scaled FP4 tensor-core rate probe that gives
the attention roofline its measured denominator: its accumulators must hold
exactly 64 * iters (all codes and scales 1.0, K = 64 per MMA), so the timed
launch really ran every MMA."""
import pytest
import torch

sa3 = pytest.importorskip("bit_quantized_attention_sa3_b200")


@pytest.mark.gpu
@pytest.mark.parametrize("n", [128, 256])
def test_probe_accumulates_every_mma(n):
    for iters in (1, 37, 4096):
        out = sa3.probe_fp4_mma(n=n, iters=iters)
        torch.cuda.synchronize()
        assert sa3.device_status() == sa3.SA3_OK
        assert torch.all(out == 64.0 * iters), (n, iters, out.min().item(), out.max().item())


@pytest.mark.gpu
def test_probe_rate_is_plausible():
    """Timed like the bench: one CTA per SM, CUDA events.  The rate must be
    positive and below twice NVIDIA's dense FP4 figure (9000 TOPS)."""
    sa3.probe_fp4_mma(n=128, iters=256)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    out = sa3.probe_fp4_mma(n=128, iters=16384)
    e1.record()
    torch.cuda.synchronize()
    assert torch.all(out == 64.0 * 16384)
    ctas = torch.cuda.get_device_properties(0).multi_processor_count
    tops = 2 * 128 * 128 * 64 * 16384 * ctas / (e0.elapsed_time(e1) * 1e-3) / 1e12
    print(f"block-scaled FP4 MMA, M=128 N=128 K=64: {tops:.0f} TOPS")
    assert 0 < tops < 18000
