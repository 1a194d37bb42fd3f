"""rfq_mma_rate_probe, the tensor-core rate measurement behind the GEMM's roofline
denominator: it runs on every SM pair (or SM), reports the flops it executed and
a clock64 span per cluster, and its rate per SM clock is within the bounds the
instruction shapes allow (never above the dense rate of kind::mxf4, 32768 flop
per SM per clock, by more than timer noise; kind::mxf8f6f4 half of that)."""
import pytest

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("variant,pair,mma_k,max_per_clock", [(0, 2, 64, 32768), (1, 1, 64, 32768),
                                                              (2, 2, 32, 16384)])
def test_probe_reports_its_work(rfq, variant, pair, mma_k, max_per_clock):
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    cycles = torch.zeros(sms, dtype=torch.int64, device="cuda")
    iters = 2000
    flops, used = rfq.mma_rate_probe(variant, iters, cycles)
    torch.cuda.synchronize()
    rfq.check_device_error()
    assert used % pair == 0 and sms // 2 <= used <= sms
    clusters = used // pair
    assert flops == clusters * iters * 8 * 2 * (128 * pair) * 256 * mma_k
    spans = cycles[:clusters].cpu()
    assert bool((spans > 0).all())
    assert int(cycles[clusters:].count_nonzero()) == 0          # words past the launched clusters untouched
    per_clock = flops / used / float(spans.max())
    assert 0.25 * max_per_clock < per_clock <= 1.02 * max_per_clock


def test_probe_rejects_bad_arguments(rfq):
    import torch
    cycles = torch.zeros(4, dtype=torch.int64, device="cuda")   # fewer words than clusters
    with pytest.raises(rfq.RFQError):
        rfq.mma_rate_probe(0, 10, cycles)
    big = torch.zeros(1024, dtype=torch.int64, device="cuda")
    with pytest.raises(rfq.RFQError):
        rfq.mma_rate_probe(0, rfq.MMA_PROBE_MAX_ITERATIONS + 1, big)
