"""GPU: the tensor-pipe peak probe (the FP4 roofline the GEMMs are compared
with) completes, reports 2 M N K flops per MMA for every CTA pair, and runs
at a rate between the slowest plausible clock and the dense FP4 datasheet
figure with margin (its operands never leave shared memory)."""
import pytest
import torch

from fp4_precision_numerics_b200 import mxfp4

pytestmark = pytest.mark.gpu


def test_mma_peak_probe_rate_and_flops():
    stream = torch.cuda.current_stream()
    flops = mxfp4.mxfp4_mma_peak_probe(64, stream)
    torch.cuda.synchronize()
    per_pair = 64 * 2.0 * 256 * 192 * 64
    pairs = flops / per_pair
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert pairs == int(pairs) and 1 <= pairs <= sms // 2
    rates = []
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fl = mxfp4.mxfp4_mma_peak_probe(8192, stream)
        e1.record(stream)
        e1.synchronize()
        rates.append(fl / (e0.elapsed_time(e1) / 1e3) / 1e12)
    mxfp4.mxfp4_check_device_status(stream)
    best = max(rates)
    assert 1000.0 < best < 12000.0, rates
