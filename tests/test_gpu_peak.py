"""The measurement probes.  The tensor-pipe peak probe that gives the int8 GEMM roofline its
denominator: every launch completes with a clean device status, and the measured rates have
the shape the hardware implies (kind::i8 moves twice the multiply-adds of kind::f16 per
instruction slot, so its rate is well above the bf16 one).  The read probe that gives the
decode GEMV its read-only ceiling."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def _rate(bl, kind, pair, iters):
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    ops = bl.mma_peak_probe(kind, pair, iters)
    b.record()
    torch.cuda.synchronize()
    return ops / (a.elapsed_time(b) * 1e-3) / 1e12


@pytest.mark.parametrize("pair", [False, True])
def test_mma_peak_probe_rates(bl, pair):
    for kind in ("int8", "bf16"):
        bl.mma_peak_probe(kind, pair, 256)
    torch.cuda.synchronize()
    assert bl.check_device_status() == 0
    r8 = max(_rate(bl, "int8", pair, 4000) for _ in range(3))
    r16 = max(_rate(bl, "bf16", pair, 4000) for _ in range(3))
    assert bl.check_device_status() == 0
    assert r16 > 200.0, r16                       # TFLOP/s: far above any CUDA-core rate
    assert r8 > 1.3 * r16, (r8, r16)
    # ops count: per CTA (pair) 4 instructions per iteration of M x N x 32 bytes of K
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    ops = bl.mma_peak_probe("int8", pair, 10)
    torch.cuda.synchronize()
    per = 2.0 * (256 * 256 if pair else 128 * 256) * 32 * 4 * 10
    units = ops / per
    assert units == int(units) and 1 <= units <= (sms // 2 if pair else sms)


@pytest.mark.parametrize("pattern", ["gemv", "coalesced"])
def test_read_peak_probe(bl, pattern):
    """The read probe reads a weight-shaped buffer with a clean device status and leaves the
    sink alone (the XOR of its loads never equals the probe's constant on these bytes); on a
    buffer larger than L2 it reads at HBM rates (well above 1 TB/s)."""
    small = torch.ones(48, 320, dtype=torch.uint8, device="cuda:0")
    sink = torch.zeros(4, dtype=torch.int32, device="cuda:0")
    assert bl.read_peak_probe(small, pattern, sink) == 48 * 320
    torch.cuda.synchronize()
    assert bl.check_device_status() == 0
    assert int(sink.abs().sum()) == 0
    big = torch.ones(28672, 8192, dtype=torch.uint8, device="cuda:0")     # 235 MB
    for _ in range(3):
        bl.read_peak_probe(big, pattern, sink)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    n = bl.read_peak_probe(big, pattern, sink)
    b.record()
    torch.cuda.synchronize()
    assert bl.check_device_status() == 0
    assert n / (a.elapsed_time(b) * 1e-3) > 1e12
