"""The tensor-pipe peak probe that gives the int8 GEMM roofline its denominator: every
launch completes with a clean device status, and the measured rates have the shape the
hardware implies (kind::i8 moves twice the multiply-adds of kind::f16 per instruction
slot, so its rate is well above the bf16 one)."""
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
