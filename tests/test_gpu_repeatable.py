"""Run-to-run repeatability of the persistent, multi-role kernels.

Every sum in these kernels has a fixed order (int32 accumulation is exact; the bf16 GEMMs
accumulate in TMEM in k order; K-split partial sums are added in split order), so repeated
calls on the same inputs must give the same bits.  A missed or mis-ordered barrier between the
roles of a persistent kernel (producer, MMA issuer, decoders, epilogue) shows up as an
occasional difference, so each shape is called many times back to back and every output is
compared with the first.  The shapes give CTA pairs several work units, short last units,
K splits with one-k-block stages, and the GEMMs' split last wave.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
REPS = 24


@pytest.mark.parametrize("T,K,N", [(64, 4096, 4096), (256, 512, 20480), (40, 256, 40000), (20, 5440, 512),
                                   (200, 1024, 40000), (12, 8192, 28672)])
def test_linear_packed_repeatable(bl, T, K, N):
    rng = np.random.default_rng(T + K + N)
    xq = torch.from_numpy(rng.integers(-128, 128, size=(T, K)).astype(np.int8)).to(DEV)
    packed = torch.from_numpy(oracle.pack(rng.integers(-1, 2, size=(N, K)).astype(np.int8))).to(DEV)
    s = torch.from_numpy(rng.uniform(5, 300, size=T).astype(np.float32)).to(DEV)
    g = torch.tensor([0.0173], device=DEV)
    ws = torch.empty(8 * T * N * 4, dtype=torch.uint8, device=DEV)
    outs = [bl.bitlinear_linear_packed(xq, s, packed, g, K, want_acc=True, ws=ws) for _ in range(REPS)]
    torch.cuda.synchronize()
    assert bl.check_device_status() == 0
    y0, a0 = outs[0]
    for y, a in outs[1:]:
        assert torch.equal(a, a0)
        assert torch.equal(y.view(torch.int16), y0.view(torch.int16))


@pytest.mark.parametrize("T,K,N", [(3800, 1280, 3840), (4096, 2048, 11008), (16384, 512, 4096)])
def test_gemms_repeatable(bl, T, K, N):
    gen = torch.Generator(device=DEV).manual_seed(T + N)
    xq = torch.randint(-127, 128, (T, K), dtype=torch.int8, device=DEV, generator=gen)
    wq = torch.randint(-1, 2, (N, K), dtype=torch.int8, device=DEV, generator=gen)
    s = torch.rand(T, device=DEV, generator=gen) * 190 + 10
    g = torch.tensor([0.0173], device=DEV)
    dY = (torch.randn(T, N, device=DEV, generator=gen) * 1e-2).to(torch.bfloat16)
    xdq = torch.randn(T, K, device=DEV, generator=gen).to(torch.bfloat16)
    wb = wq.to(torch.bfloat16)
    first = None
    for _ in range(REPS // 3):
        y, acc = bl.bitlinear_linear(xq, s, wq, g, want_acc=True)
        dxh = bl.bitlinear_grad_input(dY, wb, g)
        dw = bl.bitlinear_backward_weight(dY, xdq)
        cur = (acc, y.view(torch.int16), dxh.view(torch.int32), dw.view(torch.int32))
        if first is None:
            first = cur
        else:
            for c, f in zip(cur, first):
                assert torch.equal(c, f)
    torch.cuda.synchronize()
    assert bl.check_device_status() == 0
