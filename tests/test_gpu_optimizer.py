"""GPU parity of the fused optimizer step (clip -> AdamW -> clamp -> next step's codes).

The oracle runs the step in fp64 from the same fp32 state; the kernel runs it in fp32 with
one rounding per operation (about ten per element), so each output may differ from the
oracle by at most a few 2^-24 relative roundings of the terms that form it.  The test
bound is 2^-19 times the magnitude of those terms:
  m:  b1 |m| + (1 - b1) |g|                          (g = c dW, c the clip coefficient)
  v:  b2 v + (1 - b2) g^2                            (no cancellation: both terms >= 0)
  W:  |W| (1 - lr wd) + (lr / bc1) T_m / (sqrt(v' / bc2) + eps)
The codes of the next step are integer decisions: they are compared exactly with the
oracle's quantiser applied to the GPU's updated W (and the gamma must equal what the
quantiser computes from that W on its own, bit for bit).
"""
import numpy as np
import pytest
import torch

import oracle
from bit_ternary_qat_b200 import _lib, synth
from parity_util import f32_of, np_

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
HP = dict(lr=1e-3, betas=(0.9, 0.95), eps=1e-6, weight_decay=0.01)
HP_LOUD = dict(lr=5e-2, betas=(0.8, 0.9), eps=1e-3, weight_decay=0.3)
REL = 2.0 ** -19


def _bounds(W, dW, m, v, c, m_new, v_new, t, hp):
    lr, (b1, b2), eps, wd = hp["lr"], hp["betas"], hp["eps"], hp["weight_decay"]
    g = c * dW.astype(np.float64)
    Tm = b1 * np.abs(m.astype(np.float64)) + (1 - b1) * np.abs(g)
    Tv = b2 * v.astype(np.float64) + (1 - b2) * g * g
    bc1, bc2 = 1 - b1 ** t, 1 - b2 ** t
    den = np.sqrt(v_new.astype(np.float64) / bc2) + eps
    Tw = np.abs(W.astype(np.float64)) * (1 - lr * wd) + (lr / bc1) * Tm / den
    return REL * Tm, REL * Tv, REL * Tw


def _state(N, K, seed):
    gen = synth.generator(seed)
    W = synth.normal((N, K), 0.3, gen).clamp_(-1, 1)
    m = synth.normal((N, K), 1e-3, gen)
    v = synth.normal((N, K), 1e-3, gen).square_()
    return W, m, v


@pytest.mark.parametrize("N,K", [(16, 32), (48, 160), (512, 256), (2048, 2048), (272, 4096)])
@pytest.mark.parametrize("max_norm,hp", [(1.0, HP), (0.0, HP), (1.0, HP_LOUD)])
def test_optimizer_step_parity(bl, N, K, max_norm, hp):
    W, m, v = _state(N, K, seed=N + K)
    Wg, mg, vg = W.to(DEV), m.to(DEV), v.to(DEV)
    step = torch.zeros(1, dtype=torch.int32, device=DEV)
    gen = synth.generator(N * K)
    for t in range(1, 4):
        dW = synth.normal((N, K), 0.01 * t, gen)            # ||dW|| well above 1 for the larger shapes
        W0, m0, v0 = np_(Wg).copy(), np_(mg).copy(), np_(vg).copy()
        bl.bitlinear_optimizer_step(Wg, dW.to(DEV), mg, vg, step, max_norm=max_norm, **hp)
        torch.cuda.synchronize()
        assert int(step.item()) == t
        Wo, mo, vo, c = oracle.optimizer_step(W0, dW, m0, v0, t, max_norm=max_norm, **hp)
        bm, bv, bw = _bounds(W0, dW.numpy(), m0, v0, c, mo, vo, t, hp)
        assert np.all(np.abs(np_(mg).astype(np.float64) - mo) <= bm)
        assert np.all(np.abs(np_(vg).astype(np.float64) - vo) <= bv)
        assert np.all(np.abs(np_(Wg).astype(np.float64) - Wo) <= bw)
        assert np_(Wg).max() <= 1.0 and np_(Wg).min() >= -1.0
        if max_norm > 0 and N * K >= 512 * 256:
            assert c < 1.0                                   # the clip was active


@pytest.mark.parametrize("N,K", [(48, 160), (2048, 2048)])
def test_optimizer_step_requantizes(bl, N, K):
    W, m, v = _state(N, K, seed=7)
    Wg, mg, vg = W.to(DEV), m.to(DEV), v.to(DEV)
    step = torch.zeros(1, dtype=torch.int32, device=DEV)
    dW = synth.normal((N, K), 0.05, synth.generator(8)).to(DEV)
    q = bl.bitlinear_optimizer_step(Wg, dW, mg, vg, step, requantize=True, **HP)
    torch.cuda.synchronize()
    ref = bl.bitlinear_quant_weight(Wg.clone())           # the quantiser on its own, same W
    torch.cuda.synchronize()
    assert float(q["gamma"].item()) == float(ref["gamma"].item())
    for k in ("wq_i8", "wq_bf16", "packed"):
        assert torch.equal(q[k], ref[k])
    Wn = np_(Wg)
    g = float(q["gamma"].item())
    assert g == np.float32(oracle.absmean_gamma(Wn))
    wq = oracle.ternary_round(Wn, g)
    assert np.array_equal(np_(q["wq_i8"]), wq)
    assert np.array_equal(f32_of(q["wq_bf16"]), wq.astype(np.float32))
    assert np.array_equal(np_(q["packed"]), oracle.pack(wq))


def test_optimizer_step_in_cuda_graph(bl):
    """The step index lives on the device, so a captured step replays as steps 1, 2, 3."""
    N, K = 64, 128
    W, m, v = _state(N, K, seed=9)
    Wg, mg, vg = W.to(DEV), m.to(DEV), v.to(DEV)
    dW = synth.normal((N, K), 0.02, synth.generator(10)).to(DEV)
    step = torch.zeros(1, dtype=torch.int32, device=DEV)
    ws = bl.workspace(1, N, K, DEV)
    Wc, mc, vc = Wg.clone(), mg.clone(), vg.clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            bl.bitlinear_optimizer_step(Wc, dW, mc, vc, step, ws=ws, **HP)
    torch.cuda.current_stream().wait_stream(s)
    # capture does not execute: reset the state the capture left untouched, then replay
    step.zero_()
    Wc.copy_(Wg); mc.copy_(mg); vc.copy_(vg)
    W0, m0, v0 = np_(Wg), np_(mg), np_(vg)
    for t in range(1, 4):
        g.replay()
        torch.cuda.synchronize()
        assert int(step.item()) == t
        W0, m0, v0, c = oracle.optimizer_step(W0, np_(dW), m0, v0, t, **HP)
    assert np.max(np.abs(np_(Wc) - W0)) <= 1e-5 * max(1.0, np.max(np.abs(W0)))
    del g


def test_optimizer_step_rejects_bad_arguments(bl):
    N, K = 16, 32
    t = [torch.zeros(N, K, device=DEV) for _ in range(4)]
    step = torch.zeros(1, dtype=torch.int32, device=DEV)
    ws = bl.workspace(1, N, K, DEV)
    codes = torch.empty(N, K, dtype=torch.int8, device=DEV)

    def st(lr=1e-3, b1=0.9, b2=0.95, eps=1e-6, wd=0.01, mn=1.0, wq=None, gamma=None):
        return _lib.status("bitlinear_optimizer_step", *(x.data_ptr() for x in t), N, K, lr, b1, b2, eps, wd, mn,
                           step.data_ptr(), wq, None, None, gamma, ws.data_ptr(), ws.numel(), None)

    assert st() == 0
    for kw in (dict(lr=-1.0), dict(lr=float("nan")), dict(b1=1.0), dict(b2=-0.1), dict(eps=0.0),
               dict(wd=float("inf")), dict(mn=float("nan")), dict(wq=codes.data_ptr())):
        assert st(**kw) == 1, kw                             # BL_ERR_INVALID_ARG
    assert _lib.status("bitlinear_optimizer_step", *(x.data_ptr() for x in t), N, K, 1e-3, 0.9, 0.95, 1e-6, 0.01,
                       1.0, step.data_ptr(), None, None, None, None, ws.data_ptr(), 64, None) == 4   # workspace
    torch.cuda.synchronize()
