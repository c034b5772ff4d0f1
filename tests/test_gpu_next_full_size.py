"""GPU parity of the rows beyond the step at the sizes `bench.py --next` times them.

Same bars as the smaller parity tests: integer codes and accumulators bit for bit, scales
to <= 1 ulp (then the oracle's downstream steps are re-run with the GPU's scales), the
optimizer within the derived per-element bound of `test_gpu_optimizer.py`, and the linear
on sampled rows the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_ternary_qat_b200 import synth
from parity_util import f32_of, np_, sample_rows, ulp_diff

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = "cuda:0"
N7, K7 = 11008, 4096           # the 7B-MLP up-projection weight


def test_optimizer_step_7b_weight(bl):
    gen = synth.generator(101)
    W = synth.normal((N7, K7), 0.3, gen).clamp_(-1, 1)
    m = synth.normal((N7, K7), 1e-3, gen)
    v = synth.normal((N7, K7), 1e-3, gen).square_()
    dW = synth.normal((N7, K7), 1e-3, gen)
    Wg, mg, vg = W.to(DEV), m.to(DEV), v.to(DEV)
    step = torch.zeros(1, dtype=torch.int32, device=DEV)
    q = bl.bitlinear_optimizer_step(Wg, dW.to(DEV), mg, vg, step, requantize=True)
    torch.cuda.synchronize()
    Wo, mo, vo, c = oracle.optimizer_step(W, dW, m, v, 1)
    assert c < 1.0                                           # ||dW|| ~ 1e-3 sqrt(45M) ~ 6.7: clipped
    lr, b1, b2, eps, wd = 1e-3, 0.9, 0.95, 1e-6, 0.01
    g = c * dW.numpy().astype(np.float64)
    Tm = b1 * np.abs(m.numpy().astype(np.float64)) + (1 - b1) * np.abs(g)
    Tv = b2 * v.numpy().astype(np.float64) + (1 - b2) * g * g
    den = np.sqrt(vo.astype(np.float64) / (1 - b2)) + eps
    Tw = np.abs(W.numpy().astype(np.float64)) * (1 - lr * wd) + (lr / (1 - b1)) * Tm / den
    rel = 2.0 ** -19
    assert np.all(np.abs(np_(mg).astype(np.float64) - mo) <= rel * Tm)
    assert np.all(np.abs(np_(vg).astype(np.float64) - vo) <= rel * Tv)
    assert np.all(np.abs(np_(Wg).astype(np.float64) - Wo) <= rel * Tw)
    # the next step's codes: exactly the quantiser on the GPU's updated W
    Wn = np_(Wg)
    gam = float(q["gamma"].item())
    assert ulp_diff(np.float32(gam), np.float32(oracle.absmean_gamma(Wn))) <= 1
    wq = oracle.ternary_round(Wn, gam)
    assert np.array_equal(np_(q["wq_i8"]), wq)
    assert np.array_equal(np_(q["packed"]), oracle.pack(wq))


def test_weight_quantiser_variants_7b_weight(bl):
    W = synth.student_t3((N7, K7), 0.02, synth.generator(102)).numpy()
    W = W * np.linspace(0.25, 4.0, N7, dtype=np.float32)[:, None]
    r = bl.bitlinear_quant_weight_rows(torch.from_numpy(W).to(DEV))
    t = bl.bitlinear_quant_weight_tau(torch.from_numpy(W).to(DEV), 0.7)
    torch.cuda.synchronize()
    g_rows = np_(r["gamma_rows"])
    assert ulp_diff(g_rows, oracle.absmean_gamma_rows(W)).max() <= 1
    wq = oracle.ternary_round_rows(W, g_rows)
    assert np.array_equal(np_(r["wq_i8"]), wq)
    assert np.array_equal(np_(r["packed"]), oracle.pack(wq))
    gt = float(t["gamma"].item())
    assert ulp_diff(np.float32(gt), np.float32(oracle.absmean_gamma(W))) <= 1
    wt = oracle.ternary_tau(W, gt, 0.7)
    assert np.array_equal(np_(t["wq_i8"]), wt)
    assert np.array_equal(f32_of(t["wq_bf16"]), wt.astype(np.float32))


def test_per_tensor_activation_scale_7b_activations(bl):
    T, K = 8192, 11008
    X = synth.normal((T, K), 1.0, synth.generator(103))
    X = (X * torch.logspace(-1, 1, T)[:, None]).to(torch.bfloat16)
    o = bl.bitlinear_act_quant_tensor(X.to(DEV))
    torch.cuda.synchronize()
    r_gpu = np_(o["rinv"])
    d = ulp_diff(r_gpu, oracle.rmsnorm_rinv(X, 1e-6))
    assert d.max() <= 1 and np.mean(d > 0) < 0.01
    xq, s, xdq = oracle.act_quant_tensor(X, r_gpu)
    assert np.array_equal(np_(o["sx"]), s)
    assert np.array_equal(np_(o["xq"]), xq)
    assert np.array_equal(np_(o["xdq"]), oracle.round_bf16(xdq))


def test_per_row_linear_7b_shape(bl):
    T = 8192
    rng = np.random.default_rng(104)
    xq = rng.integers(-127, 128, size=(T, K7)).astype(np.int8)
    wq = rng.integers(-1, 2, size=(N7, K7)).astype(np.int8)
    s = rng.uniform(10, 200, size=T).astype(np.float32)
    gam = rng.uniform(1e-3, 5e-2, size=N7).astype(np.float32)
    y, acc = bl.bitlinear_linear_rows(torch.from_numpy(xq).to(DEV), torch.from_numpy(s).to(DEV),
                                      torch.from_numpy(wq).to(DEV), torch.from_numpy(gam).to(DEV), want_acc=True)
    torch.cuda.synchronize()
    rows = sample_rows(T, 10, seed=104)
    acc_o = oracle.int_gemm(xq, wq, rows=rows)
    assert np.array_equal(np_(acc)[rows], acc_o)
    assert np.array_equal(np_(y)[rows], oracle.round_bf16(oracle.linear_epilogue_rows(acc_o, gam, s[rows])))
