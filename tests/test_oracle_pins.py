"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test ties one oracle function to a closed form, a value the pages print (the
2-bit code table), a hand-derived example, a library routine (torch's RMSNorm,
bf16 cast, autograd; numpy integer matmul) or a brute-force restatement from a
different page (the scalar +-0.5 step).  A plausible slip in the oracle -- a dropped
scale, a wrong sign, a transposed operand, round-half-away instead of half-even,
per-row instead of per-tensor scale -- fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from bit_ternary_qat_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------------------------
# packing: the code table printed on the pages
# ------------------------------------------------------------------------------------

def test_pack_golden_bytes(ora):
    gd = _load("pack_codes.json")
    wq = np.array(gd["rows"], dtype=np.int8)
    packed = ora.pack(wq)
    assert packed.tolist() == gd["packed"]
    assert np.array_equal(ora.unpack(packed, gd["K"]), wq)


def test_pack_reserved_code_decodes_to_zero(ora):
    gd = _load("pack_codes.json")
    packed = np.full((1, 8), 0xFF, dtype=np.uint8)
    assert np.all(ora.unpack(packed, 32) == 0)
    assert gd["reserved_byte_0xFF_decodes_to"] == [0, 0, 0, 0]


def test_pack_roundtrip_and_no_reserved_code(ora):
    rng = np.random.default_rng(7)
    wq = rng.integers(-1, 2, size=(37, 96)).astype(np.int8)
    packed = ora.pack(wq)
    assert packed.shape == (37, 24)
    assert np.array_equal(ora.unpack(packed, 96), wq)
    # every 2-bit field is 00, 01 or 10 (the reserved 11 is never emitted)
    fields = np.stack([(packed >> (2 * j)) & 3 for j in range(4)])
    assert not np.any(fields == 3)
    # independent numpy decode: value = (c & 1) - (c >> 1) for the three used codes
    dec = np.stack([(f & 1).astype(np.int8) - (f >> 1).astype(np.int8) for f in fields], axis=-1)
    assert np.array_equal(dec.reshape(37, 96), wq)


# ------------------------------------------------------------------------------------
# weight quantiser
# ------------------------------------------------------------------------------------

def test_worked_example_end_to_end(ora):
    ex = _load("worked_example.json")
    W = np.array(ex["W"], dtype=np.float32)
    x = np.array(ex["x"], dtype=np.float32)
    gamma = ora.absmean_gamma(W)
    assert gamma == ex["gamma"]
    wq = ora.ternary_round(W, gamma)
    assert wq.tolist() == ex["Wq"]
    xq, s, xdq = ora.act_quant(x)            # no RMSNorm
    assert s.tolist() == ex["s"]
    assert xq.tolist() == ex["xq"]
    assert xdq.tolist() == ex["xdq"]
    acc = ora.int_gemm(xq, wq)
    assert acc.tolist() == ex["acc"]
    y = ora.linear_epilogue(acc, gamma, s)
    assert y.tolist() == ex["y"]


def test_gamma_closed_forms(ora):
    # constant magnitude c -> gamma = c, codes = sign
    c = np.float32(0.03)
    W = np.array([[c, -c, c, -c] * 8], dtype=np.float32)
    assert ora.absmean_gamma(W) == c
    assert ora.ternary_round(W, c).tolist() == [[1, -1, 1, -1] * 8]
    # all-zero weights: mean 0 -> clamped to 1e-5, every code 0
    Z = np.zeros((4, 32), dtype=np.float32)
    assert ora.absmean_gamma(Z) == np.float32(1e-5)
    assert np.all(ora.ternary_round(Z, ora.absmean_gamma(Z)) == 0)
    # per-TENSOR scale: scaling one row must change gamma and other rows' codes
    rng = np.random.default_rng(0)
    W = rng.normal(0, 0.02, size=(8, 64)).astype(np.float32)
    g0 = ora.absmean_gamma(W)
    W2 = W.copy()
    W2[0] *= 10
    g1 = ora.absmean_gamma(W2)
    assert g1 > 2 * g0
    assert np.mean(np.abs(W)) == pytest.approx(g0, rel=1e-6)


def test_scalar_step_equivalence(ora):
    """P4 §1's scalar rule (x > .5 -> 1, x < -.5 -> -1, else 0) applied to fl32(W/gamma)
    must reproduce clamp(round_half_even(W/gamma), -1, 1) for every value, ties included."""
    rng = np.random.default_rng(3)
    W = rng.normal(0, 0.02, size=(64, 128)).astype(np.float32)
    gamma = ora.absmean_gamma(W)
    g32 = np.float32(gamma)
    # plant exact ties and boundary neighbours
    special = np.array([0.5, -0.5, 1.5, -1.5, 2.5, -2.5, 0.0, -0.0, 1.0, -1.0], dtype=np.float32) * g32
    W.flat[: special.size] = special
    v = (W / g32).astype(np.float32)
    step = np.where(v > 0.5, 1, np.where(v < -0.5, -1, 0)).astype(np.int8)
    assert np.array_equal(ora.ternary_round(W, gamma), step)


def _zero_fraction_gaussian():
    # W ~ N(0, s^2), gamma -> s*sqrt(2/pi); zero iff |W| <= gamma/2  => P(|Z| <= sqrt(2/pi)/2)
    a = 0.5 * math.sqrt(2.0 / math.pi)
    return math.erf(a / math.sqrt(2.0))


def _zero_fraction_t3():
    # t3: E|T| = 2*sqrt(3)/pi; P(|T| <= a) = (2/pi) * (a/(sqrt3 (1 + a^2/3)) + atan(a/sqrt3))
    a = 0.5 * 2.0 * math.sqrt(3.0) / math.pi
    return (2.0 / math.pi) * (a / (math.sqrt(3.0) * (1.0 + a * a / 3.0)) + math.atan(a / math.sqrt(3.0)))


def test_zero_fraction_gaussian(ora):
    """P3 §6 monitors (w_quant == 0).mean(); for Gaussian W it has the closed form 0.31006."""
    p = _zero_fraction_gaussian()
    assert p == pytest.approx(0.31006, abs=2e-5)
    W = synth.normal((2048, 2048), 0.02, synth.generator(11)).numpy()
    _, wq = ora.quant_weight(W)
    frac = float(np.mean(wq == 0))
    n = W.size
    sigma = math.sqrt(p * (1 - p) / n) + 0.0003      # binomial + sampling noise of gamma
    assert abs(frac - p) < 4 * sigma, (frac, p)
    # symmetric: +1 and -1 equally likely
    assert abs(np.mean(wq == 1) - np.mean(wq == -1)) < 4 * math.sqrt(0.35 / n)


def test_zero_fraction_student_t3(ora):
    p = _zero_fraction_t3()
    assert p == pytest.approx(0.38019, abs=2e-5)
    W = synth.student_t3((2048, 2048), 0.02, synth.generator(12)).numpy()
    _, wq = ora.quant_weight(W)
    frac = float(np.mean(wq == 0))
    assert abs(frac - p) < 0.004, (frac, p)


# ------------------------------------------------------------------------------------
# activation quantiser and RMSNorm
# ------------------------------------------------------------------------------------

def test_rmsnorm_matches_torch(ora):
    torch.manual_seed(0)
    X = torch.randn(33, 96)
    g = 1.0 + 0.1 * torch.randn(96)
    eps = 1e-6
    r = ora.rmsnorm_rinv(X, eps)
    ref = torch.nn.functional.rms_norm(X.double(), (96,), weight=g.double(), eps=eps)
    ours = X.double() * torch.from_numpy(r).double()[:, None] * g.double()
    assert torch.allclose(ours, ref, rtol=2e-7, atol=0)


def test_act_quant_invariants(ora):
    rng = np.random.default_rng(5)
    X = rng.normal(0, 1, size=(50, 160)).astype(np.float32)
    X[3] = 0.0                         # all-zero row: s = 127/1e-5, codes 0
    X[4] = 2.5                         # constant row: every code +127
    X[5, 7] = 1e-7                     # row below the 1e-5 clamp except one tiny entry
    X[5, :7] = 0
    X[5, 8:] = 0
    r = ora.rmsnorm_rinv(X, 1e-6)
    xq, s, xdq = ora.act_quant(X, r)
    assert xq.min() >= -127 and xq.max() <= 127          # -128 unreachable
    assert np.all(xq[3] == 0) and s[3] == np.float32(127.0) / np.float32(1e-5)
    assert np.all(xq[4] == 127)
    for t in range(50):
        if t in (3, 5):
            continue
        assert np.max(np.abs(xq[t])) == 127                # the absmax entry maps to +-127
    # rows are independent: per-token, not per-tensor
    X2 = X.copy()
    X2[10] *= 100
    xq2, s2, _ = ora.act_quant(X2, ora.rmsnorm_rinv(X2, 1e-6))
    keep = [t for t in range(50) if t != 10]
    assert np.array_equal(xq2[keep], xq[keep])
    # reconstruction error bound |x_hat - x_dq| <= 0.5/s (+ fp32 rounding)
    xhat = (X * r[:, None]).astype(np.float32)
    err = np.abs(xhat - xdq)
    bound = 0.5 / s[:, None] * (1 + 1e-6) + 1e-7 * np.abs(xhat)
    assert np.all(err <= bound)


def test_act_quant_scale_invariance(ora):
    """With gain 1 RMSNorm only rescales a row, which the per-row absmax scale cancels:
    codes of x and of RMSNorm(x) agree up to +-1 flips at rounding ties."""
    rng = np.random.default_rng(9)
    X = rng.normal(0, 3, size=(64, 256)).astype(np.float32)
    q_norm, _, _ = ora.act_quant(X, ora.rmsnorm_rinv(X, 1e-6))
    q_raw, _, _ = ora.act_quant(X)
    d = np.abs(q_norm.astype(int) - q_raw.astype(int))
    assert d.max() <= 1
    assert np.mean(d) < 1e-3


def test_round_bf16_matches_torch(ora):
    torch.manual_seed(1)
    x = torch.cat([torch.randn(4096) * 10, torch.tensor([1.0 + 2**-8, 1.0 + 3 * 2**-8, -1.0 - 2**-8, 65504.0])])
    ours = ora.round_bf16(x)
    ref = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# ------------------------------------------------------------------------------------
# contraction and epilogue
# ------------------------------------------------------------------------------------

def test_int_gemm_matches_numpy(ora):
    rng = np.random.default_rng(2)
    for T, N, K in [(1, 1, 32), (7, 13, 64), (33, 20, 96)]:
        xq = rng.integers(-127, 128, size=(T, K)).astype(np.int8)
        wq = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
        ref = xq.astype(np.int64) @ wq.astype(np.int64).T
        assert np.array_equal(ora.int_gemm(xq, wq), ref.astype(np.int32))
        rows = [T - 1, 0]
        assert np.array_equal(ora.int_gemm(xq, wq, rows=rows), ref[rows].astype(np.int32))


def test_forward_quantisation_error_bound(ora):
    """y must approximate x_hat . (W_q gamma)^T within the activation rounding error:
    |y - x_hat W_dq^T| <= 0.5 gamma nnz(W_q[n]) / s_t (+ fp32 rounding)."""
    li = synth.random_case(48, 160, 72, seed=21, dtype="f32")
    f = ora.forward(li.X, li.W)
    xhat = (li.X.numpy() * f["rinv"][:, None]).astype(np.float64)
    wdq = f["wq"].astype(np.float64) * f["gamma"]
    exact = xhat @ wdq.T
    nnz = np.sum(f["wq"] != 0, axis=1)
    bound = 0.5 * f["gamma"] * nnz[None, :] / f["s"][:, None].astype(np.float64)
    err = np.abs(f["y"] - exact)
    assert np.all(err <= bound * (1 + 1e-5) + 1e-6 * np.abs(exact))
    # and the bound is informative: y is far closer to x_hat W_dq^T than a transposed or
    # unscaled contraction would be
    assert np.max(err) < 0.05 * np.max(np.abs(exact))


def test_gemv_matches_unpacked_contraction(ora):
    rng = np.random.default_rng(4)
    N, K, B = 40, 128, 3
    wq = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    packed = ora.pack(wq)
    x = rng.normal(0, 1, size=(B, K)).astype(np.float32)
    xq, s, _ = ora.act_quant(x)
    acc, y = ora.gemv(packed, 0.0125, K, xq, s)
    ref = xq.astype(np.int64) @ wq.astype(np.int64).T
    assert np.array_equal(acc, ref.astype(np.int32))
    assert np.array_equal(y, ora.linear_epilogue(acc, 0.0125, s))


# ------------------------------------------------------------------------------------
# backward
# ------------------------------------------------------------------------------------

def test_backward_matches_autograd(ora):
    """The oracle's hand-written STE backward equals torch float64 autograd through the
    straight-through construction x + (q(x) - x).detach() (P3 §2.1-§3.2)."""
    li = synth.random_case(12, 64, 40, seed=31, dtype="f32", with_gain=True)
    eps = 1e-6
    f = ora.forward(li.X, li.W, g=li.g, eps=eps)
    dX, dW, dg, _ = ora.backward(li.X, li.dY, f, g=li.g)

    x = li.X.double().clone().requires_grad_(True)
    w = li.W.double().clone().requires_grad_(True)
    gg = li.g.double().clone().requires_grad_(True)
    xhat = torch.nn.functional.rms_norm(x, (64,), weight=gg, eps=eps)
    x_dq_value = torch.from_numpy(f["xdq"]).double()
    w_dq_value = torch.from_numpy(f["wq"]).double() * f["gamma"]
    x_ste = xhat + (x_dq_value - xhat).detach()
    w_ste = w + (w_dq_value - w).detach()
    y = x_ste @ w_ste.t()
    y.backward(li.dY.double())
    assert np.allclose(dW, w.grad.numpy(), rtol=1e-5, atol=1e-9)
    assert np.allclose(dX, x.grad.numpy(), rtol=1e-5, atol=1e-6 * np.abs(dX).max())
    assert np.allclose(dg, gg.grad.numpy(), rtol=1e-5, atol=1e-6 * np.abs(dg).max())


def test_rmsnorm_backward_finite_differences(ora):
    rng = np.random.default_rng(8)
    T, K = 3, 48
    X = rng.normal(0, 1, size=(T, K))
    g = 1 + 0.2 * rng.normal(size=K)
    c = rng.normal(size=(T, K))               # upstream gradient w.r.t. x_hat
    eps = 1e-6

    def f(Xv):
        r = 1.0 / np.sqrt(np.mean(Xv * Xv, axis=1, keepdims=True) + eps)
        return np.sum(c * Xv * r * g)

    num = np.zeros_like(X)
    h = 1e-6
    for i in range(T):
        for k in range(K):
            Xp = X.copy(); Xp[i, k] += h
            Xm = X.copy(); Xm[i, k] -= h
            num[i, k] = (f(Xp) - f(Xm)) / (2 * h)
    X32 = X.astype(np.float32)
    r = ora.rmsnorm_rinv(X32, eps)
    dX, dg = ora.rmsnorm_backward(X32, r, g.astype(np.float32), c.astype(np.float32))
    assert np.allclose(dX, num, rtol=1e-4, atol=1e-5)
    dg_ref = np.sum(c * X32.astype(np.float64) * r[:, None].astype(np.float64), axis=0)
    assert np.allclose(dg, dg_ref, rtol=1e-5, atol=1e-6)


def test_oracle_row_sampling_consistency(ora):
    """Sampled-row entry points (used at full sizes) equal the all-rows results."""
    li = synth.random_case(20, 64, 24, seed=41, dtype="f32")
    f = ora.forward(li.X, li.W)
    rows = [19, 3, 7]
    dxh_all = ora.grad_input_hat(li.dY, f["wq"], f["gamma"])
    assert np.array_equal(ora.grad_input_hat(li.dY, f["wq"], f["gamma"], rows=rows), dxh_all[rows])
    dW_all = ora.grad_weight(li.dY, f["xdq"])
    assert np.array_equal(ora.grad_weight(li.dY, f["xdq"], wrows=[5, 0]), dW_all[[5, 0]])
    dX_all, _ = ora.rmsnorm_backward(li.X, f["rinv"], None, dxh_all)
    dX_r, _ = ora.rmsnorm_backward(li.X, f["rinv"], None, dxh_all[rows], rows=rows)
    assert np.array_equal(dX_r, dX_all[rows])


# ------------------------------------------------------------------------------------
# the gain vector of the RMSNorm in front of the activation quantiser (P3 §3.1: the
# layer's RMSNorm(in_features) output feeds activation_quant)
# ------------------------------------------------------------------------------------

def _gain_case(T=48, K=192, seed=13):
    """Rows of N(0,1) with a gain vector spread wide enough (0.05 .. 4) that it moves the
    absmax entry of most rows, so a mishandled gain changes the scale, not just rounding."""
    gen = torch.Generator().manual_seed(seed)
    X = torch.randn(T, K, generator=gen, dtype=torch.float32)
    g = torch.exp(torch.randn(K, generator=gen, dtype=torch.float32) * 0.8).clamp(0.05, 4.0)
    return X, g


def _per_token_f64(X, g, eps):
    """Library RMSNorm (torch, float64) followed by the per-token absmax quantiser written
    in float64: s = 127 / max|x_hat|, v = x_hat s, q = clamp(round-half-even(v))."""
    K = X.shape[1]
    xh = torch.nn.functional.rms_norm(X.double(), (K,), weight=g.double(), eps=eps).numpy()
    m = np.max(np.abs(xh), axis=1, keepdims=True)
    s = 127.0 / np.maximum(m, 1e-5)
    v = xh * s
    return np.clip(np.rint(v), -128, 127), s[:, 0], v


def _per_tensor_f64(X, g, eps):
    K = X.shape[1]
    xh = torch.nn.functional.rms_norm(X.double(), (K,), weight=g.double(), eps=eps).numpy()
    s = 127.0 / max(float(np.max(np.abs(xh))), 1e-5)
    v = xh * s
    return np.clip(np.rint(v), -128, 127), np.full(X.shape[0], s), v


def _agrees_f64(xq, s, xdq, ref):
    """fp32 oracle output vs the float64 restatement.  x_hat in fp32 carries three roundings
    (r, x r, (x r) g) and s one more, so s agrees to 2^-20 relative and x_hat s to
    127 * 2^-20 absolute (< 1.3e-4): a code may differ by one only where the float64
    product lies that close to a .5 tie.  X_dq = q / s to 2^-20 relative."""
    ref_q, ref_s, ref_v = ref
    if not np.all(np.abs(s.astype(np.float64) - ref_s) <= 2.0 ** -20 * ref_s):
        return False
    d = xq.astype(np.int64) - ref_q.astype(np.int64)
    near_tie = np.abs(np.abs(ref_v - np.floor(ref_v)) - 0.5) < 1.3e-4
    if not (np.all(np.abs(d) <= 1) and np.all((d == 0) | near_tie)):
        return False
    want = xq.astype(np.float64) / ref_s[:, None]
    return bool(np.all(np.abs(xdq.astype(np.float64) - want) <= 2.0 ** -20 * np.abs(want)))


def test_act_quant_gain_matches_torch_rms_norm(ora):
    X, g = _gain_case()
    eps = 1e-6
    r = ora.rmsnorm_rinv(X, eps)
    xq, s, xdq = ora.act_quant(X, r, g)
    ref = _per_token_f64(X, g, eps)
    assert _agrees_f64(xq, s, xdq, ref)
    # the case is informative: the gain moved the absmax entry of most rows
    arg_gain = np.argmax(np.abs(ref[2]), axis=1)
    arg_raw = np.argmax(np.abs(X.numpy()), axis=1)
    assert np.mean(arg_gain != arg_raw) > 0.5


def test_act_quant_gain_pin_rejects_planted_mistakes(ora):
    """Each plausible slip in the gain path, planted by feeding the oracle the mistaken
    operands, must fail the float64 pin above."""
    X, g = _gain_case()
    eps = 1e-6
    Xn, gn = X.numpy(), g.numpy()
    r = ora.rmsnorm_rinv(X, eps)
    ref = _per_token_f64(X, g, eps)
    mistakes = {
        # gain dropped (x_hat = x r)
        "dropped": ora.act_quant(X, r, None),
        # gain applied before the normalisation statistic (r taken over x g)
        "inside_rms": ora.act_quant((Xn * gn).astype(np.float32), ora.rmsnorm_rinv(Xn * gn, eps), None),
        # gain indexed in reverse (a transposed / mis-strided gain read)
        "reversed": ora.act_quant(X, r, gn[::-1].copy()),
        # gain applied twice
        "squared": ora.act_quant(X, r, (gn * gn).astype(np.float32)),
        # gain divided instead of multiplied
        "inverted": ora.act_quant(X, r, (1.0 / gn).astype(np.float32)),
    }
    for name, (q_b, s_b, xdq_b) in mistakes.items():
        assert not _agrees_f64(q_b, s_b, xdq_b, ref), name


def test_act_quant_tensor_gain_matches_torch_rms_norm(ora):
    X, g = _gain_case(T=40, K=160, seed=17)
    eps = 1e-6
    r = ora.rmsnorm_rinv(X, eps)
    xq, s, xdq = ora.act_quant_tensor(X, r, g)
    ref = _per_tensor_f64(X, g, eps)
    assert _agrees_f64(xq, s, xdq, ref)
    Xn, gn = X.numpy(), g.numpy()
    mistakes = {
        "dropped": ora.act_quant_tensor(X, r, None),
        "inside_rms": ora.act_quant_tensor((Xn * gn).astype(np.float32), ora.rmsnorm_rinv(Xn * gn, eps), None),
        "reversed": ora.act_quant_tensor(X, r, gn[::-1].copy()),
        "per_token_scale": ora.act_quant(X, r, g),
    }
    for name, (q_b, s_b, xdq_b) in mistakes.items():
        assert not _agrees_f64(q_b, s_b, xdq_b, ref), name
