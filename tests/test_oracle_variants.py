"""Pins of the oracle's quantiser variants to facts that do not come from the oracle.

The variants are the cheap parameterisations the pages print beside the b1.58 defaults:
a per-output-row weight scale (P4 §9 "Quantizer"), a zero threshold tau = 0.7 gamma
(P2, section on the straight-through estimator) and a per-tensor activation scale
(P5 §5.1 quantize_activation).  Each pin is a closed form, a statistical law, a reduction
to an already pinned default, or an invariant that a plausible slip (per-tensor instead
of per-row, <= instead of <, a per-token max) breaks.
"""
import math

import numpy as np
import pytest

from bit_ternary_qat_b200 import synth


# ------------------------------------------------------------------------------------
# per-row weight scale
# ------------------------------------------------------------------------------------

def test_rows_gamma_closed_form(ora):
    c = np.array([0.5, 0.03, 2.0**-10, 7.0], dtype=np.float32)
    signs = np.array([1, -1, -1, 1, 1, 1, -1, 1] * 4, dtype=np.float32)
    W = c[:, None] * signs[None, :]
    g = ora.absmean_gamma_rows(W)
    assert g.tolist() == c.tolist()
    assert np.array_equal(ora.ternary_round_rows(W, g), np.broadcast_to(signs, W.shape).astype(np.int8))
    # an all-zero row takes the 1e-5 floor and all-zero codes; other rows are unaffected
    W[2] = 0.0
    g2, q2 = ora.quant_weight_rows(W)
    assert g2[2] == np.float32(1e-5) and np.all(q2[2] == 0)
    assert g2[[0, 1, 3]].tolist() == c[[0, 1, 3]].tolist()


def test_rows_gamma_is_per_row(ora):
    """Scaling one row by a power of two scales only its gamma and leaves every code as
    it was; the per-tensor quantiser changes other rows' codes under the same edit."""
    rng = np.random.default_rng(13)
    W = rng.normal(0, 0.02, size=(16, 96)).astype(np.float32)
    g, q = ora.quant_weight_rows(W)
    W2 = W.copy()
    W2[5] *= 64.0
    g2, q2 = ora.quant_weight_rows(W2)
    assert np.array_equal(q2, q)
    assert g2[5] == np.float32(64.0) * g[5]
    assert np.array_equal(np.delete(g2, 5), np.delete(g, 5))
    # each row's gamma equals the per-tensor gamma of that row alone
    for n in (0, 5, 15):
        assert g[n] == ora.absmean_gamma(W[n:n + 1])
        assert np.array_equal(q[n], ora.ternary_round(W[n:n + 1], g[n])[0])
    _, qt = ora.quant_weight(W2)
    _, qt0 = ora.quant_weight(W)
    assert not np.array_equal(np.delete(qt, 5, 0), np.delete(qt0, 5, 0))


def test_rows_zero_fraction_independent_of_row_scale(ora):
    """With per-row gamma, a Gaussian row has zero fraction P(|Z| <= sqrt(2/pi)/2) = 0.31006
    whatever its standard deviation; a shared gamma would zero small-sigma rows far more."""
    p = math.erf(0.5 * math.sqrt(2.0 / math.pi) / math.sqrt(2.0))
    gen = synth.generator(17)
    sig = np.array([0.002, 0.02, 0.2, 2.0], dtype=np.float64)
    W = np.concatenate([synth.normal((64, 4096), float(s), gen).numpy() for s in sig])
    _, q = ora.quant_weight_rows(W)
    n = 64 * 4096
    for i in range(4):
        frac = float(np.mean(q[64 * i:64 * (i + 1)] == 0))
        assert abs(frac - p) < 4 * math.sqrt(p * (1 - p) / n) + 0.002, (i, frac, p)


def test_rows_epilogue_reduces_to_per_tensor(ora):
    rng = np.random.default_rng(19)
    acc = rng.integers(-20000, 20000, size=(6, 10)).astype(np.int32)
    s = rng.uniform(5, 300, size=6).astype(np.float32)
    y_t = ora.linear_epilogue(acc, 0.0173, s)
    y_r = ora.linear_epilogue_rows(acc, np.full(10, 0.0173, dtype=np.float32), s)
    assert np.array_equal(y_r, y_t)
    # a per-column scale multiplies column n only (power-of-two factor: exact)
    g = np.full(10, 0.0173, dtype=np.float32)
    g[3] *= 4
    y4 = ora.linear_epilogue_rows(acc, g, s)
    assert np.array_equal(y4[:, 3], 4 * y_t[:, 3])
    assert np.array_equal(np.delete(y4, 3, 1), np.delete(y_t, 3, 1))


def test_rows_forward_error_bound(ora):
    """x_hat . (W_q gamma_n)^T is reached within the activation rounding error when the
    contraction runs on the per-row codes and the epilogue applies gamma_n / s_t."""
    li = synth.random_case(24, 128, 40, seed=23, dtype="f32")
    X = li.X.numpy()
    W = li.W.numpy() * np.linspace(0.1, 3.0, 40, dtype=np.float32)[:, None]
    r = ora.rmsnorm_rinv(X, 1e-6)
    xq, s, _ = ora.act_quant(X, r)
    g, q = ora.quant_weight_rows(W)
    y = ora.linear_epilogue_rows(ora.int_gemm(xq, q), g, s)
    xhat = (X * r[:, None]).astype(np.float64)
    exact = xhat @ (q.astype(np.float64) * g[:, None].astype(np.float64)).T
    nnz = np.sum(q != 0, axis=1)
    bound = 0.5 * g[None, :].astype(np.float64) * nnz[None, :] / s[:, None].astype(np.float64)
    assert np.all(np.abs(y - exact) <= bound * (1 + 1e-5) + 1e-6 * np.abs(exact))


# ------------------------------------------------------------------------------------
# zero threshold tau = f * gamma
# ------------------------------------------------------------------------------------

def test_tau_half_is_the_round_rule(ora):
    """0.5 gamma is exact in fp32, so |W| < 0.5 gamma zeroes exactly the weights the
    round/clamp rule zeroes, except exact ties fl(W/gamma) = +-0.5, where round-half-even
    gives 0 and the threshold keeps the sign."""
    rng = np.random.default_rng(29)
    W = rng.normal(0, 0.02, size=(64, 256)).astype(np.float32)
    gamma = ora.absmean_gamma(W)
    W.flat[:4] = np.array([0.5, -0.5, 0.49999997, 1.5], dtype=np.float32) * np.float32(gamma)
    qt = ora.ternary_tau(W, gamma, 0.5)
    qr = ora.ternary_round(W, gamma)
    tie = np.abs((W / np.float32(gamma)).astype(np.float32)) == np.float32(0.5)
    assert tie.sum() >= 2
    assert np.array_equal(qt[~tie], qr[~tie])
    assert np.all(qr[tie] == 0) and np.array_equal(qt[tie], np.sign(W[tie]).astype(np.int8))


def test_tau_zero_fraction_gaussian(ora):
    """Gaussian W with tau = 0.7 gamma: zero fraction P(|Z| < 0.7 sqrt(2/pi)) = erf(0.7/sqrt(pi))."""
    p = math.erf(0.7 / math.sqrt(math.pi))
    assert p == pytest.approx(0.42351, abs=2e-5)
    W = synth.normal((2048, 2048), 0.02, synth.generator(31)).numpy()
    gamma = ora.absmean_gamma(W)
    q = ora.ternary_tau(W, gamma, 0.7)
    frac = float(np.mean(q == 0))
    assert abs(frac - p) < 4 * math.sqrt(p * (1 - p) / W.size) + 0.0004, (frac, p)
    assert set(np.unique(q).tolist()) == {-1, 0, 1}
    nz = q != 0
    assert np.array_equal(q[nz], np.sign(W[nz]).astype(np.int8))


def test_tau_boundary_and_monotonicity(ora):
    gamma = np.float32(0.0125)
    tau = np.float32(np.float32(0.7) * gamma)
    below = np.nextafter(tau, np.float32(0))
    W = np.array([tau, -tau, below, -below, 0.0, -0.0, 10.0, -10.0], dtype=np.float32)
    q = ora.ternary_tau(W, gamma, 0.7)
    assert q.tolist() == [1, -1, 0, 0, 0, 0, 1, -1]
    rng = np.random.default_rng(37)
    X = rng.normal(0, 0.02, size=4096).astype(np.float32)
    g = ora.absmean_gamma(X)
    zeros = [np.mean(ora.ternary_tau(X, g, f) == 0) for f in (0.0, 0.3, 0.5, 0.7, 0.8, 2.0)]
    assert zeros[0] == 0.0
    # a zero threshold keeps every sign, and an exact zero weight still has code 0
    assert ora.ternary_tau(np.array([0.0, -0.0, 1e-30, -1e-30], dtype=np.float32), g, 0.0).tolist() == [0, 0, 1, -1]
    assert all(a <= b for a, b in zip(zeros, zeros[1:]))


# ------------------------------------------------------------------------------------
# per-tensor activation scale
# ------------------------------------------------------------------------------------

def test_act_tensor_single_token_is_per_token(ora):
    rng = np.random.default_rng(41)
    x = rng.normal(0, 2, size=(1, 200)).astype(np.float32)
    r = ora.rmsnorm_rinv(x, 1e-6)
    for rr in (None, r):
        a = ora.act_quant_tensor(x, rr)
        b = ora.act_quant(x, rr)
        for u, v in zip(a, b):
            assert np.array_equal(u, v)


def test_act_tensor_shared_scale(ora):
    """One s for the whole tensor: the absmax entry of the tensor maps to +-127, a token
    whose own max is 1/4 of it reaches at most 32, and rows are no longer independent."""
    rng = np.random.default_rng(43)
    X = rng.uniform(-1, 1, size=(8, 64)).astype(np.float32)
    X[2, 9] = 4.0
    X[5] *= 0.25
    q, s, xdq = ora.act_quant_tensor(X)
    assert np.all(s == s[0]) and s[0] == np.float32(127.0) / np.float32(4.0)
    assert q[2, 9] == 127 and int(np.abs(q).max()) == 127
    assert int(np.abs(q[5]).max()) <= 32
    # exact rounding: codes equal round-half-even of x * s computed in float64 except
    # where fl32 rounding of the product lands on a tie (not the case for these values)
    ref = np.clip(np.rint(X.astype(np.float64) * float(s[0])), -128, 127).astype(np.int8)
    assert np.array_equal(q, ref)
    assert np.max(np.abs(X - xdq)) <= 0.5 / s[0] * (1 + 1e-6)
    # raising one token's magnitude changes every other token's codes
    X2 = X.copy()
    X2[0, 0] = 8.0
    q2, s2, _ = ora.act_quant_tensor(X2)
    assert s2[0] == s[0] / 2
    assert not np.array_equal(q2[1:], q[1:])


def test_act_tensor_equal_row_max_is_per_token(ora):
    """When every token has the same absmax the per-tensor and per-token scales agree."""
    rng = np.random.default_rng(47)
    X = rng.uniform(-1, 1, size=(12, 80)).astype(np.float32)
    X[:, 0] = np.where(np.arange(12) % 2 == 0, 1.5, -1.5)
    a = ora.act_quant_tensor(X)
    b = ora.act_quant(X)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
