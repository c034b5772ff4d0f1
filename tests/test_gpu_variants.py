"""GPU parity of the quantiser variants against the CPU oracle (through the C ABI).

Per-row weight scale (P4 §9 "Quantizer"), zero threshold tau = f * gamma (P2) and
per-tensor activation scale (P5 §5.1).  Integer codes, packed bytes, scales and the
linear / GEMV outputs are compared bit for bit; where a reduction order could move an
fp32 scale by one ulp the test allows <= 1 ulp and re-runs the oracle's downstream
steps with the GPU's value, as the default-path tests do.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_ternary_qat_b200 import _lib, synth
from parity_util import TOL, f32_of, max_rel_err, np_, sample_rows, ulp_diff

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _gpu(t):
    if isinstance(t, np.ndarray):
        t = torch.from_numpy(t)
    return t.to(DEV).contiguous()


def _signed_bf16_bits(wq, mag_bits):
    """bf16 bits of wq * m for codes wq in {-1, 0, 1} and bf16 magnitudes m (per row)."""
    mag = np.broadcast_to(np.asarray(mag_bits, dtype=np.uint16).reshape(-1, 1), wq.shape)
    out = np.where(wq > 0, mag, np.where(wq < 0, mag | np.uint16(0x8000), np.uint16(0)))
    return out.astype(np.uint16)


# ------------------------------------------------------------------------------------
# per-row weight scale
# ------------------------------------------------------------------------------------

def _check_quant_rows(bl, W):
    o = bl.bitlinear_quant_weight_rows(_gpu(W))
    torch.cuda.synchronize()
    g_gpu = np_(o["gamma_rows"])
    g_ora = oracle.absmean_gamma_rows(W)
    assert ulp_diff(g_gpu, g_ora).max() <= 1
    wq = oracle.ternary_round_rows(W, g_gpu)          # conditional on the GPU's gammas
    assert np.array_equal(np_(o["wq_i8"]), wq)
    assert np.array_equal(np_(o["packed"]), oracle.pack(wq))
    assert np.array_equal(np_(o["wq_bf16"]), _signed_bf16_bits(wq, oracle.round_bf16(g_gpu)))
    return g_gpu, wq, o


@pytest.mark.parametrize("N,K,dist,seed", [
    (512, 256, "normal", 0), (48, 160, "normal", 1), (16, 32, "normal", 2), (2064, 416, "student_t3", 3),
    (2048, 2048, "normal", 4), (64, 11008, "normal", 5)])
def test_quant_weight_rows_parity(bl, N, K, dist, seed):
    gen = synth.generator(seed)
    W = synth.student_t3((N, K), 0.02, gen) if dist == "student_t3" else synth.normal((N, K), 0.02, gen)
    # rows of very different scale: a shared gamma would not reproduce these codes
    W = W * torch.logspace(-2, 2, N, dtype=torch.float32)[:, None]
    g, _, _ = _check_quant_rows(bl, W.numpy())
    assert np.array_equal(g, oracle.absmean_gamma_rows(W.numpy()))     # expected exactly equal


def test_quant_weight_rows_edge_cases(bl):
    rng = np.random.default_rng(6)
    W = rng.normal(0, 0.02, size=(32, 128)).astype(np.float32)
    W[0] = 0.0                                        # gamma floor 1e-5, codes 0
    W[1] = np.float32(0.0375) * np.where(np.arange(128) % 2 == 0, 1, -1).astype(np.float32)
    g_row = oracle.absmean_gamma_rows(W)
    W[2, :4] = np.array([0.5, -0.5, 1.5, -2.5], dtype=np.float32) * g_row[2]   # ties after
    g, wq, _ = _check_quant_rows(bl, W)
    assert g[0] == np.float32(1e-5) and np.all(wq[0] == 0)
    assert g[1] == np.float32(0.0375) and np.all(np.abs(wq[1]) == 1)


# ------------------------------------------------------------------------------------
# zero threshold
# ------------------------------------------------------------------------------------

@pytest.mark.parametrize("tau", [0.0, 0.5, 0.7, 0.8, 2.0])
@pytest.mark.parametrize("N,K,seed", [(512, 256, 0), (48, 160, 1), (2048, 2048, 2)])
def test_quant_weight_tau_parity(bl, N, K, seed, tau):
    W = synth.normal((N, K), 0.02, synth.generator(seed)).numpy().copy()
    W[0, :8] = 0.0                                    # exact zeros keep code 0 at every tau
    o = bl.bitlinear_quant_weight_tau(_gpu(W), tau)
    torch.cuda.synchronize()
    g = float(o["gamma"].item())
    assert ulp_diff(np.float32(g), np.float32(oracle.absmean_gamma(W))) <= 1
    wq = oracle.ternary_tau(W, g, tau)
    assert np.array_equal(np_(o["wq_i8"]), wq)
    assert np.array_equal(f32_of(o["wq_bf16"]), wq.astype(np.float32))
    assert np.array_equal(np_(o["packed"]), oracle.pack(wq))
    assert np.all(wq[0, :8] == 0)


def test_quant_weight_tau_boundary(bl):
    """Weights exactly at tau and one ulp below it, for the page's 0.7."""
    rng = np.random.default_rng(8)
    W = rng.normal(0, 0.02, size=(16, 64)).astype(np.float32)
    g = oracle.absmean_gamma(W)
    tau = np.float32(np.float32(0.7) * np.float32(g))
    below = np.nextafter(tau, np.float32(0))
    W[3, :4] = [tau, -tau, below, -below]
    # the four planted values move gamma; re-plant around the new gamma until it is stable
    for _ in range(4):
        g = oracle.absmean_gamma(W)
        tau = np.float32(np.float32(0.7) * np.float32(g))
        below = np.nextafter(tau, np.float32(0))
        W[3, :4] = [tau, -tau, below, -below]
    o = bl.bitlinear_quant_weight_tau(_gpu(W), 0.7)
    torch.cuda.synchronize()
    gg = float(o["gamma"].item())
    wq = oracle.ternary_tau(W, gg, 0.7)
    assert np.array_equal(np_(o["wq_i8"]), wq)
    if gg == g:
        assert wq[3, :4].tolist() == [1, -1, 0, 0]


def test_quant_weight_tau_rejects_bad_factor(bl):
    W = torch.zeros(16, 32, device=DEV)
    gamma = torch.empty(1, device=DEV)
    ws = bl.workspace(1, 16, 32, DEV)
    for bad in (-0.1, float("nan"), float("inf")):
        st = _lib.status("bitlinear_quant_weight_tau", W.data_ptr(), 16, 32, bad, None, None, None,
                         gamma.data_ptr(), ws.data_ptr(), ws.numel(), None)
        assert st == 1                                # BL_ERR_INVALID_ARG


# ------------------------------------------------------------------------------------
# per-tensor activation scale
# ------------------------------------------------------------------------------------

def _check_act_tensor(bl, X, g, apply_norm, eps=1e-6):
    o = bl.bitlinear_act_quant_tensor(_gpu(X), apply_rmsnorm=apply_norm, g=None if g is None else _gpu(g), eps=eps)
    torch.cuda.synchronize()
    rinv = None
    if apply_norm:
        r_gpu = np_(o["rinv"])
        d = ulp_diff(r_gpu, oracle.rmsnorm_rinv(X, eps))
        assert d.max() <= 1 and np.mean(d > 0) < 0.01
        rinv = r_gpu
    xq, s, xdq = oracle.act_quant_tensor(X, rinv, g if apply_norm else None)
    assert np.array_equal(np_(o["sx"]), s)
    assert np.array_equal(np_(o["xq"]), xq)
    if X.dtype == torch.bfloat16:
        assert np.array_equal(np_(o["xdq"]), oracle.round_bf16(xdq))
    else:
        assert np.array_equal(np_(o["xdq"]), xdq)
    return o


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("T,K", [(1, 32), (7, 256), (300, 2080), (64, 11008), (9999, 128)])
@pytest.mark.parametrize("norm,gain", [(True, False), (True, True), (False, False)])
def test_act_quant_tensor_parity(bl, dtype, T, K, norm, gain):
    li = synth.random_case(T, K, 16, seed=T + K, dtype=dtype, with_gain=gain)
    X = li.X
    if T > 1:
        # token magnitudes over four decades: a per-token scale would give other codes
        X = (X.float() * torch.logspace(-2, 2, T)[:, None]).to(X.dtype)
    _check_act_tensor(bl, X, li.g, norm)


def test_act_quant_tensor_edge_cases(bl):
    X = torch.randn(6, 64, generator=synth.generator(3))
    X[0] = 0.0
    X[3] *= 1e4
    for norm in (True, False):
        _check_act_tensor(bl, X, None, norm)
        _check_act_tensor(bl, X.to(torch.bfloat16), None, norm)
    Z = torch.zeros(5, 96)                            # whole tensor zero: s = 127/1e-5, codes 0
    o = _check_act_tensor(bl, Z, None, False)
    assert np.all(np_(o["xq"]) == 0)


# ------------------------------------------------------------------------------------
# linear and GEMV with per-row weight scales
# ------------------------------------------------------------------------------------

@pytest.mark.parametrize("T,K,N", [(64, 256, 512), (300, 160, 400), (129, 4096, 272), (1, 32, 16),
                                   (513, 1024, 2064), (4096, 2048, 2048)])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_linear_rows_parity(bl, T, K, N, out):
    rng = np.random.default_rng(T * 5 + N)
    xq = rng.integers(-127, 128, size=(T, K)).astype(np.int8)
    wq = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    s = rng.uniform(10, 200, size=T).astype(np.float32)
    gam = rng.uniform(1e-3, 5e-2, size=N).astype(np.float32)
    y, acc = bl.bitlinear_linear_rows(_gpu(xq), _gpu(s), _gpu(wq), _gpu(gam),
                                      out_dtype=torch.bfloat16 if out == "bf16" else torch.float32, want_acc=True)
    torch.cuda.synchronize()
    rows = None if T * N <= 600_000 else sample_rows(T, 40, seed=T)
    acc_ora = oracle.int_gemm(xq, wq, rows=rows)
    acc_gpu = np_(acc) if rows is None else np_(acc)[rows]
    assert np.array_equal(acc_gpu, acc_ora)
    y_ora = oracle.linear_epilogue_rows(acc_ora, gam, s if rows is None else s[rows])
    y_gpu = np_(y) if rows is None else np_(y)[rows]
    if out == "bf16":
        assert np.array_equal(y_gpu, oracle.round_bf16(y_ora))
    else:
        assert np.array_equal(y_gpu, y_ora)


@pytest.mark.parametrize("N,K", [(48, 64), (400, 192), (1024, 8192), (4800, 704)])
@pytest.mark.parametrize("B", [1, 5, 16])
def test_gemv_rows_parity(bl, N, K, B):
    W, x = synth.decode_inputs(B, N, K, seed=N + K + B)
    W = W * torch.logspace(-1, 1, N, dtype=torch.float32)[:, None]
    qw = bl.bitlinear_quant_weight_rows(_gpu(W), want_i8=False, want_bf16=False)
    aq = bl.bitlinear_act_quant(_gpu(x), apply_rmsnorm=False, want_xdq=False)
    y, acc = bl.ternary_gemv_rows(qw["packed"], qw["gamma_rows"], K, aq["xq"], aq["sx"], want_acc=True)
    torch.cuda.synchronize()
    acc_o, _ = oracle.gemv(np_(qw["packed"]), 1.0, K, np_(aq["xq"]), np_(aq["sx"]))
    assert np.array_equal(np_(acc), acc_o)
    assert np.array_equal(np_(y), oracle.linear_epilogue_rows(acc_o, np_(qw["gamma_rows"]), np_(aq["sx"])))


@pytest.mark.parametrize("T,K,N,dtype", [(256, 512, 384, "bf16"), (300, 1024, 2064, "bf16")])
def test_rows_layer_forward_and_grad_input(bl, T, K, N, dtype):
    """Per-row layer: quantisers, linear with gamma_n / s_t, and the input-side gradient
    dX_hat = dY . (W_q * bf16(gamma_n)) from the dequantised bf16 weight with gamma = 1."""
    li = synth.random_case(T, K, N, seed=T + N, dtype=dtype)
    W = li.W * torch.linspace(0.2, 5.0, N)[:, None]
    qw = bl.bitlinear_quant_weight_rows(_gpu(W))
    aq = bl.bitlinear_act_quant(_gpu(li.X))
    y, acc = bl.bitlinear_linear_rows(aq["xq"], aq["sx"], qw["wq_i8"], qw["gamma_rows"], want_acc=True)
    one = torch.ones(1, device=DEV)
    dxh = bl.bitlinear_grad_input(_gpu(li.dY), qw["wq_bf16"], one)
    torch.cuda.synchronize()
    g = np_(qw["gamma_rows"])
    wq = oracle.ternary_round_rows(W.numpy(), g)
    assert np.array_equal(np_(qw["wq_i8"]), wq)
    rows = sample_rows(T, 24, seed=N)
    acc_o = oracle.int_gemm(np_(aq["xq"]), wq, rows=rows)
    assert np.array_equal(np_(acc)[rows], acc_o)
    y_o = oracle.linear_epilogue_rows(acc_o, g, np_(aq["sx"])[rows])
    assert np.array_equal(np_(y)[rows], oracle.round_bf16(y_o))
    wdq = f32_of(qw["wq_bf16"]).astype(np.float64)
    assert np.array_equal(wdq, wq.astype(np.float64) * f32_of(torch.from_numpy(g).to(torch.bfloat16))[:, None])
    dY = f32_of(li.dY).astype(np.float64)
    ref = dY[rows] @ wdq
    assert max_rel_err(np_(dxh)[rows], ref) <= TOL[dtype]
