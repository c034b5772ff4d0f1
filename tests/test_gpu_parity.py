"""GPU parity: the CUDA path, called through the C ABI, against the CPU oracle.

Bit-exact: gamma, W_q (int8 / bf16), packed bytes, r, s, x_q, X_dq, int32 accumulators,
Y (the epilogue is the same fp32 arithmetic on exact integers) and the GEMV.  Where a
reduction order could move an fp32 result by one ulp (r from sum x^2, gamma from
sum |W|), the test asserts <= 1 ulp and re-runs the oracle's downstream steps with the
GPU's value, so every integer code is still compared exactly.
Float gradients: max|gpu - oracle| / max|oracle| <= 2e-3 (bf16 layer) or 1e-4 (fp32).
"""
import numpy as np
import pytest
import torch

import oracle
from bit_ternary_qat_b200 import synth
from parity_util import TOL, f32_of, max_rel_err, np_, sample_rows, ulp_diff

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _gpu(t):
    return t.to(DEV).contiguous()


# ------------------------------------------------------------------------------------
# failure path: bounded waits report a timeout instead of hanging
# ------------------------------------------------------------------------------------

def test_bounded_wait_reports_timeout(bl):
    assert bl.check_device_status() == 0
    bl.selftest_bounded_wait(50_000_000)            # 50 ms on a barrier nothing arrives on
    assert bl.check_device_status() == 6            # BL_ERR_TIMEOUT
    assert bl.check_device_status() == 0            # cleared; the context is still usable
    x = torch.ones(4, device=DEV)
    assert float(x.sum()) == 4.0


# ------------------------------------------------------------------------------------
# weight quantiser and packing
# ------------------------------------------------------------------------------------

def _check_quant_weight(bl, W):
    N, K = W.shape
    out = bl.bitlinear_quant_weight(_gpu(W))
    torch.cuda.synchronize()
    g_gpu = float(out["gamma"].item())
    g_ora = oracle.absmean_gamma(W)
    assert ulp_diff(np.float32(g_gpu), np.float32(g_ora)) <= 1, (g_gpu, g_ora)
    wq = oracle.ternary_round(W, g_gpu)               # conditional on the GPU's gamma
    assert np.array_equal(np_(out["wq_i8"]), wq)
    assert np.array_equal(f32_of(out["wq_bf16"]), wq.astype(np.float32))
    assert np.array_equal(np_(out["packed"]), oracle.pack(wq))
    return g_gpu, wq, out


@pytest.mark.parametrize("N,K,dist,seed", [
    (512, 256, "normal", 0), (48, 160, "normal", 1), (16, 32, "normal", 2), (2064, 416, "student_t3", 3),
    (2048, 2048, "normal", 4)])
def test_quant_weight_parity(bl, N, K, dist, seed):
    gen = synth.generator(seed)
    W = synth.student_t3((N, K), 0.02, gen) if dist == "student_t3" else synth.normal((N, K), 0.02, gen)
    g, wq, _ = _check_quant_weight(bl, W)
    assert g == np.float32(oracle.absmean_gamma(W))    # expected exactly equal


def test_quant_weight_edge_cases(bl):
    Z = torch.zeros(32, 64)
    g, wq, _ = _check_quant_weight(bl, Z)
    assert g == np.float32(1e-5) and np.all(wq == 0)
    c = np.float32(0.0375)
    W = torch.full((16, 32), float(c))
    W[::2] *= -1
    g, wq, _ = _check_quant_weight(bl, W)
    assert g == c
    # exact ties at +-0.5 gamma and +-1.5 gamma: W/gamma must round half to even
    rng = np.random.default_rng(0)
    W = torch.from_numpy(rng.normal(0, 0.02, size=(64, 128)).astype(np.float32))
    g0 = oracle.absmean_gamma(W)
    flat = W.view(-1)
    for i, m in enumerate([0.5, -0.5, 1.5, -1.5, 2.5, 0.49999997, 0.50000006]):
        flat[i] = float(np.float32(m) * np.float32(g0))
    _check_quant_weight(bl, W)


def test_quant_weight_deterministic(bl):
    W = synth.normal((1024, 1024), 0.02, synth.generator(5))
    a = bl.bitlinear_quant_weight(_gpu(W))
    b = bl.bitlinear_quant_weight(_gpu(W))
    torch.cuda.synchronize()
    assert torch.equal(a["gamma"], b["gamma"])
    assert torch.equal(a["packed"], b["packed"])


def test_ternary_pack_parity(bl):
    rng = np.random.default_rng(9)
    wq = rng.integers(-1, 2, size=(80, 96)).astype(np.int8)
    packed = bl.ternary_pack(_gpu(torch.from_numpy(wq)))
    assert np.array_equal(np_(packed), oracle.pack(wq))


# ------------------------------------------------------------------------------------
# activation quantiser (RMSNorm fused)
# ------------------------------------------------------------------------------------

def _check_act_quant(bl, X, g, apply_norm, eps=1e-6):
    o = bl.bitlinear_act_quant(_gpu(X), apply_rmsnorm=apply_norm, g=None if g is None else _gpu(g), eps=eps)
    torch.cuda.synchronize()
    rinv = None
    if apply_norm:
        r_gpu = np_(o["rinv"])
        r_ora = oracle.rmsnorm_rinv(X, eps)
        d = ulp_diff(r_gpu, r_ora)
        assert d.max() <= 1, d.max()
        assert np.mean(d > 0) < 0.01
        rinv = r_gpu
    xq, s, xdq = oracle.act_quant(X, rinv, g if apply_norm else None)
    assert np.array_equal(np_(o["sx"]), s)
    assert np.array_equal(np_(o["xq"]), xq)
    if X.dtype == torch.bfloat16:
        assert np.array_equal(np_(o["xdq"]), oracle.round_bf16(xdq))
    else:
        assert np.array_equal(np_(o["xdq"]), xdq)
    return o


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("T,K", [(1, 32), (7, 256), (300, 2080), (64, 11008)])
@pytest.mark.parametrize("norm,gain", [(True, False), (True, True), (False, False)])
def test_act_quant_parity(bl, dtype, T, K, norm, gain):
    li = synth.random_case(T, K, 16, seed=T + K, dtype=dtype, with_gain=gain)
    _check_act_quant(bl, li.X, li.g, norm)


def test_act_quant_edge_rows(bl):
    X = torch.randn(6, 64, generator=synth.generator(3))
    X[0] = 0.0                  # all zero -> s = 127/1e-5, codes 0
    X[1] = 3.0                  # constant
    X[2, :] = 0.0
    X[2, 5] = -1e-30            # tiny absmax below the clamp
    X[3] *= 1e4
    for norm in (True, False):
        _check_act_quant(bl, X, None, norm)
        _check_act_quant(bl, X.to(torch.bfloat16), None, norm)


# ------------------------------------------------------------------------------------
# int8 x ternary tcgen05 GEMM + epilogue
# ------------------------------------------------------------------------------------

@pytest.mark.parametrize("T,K,N", [(64, 256, 512), (300, 160, 400), (129, 4096, 272), (1, 32, 16),
                                   (513, 1024, 2064), (4096, 2048, 2048)])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_linear_parity(bl, T, K, N, out):
    rng = np.random.default_rng(T * 7 + N)
    xq = rng.integers(-127, 128, size=(T, K)).astype(np.int8)
    wq = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    s = rng.uniform(10, 200, size=T).astype(np.float32)
    gamma = np.float32(0.0173)
    y, acc = bl.bitlinear_linear(_gpu(torch.from_numpy(xq)), _gpu(torch.from_numpy(s)),
                                 _gpu(torch.from_numpy(wq)), _gpu(torch.tensor([gamma])),
                                 out_dtype=torch.bfloat16 if out == "bf16" else torch.float32, want_acc=True)
    torch.cuda.synchronize()
    rows = None if T * N <= 600_000 else sample_rows(T, 40, seed=T)
    acc_ora = oracle.int_gemm(xq, wq, rows=rows)
    acc_gpu = np_(acc) if rows is None else np_(acc)[rows]
    assert np.array_equal(acc_gpu, acc_ora)
    y_ora = oracle.linear_epilogue(acc_ora, float(gamma), s if rows is None else s[rows])
    y_gpu = np_(y) if rows is None else np_(y)[rows]
    if out == "bf16":
        assert np.array_equal(y_gpu, oracle.round_bf16(y_ora))
    else:
        assert np.array_equal(y_gpu, y_ora)
    if rows is not None:
        # every output, via an exact property: acc equals the int64 product on all rows
        full = torch.from_numpy(xq).to(DEV).float() @ torch.from_numpy(wq).to(DEV).float().t()
        assert torch.equal(acc.float(), full)      # |acc| < 2^24: exact in fp32


# ------------------------------------------------------------------------------------
# whole layer: forward then backward
# ------------------------------------------------------------------------------------

def _layer_case(bl, li, eps=1e-6):
    dt = "bf16" if li.X.dtype == torch.bfloat16 else "f32"
    T, K = li.X.shape
    N = li.W.shape[0]
    g_gpu, wq, qw = _check_quant_weight(bl, li.W)
    g = None if li.g is None else _gpu(li.g)
    f = bl.bitlinear_forward(_gpu(li.X), qw["wq_i8"], qw["gamma"], g=g, eps=eps, want_acc=True)
    dX, dW, dg = bl.bitlinear_backward(_gpu(li.dY), _gpu(li.X), f["xdq"], f["rinv"], qw["wq_bf16"], qw["gamma"],
                                       g=g)
    torch.cuda.synchronize()
    return dt, g_gpu, wq, f, dX, dW, dg


def test_single_workload_seed0(bl):
    """The single-layer fp32 workload exactly as specified (X 64x256, W 512x256, dY 64x512,
    seed 0, gain 1): every code, accumulator and output exact, gradients within 1e-4."""
    li = synth.workload_inputs("single")[0]
    assert li.X.dtype == torch.float32 and tuple(li.X.shape) == (64, 256) and tuple(li.W.shape) == (512, 256)
    dt, g_gpu, wq, f, dX, dW, dg = _layer_case(bl, li)
    r_gpu = np_(f["rinv"])
    assert ulp_diff(r_gpu, oracle.rmsnorm_rinv(li.X, 1e-6)).max() <= 1
    ref = oracle.forward(li.X, li.W, rinv=r_gpu, gamma=g_gpu, out_dtype="f32")
    for k_gpu, k_ref in (("xq", "xq"), ("sx", "s"), ("acc", "acc"), ("y", "y"), ("xdq", "xdq")):
        assert np.array_equal(np_(f[k_gpu]), ref[k_ref]), k_gpu
    dX_o, dW_o, dg_o, _ = oracle.backward(li.X, li.dY, ref)
    for name, a, b in (("dX", dX, dX_o), ("dW", dW, dW_o), ("dg", dg, dg_o)):
        assert max_rel_err(np_(a), b) <= TOL["f32"], name


@pytest.mark.parametrize("T,K,N,dtype,gain", [
    (64, 256, 512, "f32", False),        # the single-layer fp32 shape on another seed
    (3800, 1280, 3840, "bf16", False),   # 225 / 75 / 75 pair tiles: the 2-SM GEMMs' last partial
                                         # wave runs as half tiles (ragged rows and columns too)
    (300, 160, 400, "bf16", True),
    (257, 512, 144, "f32", True),
    (130, 1024, 784, "bf16", False),
])
def test_layer_parity(bl, T, K, N, dtype, gain):
    li = synth.random_case(T, K, N, seed=100 + T, dtype=dtype, with_gain=gain,
                           dy_std=1.0 if dtype == "f32" else 1e-2)
    dt, g_gpu, wq, f, dX, dW, dg = _layer_case(bl, li)
    r_gpu = np_(f["rinv"])
    assert ulp_diff(r_gpu, oracle.rmsnorm_rinv(li.X, 1e-6)).max() <= 1
    ref = oracle.forward(li.X, li.W, g=li.g, rinv=r_gpu, gamma=g_gpu, out_dtype=dt)
    assert np.array_equal(np_(f["xq"]), ref["xq"])
    assert np.array_equal(np_(f["sx"]), ref["s"])
    assert np.array_equal(np_(f["acc"]), ref["acc"])
    if dt == "bf16":
        assert np.array_equal(np_(f["y"]), ref["y_bf16"])
        assert np.array_equal(np_(f["xdq"]), ref["xdq_bf16"])
    else:
        assert np.array_equal(np_(f["y"]), ref["y"])
        assert np.array_equal(np_(f["xdq"]), ref["xdq"])
    dX_o, dW_o, dg_o, _ = oracle.backward(li.X, li.dY, ref, g=li.g)
    tol = TOL[dt]
    assert max_rel_err(np_(dW), dW_o) <= tol
    assert max_rel_err(np_(dX), dX_o) <= tol
    assert max_rel_err(np_(dg), dg_o) <= tol


@pytest.mark.parametrize("T,K,N,dtype,gain", [
    (7, 256, 144, "bf16", False),        # ragged T
    (129, 2048, 272, "bf16", True),      # longest row of the warp-per-row quantiser (256 vectors)
    (300, 1024, 400, "f32", False),
    (33, 4096, 160, "bf16", False),      # block-per-row quantiser
])
def test_forward_qat_matches_separate_calls(bl, T, K, N, dtype, gain):
    """bitlinear_forward_qat == bitlinear_quant_weight + bitlinear_forward, bit for bit, and
    its codes / accumulators against the oracle."""
    li = synth.random_case(T, K, N, seed=300 + T, dtype=dtype, with_gain=gain)
    X, W = _gpu(li.X), _gpu(li.W)
    g = None if li.g is None else _gpu(li.g)
    fq = bl.bitlinear_forward_qat(X, W, g=g, want_acc=True)
    qw = bl.bitlinear_quant_weight(W)
    f = bl.bitlinear_forward(X, qw["wq_i8"], qw["gamma"], g=g, want_acc=True)
    torch.cuda.synchronize()
    for k in ("gamma", "wq_i8", "wq_bf16", "packed"):
        assert torch.equal(fq[k], qw[k]), k
    for k in ("y", "xq", "sx", "rinv", "xdq", "acc"):
        assert torch.equal(fq[k], f[k]), k
    g_gpu = float(fq["gamma"].item())
    ref = oracle.forward(li.X, li.W, g=li.g, rinv=np_(fq["rinv"]), gamma=g_gpu, out_dtype=dtype)
    assert np.array_equal(np_(fq["wq_i8"]), ref["wq"])
    assert np.array_equal(np_(fq["xq"]), ref["xq"])
    assert np.array_equal(np_(fq["acc"]), ref["acc"])


_WORKLOAD_CACHE = {}


def _workload_layer(workload, layer):
    """One layer's inputs; a workload's draws are made once per test session (they are
    sequential, so layer i needs every earlier layer's draws)."""
    if workload not in _WORKLOAD_CACHE:
        _WORKLOAD_CACHE.clear()
        _WORKLOAD_CACHE[workload] = synth.workload_inputs(workload)
    return _WORKLOAD_CACHE[workload][layer]


@pytest.mark.parametrize("workload,layer", [("square", 0), ("mlp7b", 0), ("mlp7b", 1)] +
                         [("layer7b", i) for i in range(7)])
def test_workload_full_size(bl, workload, layer):
    """Full-size layers of the benchmark workloads (square 2048->2048 x 4096 tokens; the
    7B MLP's 4096->11008 and 11008->4096 x 8192 tokens with Student-t weights; all seven
    projections of the 7B layer at 16384 tokens: q, k, v, o 4096->4096, gate and up
    4096->11008, down 11008->4096), bf16: every code exact, sampled rows of the
    accumulators / outputs / gradients against the oracle, the rest through exact
    properties."""
    li = _workload_layer(workload, layer)
    dt, g_gpu, wq, f, dX, dW, dg = _layer_case(bl, li)
    T, K = li.X.shape
    r_gpu = np_(f["rinv"])
    assert ulp_diff(r_gpu, oracle.rmsnorm_rinv(li.X, 1e-6)).max() <= 1
    xq, s, xdq = oracle.act_quant(li.X, r_gpu, None)
    assert np.array_equal(np_(f["xq"]), xq)
    assert np.array_equal(np_(f["sx"]), s)
    assert np.array_equal(np_(f["xdq"]), oracle.round_bf16(xdq))
    # zero fraction of the ternary codes (P3 §6: healthy 30-50%; closed forms 0.31006 for
    # Gaussian and 0.38019 for Student-t3 weights, the latter with a wider band because the
    # sample mean of |t3| converges slowly)
    zf = float(np.mean(wq == 0))
    if synth.WORKLOADS[workload].w_dist == "normal":
        assert abs(zf - 0.31006) < 0.002
    else:
        assert abs(zf - 0.38019) < 0.004
    rows = sample_rows(T, 32, seed=1)
    acc_o = oracle.int_gemm(xq, wq, rows=rows)
    assert np.array_equal(np_(f["acc"])[rows], acc_o)
    assert np.array_equal(np_(f["y"])[rows], oracle.round_bf16(oracle.linear_epilogue(acc_o, g_gpu, s[rows])))
    # backward on sampled rows (dX) and sampled weight rows (dW)
    xdq_saved = f32_of(f["xdq"])
    dxh = oracle.grad_input_hat(li.dY, wq, g_gpu, rows=rows)
    dX_o, _ = oracle.rmsnorm_backward(li.X, r_gpu, None, dxh, rows=rows, want_dg=False)
    assert max_rel_err(np_(dX)[rows], dX_o) <= TOL["bf16"]
    wrows = sample_rows(li.W.shape[0], 16, seed=2)
    dW_o = oracle.grad_weight(li.dY, xdq_saved, wrows=wrows)
    assert max_rel_err(np_(dW)[wrows], dW_o) <= TOL["bf16"]
    # dW over every entry: against an fp32 torch contraction of the same exact operands
    dW_t = li.dY.to(DEV).float().t() @ f["xdq"].float()
    assert max_rel_err(np_(dW), dW_t.cpu().numpy()) <= 1e-4


# ------------------------------------------------------------------------------------
# decode GEMV over packed weights
# ------------------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(48, 64), (400, 192), (1024, 8192), (272, 4096), (160, 704), (4800, 704)])
@pytest.mark.parametrize("B", [1, 2, 4, 5, 8, 9, 16])
def test_gemv_parity(bl, N, K, B):
    W, x = synth.decode_inputs(B, N, K, seed=N + K + B)
    qw = bl.bitlinear_quant_weight(_gpu(W))
    aq = bl.bitlinear_act_quant(_gpu(x), apply_rmsnorm=False, want_xdq=False)
    y, acc = bl.ternary_gemv(qw["packed"], qw["gamma"], K, aq["xq"], aq["sx"], want_acc=True)
    torch.cuda.synchronize()
    g = float(qw["gamma"].item())
    acc_o, y_o = oracle.gemv(np_(qw["packed"]), g, K, np_(aq["xq"]), np_(aq["sx"]))
    assert np.array_equal(np_(acc), acc_o)
    assert np.array_equal(np_(y), y_o)


def test_gemv_reserved_code_decodes_to_zero(bl):
    rng = np.random.default_rng(4)
    N, K, B = 64, 128, 3
    packed = rng.integers(0, 256, size=(N, K // 4)).astype(np.uint8)   # includes 11 codes
    xq = rng.integers(-127, 128, size=(B, K)).astype(np.int8)
    s = np.full(B, 50.0, dtype=np.float32)
    y, acc = bl.ternary_gemv(_gpu(torch.from_numpy(packed)), _gpu(torch.tensor([0.02])), K,
                             _gpu(torch.from_numpy(xq)), _gpu(torch.from_numpy(s)), want_acc=True)
    acc_o, _ = oracle.gemv(packed, 0.02, K, xq, s)
    assert np.array_equal(np_(acc), acc_o)


def test_gemv_extreme_magnitudes(bl):
    """Longest rows (K = 65536), all codes -1 / +1 / reserved, activations at -128 and 127."""
    N, K, B = 64, 65536, 2                           # B * K bytes of activations fill shared memory
    rows = []
    for r in range(N):
        code = (2, 1, 3, 0)[r % 4]                   # -1, +1, reserved, 0
        byte = code | (code << 2) | (code << 4) | (code << 6)
        rows.append(np.full(K // 4, byte, dtype=np.uint8))
    packed = np.stack(rows)
    xq = np.empty((B, K), dtype=np.int8)
    xq[0] = -128
    xq[1] = np.where(np.arange(K) % 2 == 0, -128, 127)
    s = np.array([1.0, 0.25], dtype=np.float32)
    y, acc = bl.ternary_gemv(_gpu(torch.from_numpy(packed)), _gpu(torch.tensor([0.75])), K,
                             _gpu(torch.from_numpy(xq)), _gpu(torch.from_numpy(s)), want_acc=True)
    torch.cuda.synchronize()
    acc_o, y_o = oracle.gemv(packed, 0.75, K, xq, s)
    assert int(np.abs(acc_o).max()) == 128 * K
    assert np.array_equal(np_(acc), acc_o)
    assert np.array_equal(np_(y), y_o)


def test_decode_workload_full_size(bl):
    """W 28672 x 8192 packed, batch 1, 4, 16: every accumulator against the oracle."""
    for B in (1, 4, 16):
        W, x = synth.decode_inputs(B)
        qw = bl.bitlinear_quant_weight(_gpu(W), want_bf16=False)
        aq = bl.bitlinear_act_quant(_gpu(x), apply_rmsnorm=False, want_xdq=False)
        y, acc = bl.ternary_gemv(qw["packed"], qw["gamma"], 8192, aq["xq"], aq["sx"], want_acc=True)
        torch.cuda.synchronize()
        if B == 1:
            g, wq, _ = _check_quant_weight(bl, W)
            assert abs(float(np.mean(wq == 0)) - 0.31006) < 0.001
        acc_o, y_o = oracle.gemv(np_(qw["packed"]), float(qw["gamma"].item()), 8192, np_(aq["xq"]), np_(aq["sx"]))
        assert np.array_equal(np_(acc), acc_o)
        assert np.array_equal(np_(y), y_o)
